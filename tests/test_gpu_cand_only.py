"""GPU parity of cand_only_attn_fwd (candidate queries over frozen history K/V plus their own K/V)
against the oracle, its equality with the candidate rows of the full op, and the two candidate-only
workloads at full size on sampled rows, plus key counts on and around the 128-key tile edges,
history padding at the ends of a key interval, and many short users over several head counts."""

import numpy as np
import pytest
import torch

import oracle
import synth
from candidate_isolated_jagged_b200 import jca
from helpers import CandOnlyRun, FullRun, assert_close, assert_close_bf16, dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [16, 32, 64, 128])
def test_small_cand_only(d):
    cb = synth.custom_cand_only([0, 7, 128, 129, 300], [3, 0, 200, 1, 130], H=2, d=d, seed=d)
    r = CandOnlyRun(cb)
    ref = r.reference()
    assert_close(r.run(), ref, f"cand-only d={d}")
    assert_close_bf16(r.run(out_fp32=False), ref, f"cand-only bf16 d={d}")


def test_cand_only_history_padding():
    cb = synth.custom_cand_only([5, 140, 0, 33], [2, 150, 4, 1], H=3, d=64, seed=2)
    rng = np.random.default_rng(0)
    hseg = (rng.random(cb.Th) > 0.25).astype(np.int8)
    r = CandOnlyRun(cb, hist_seg=hseg)
    assert_close(r.run(), r.reference(), "cand-only with history padding")


@pytest.mark.parametrize("d", [32, 128])
def test_cand_only_equals_full_candidate_rows(d):
    b = synth.custom_batch([60, 0, 250], prefix=[2, 0, 4], n_cand=[33, 5, 140], H=2, d=d, seed=5)
    full = FullRun(b)
    out_full = full.run()
    off = full.off_np
    hist_idx, cand_idx, hl, cc = [], [], [], []
    for u in range(b.B):
        s, e, cs = int(off[u]), int(off[u + 1]), int(off[u] + b.cand_start[u])
        hist_idx += range(s, cs)
        cand_idx += range(cs, e)
        hl.append(cs - s)
        cc.append(e - cs)
    hi = torch.tensor(hist_idx, dtype=torch.long, device=dev())
    ci = torch.tensor(cand_idx, dtype=torch.long, device=dev())
    coff = torch.tensor(oracle.offsets_from_lengths(cc), device=dev())
    hoff = torch.tensor(oracle.offsets_from_lengths(hl), device=dev())
    got = jca.cand_only(full.q[ci], full.k[ci], full.v[ci], coff, full.k[hi], full.v[hi], hoff,
                        out_fp32=True)
    if d < 64:
        # same key tiles, same per-row arithmetic: identical bits
        assert torch.equal(got, out_full[ci])
    else:
        # Heads of 64 or more take each candidate's own term through the tensor core in the
        # candidate-only layer (its weight rounded to bf16 as a PV operand, like every other
        # weight), the full layer on CUDA cores in fp32: the same within the parity bar, and both
        # against the oracle.
        assert_close(got, out_full[ci].cpu().double().numpy(),
                     f"cand-only vs full candidate rows d={d}")
        ref = full.reference()
        assert_close(got, np.asarray(ref)[cand_idx], f"cand-only d={d}")


def test_cand_only256_sampled():
    cb = synth.cand_only256()
    r = CandOnlyRun(cb)
    out = r.run()
    rng = np.random.default_rng(4)
    rows = np.unique(np.concatenate([rng.integers(0, cb.Nc, 400), r.coff_np[:-1],
                                     r.coff_np[1:] - 1, np.arange(512, 1024)]))
    assert_close(out[torch.tensor(rows, device=dev())], r.reference(cand_rows=rows),
                 "cand_only256 sampled")


def test_retrieval_sampled():
    cb = synth.retrieval()
    r = CandOnlyRun(cb)
    out = r.run()
    rng = np.random.default_rng(6)
    rows = np.unique(np.concatenate([rng.integers(0, cb.Nc, 600), r.coff_np[:-1],
                                     r.coff_np[1:] - 1]))
    assert_close(out[torch.tensor(rows, device=dev())], r.reference(cand_rows=rows),
                 "retrieval sampled")


def test_cand_only_bad_history_segment():
    cb = synth.custom_cand_only([4, 4], [2, 2], H=1, d=16, seed=1)
    hseg = np.array([1, 1, -1, 1, 1, 0, 1, 1], dtype=np.int8)
    r = CandOnlyRun(cb, hist_seg=hseg)
    out = torch.full(r.cq.shape, 3.0, dtype=torch.float32, device=dev())
    st = jca.new_status(dev())
    jca.cand_only_attn_fwd(r.cq, r.ck, r.cv, r.coff, r.hk, r.hv, r.hoff, out, r.hseg, status=st)
    assert int(st.item()) == 5
    assert torch.all(out == 3.0)


@pytest.mark.parametrize("idx", [torch.int32, torch.int64])
@pytest.mark.parametrize("d", [16, 32, 64])
def test_cand_only_key_and_row_boundaries(d, idx):
    # key counts 0..600 on and around the 128-key tile edges; candidate counts on and around the
    # 128-row tile edges
    hist = [1, 2, 15, 16, 17, 127, 128, 129, 255, 256, 257, 0, 600]
    cands = [129, 1, 300, 128, 5, 256, 3, 127, 140, 700, 9, 4, 130]
    cb = synth.custom_cand_only(hist, cands, H=3, d=d, seed=30 + d)
    r = CandOnlyRun(cb, idx=idx)
    ref = r.reference()
    out = r.run()
    assert_close(out, ref, f"cand-only boundaries d={d}")
    assert_close_bf16(r.run(out_fp32=False), ref, f"cand-only boundaries bf16 d={d}")
    assert torch.equal(out, r.run())   # the same bits every call


@pytest.mark.parametrize("d", [16, 32, 64])
def test_cand_only_history_holes_at_interval_ends(d):
    # padding rows inside the key interval are masked; padding at both ends of a 300-row history
    # shrinks its key interval to 256 keys
    hist = [40, 256, 200, 300, 3, 130]
    cands = [300, 77, 1000, 64, 260, 1]
    cb = synth.custom_cand_only(hist, cands, H=2, d=d, seed=40 + d)
    rng = np.random.default_rng(d)
    hseg = (rng.random(cb.Th) > 0.25).astype(np.int8)
    off = oracle.offsets_from_lengths(hist)
    s3 = int(off[3])
    hseg[s3:s3 + 300] = 1
    hseg[s3:s3 + 20] = 0
    hseg[s3 + 276:s3 + 300] = 0
    r = CandOnlyRun(cb, hist_seg=hseg)
    assert_close(r.run(), r.reference(), f"cand-only with history padding d={d}")


@pytest.mark.parametrize("H,d", [(2, 32), (5, 32), (6, 16), (3, 64)])
def test_cand_only_many_short_users(H, d):
    # 150 short users with few candidates each: many items of a single key tile and a single
    # query tile, over several head counts
    rng = np.random.default_rng(7 + H)
    hist = rng.integers(1, 257, 150)
    cands = rng.integers(1, 300, 150)
    cb = synth.custom_cand_only(hist, cands, H=H, d=d, seed=8)
    r = CandOnlyRun(cb)
    assert_close(r.run(), r.reference(), f"cand-only, 150 users, H={H}, d={d}")
