"""GPU parity of cand_only_attn_fwd (candidate queries over frozen history K/V plus their own K/V)
against the oracle, its equality with the candidate rows of the full op, and the two candidate-only
workloads at full size on sampled rows."""

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


def test_cand_only_equals_full_candidate_rows():
    b = synth.custom_batch([60, 0, 250], prefix=[2, 0, 4], n_cand=[33, 5, 140], H=2, d=128, seed=5)
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
    # same key tiles, same per-row arithmetic: identical bits
    assert torch.equal(got, out_full[ci])


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
