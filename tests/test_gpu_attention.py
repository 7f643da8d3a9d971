"""GPU parity of jagged_cand_attn_fwd against the fp64 oracle (max-abs 1e-2, rel-L2 5e-3 in fp32
output mode; bf16 output within 1e-2 + half a bf16 ulp), on the named workloads, edge cases and the
invariants the pages state."""

import numpy as np
import pytest
import torch

import oracle
import synth
from candidate_isolated_jagged_b200 import jca
from helpers import FullRun, assert_close, assert_close_bf16, dev, sample_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("idx", [torch.int32, torch.int64])
def test_tiny(idx):
    r = FullRun(synth.tiny(), idx)
    ref = r.reference()
    assert_close(r.run(out_fp32=True), ref, "tiny fp32")
    assert_close_bf16(r.run(out_fp32=False), ref, "tiny bf16")


def test_three_users_with_padding():
    r = FullRun(synth.three_users())
    ref = r.reference()
    out = r.run(out_fp32=True)
    assert_close(out, ref, "three_users")
    pad = np.nonzero(r.seg_np == 0)[0]
    assert pad.size == 10 and torch.all(out[torch.tensor(pad, device=dev())] == 0)
    assert_close_bf16(r.run(out_fp32=False), ref, "three_users bf16")


@pytest.mark.parametrize("d", [16, 32, 64, 128])
def test_head_dims_and_tile_edges(d):
    # lengths around tile boundaries; empty users; users without history; without candidates
    hist = [0, 1, 126, 127, 128, 129, 255, 256, 300, 0, 5]
    pre = [0, 1, 1, 2, 0, 4, 1, 0, 3, 0, 2]
    nc = [3, 0, 2, 1, 127, 0, 64, 1, 200, 0, 0]
    b = synth.custom_batch(hist, prefix=pre, n_cand=nc, H=3, d=d, seed=d)
    r = FullRun(b)
    assert_close(r.run(), r.reference(), f"edges d={d}")


def test_holes_anywhere():
    hist = [3, 40, 0, 2, 300]
    pre = [1, 2, 0, 1, 4]
    nc = [2, 130, 2, 0, 5]
    b0 = synth.custom_batch(hist, prefix=pre, n_cand=nc, H=2, d=64, seed=7)
    rng = np.random.default_rng(5)
    valid = (rng.random(b0.T) > 0.15).astype(np.uint8)
    b = synth.custom_batch(hist, prefix=pre, n_cand=nc, H=2, d=64, seed=7, valid_override=valid)
    r = FullRun(b)
    assert_close(r.run(), r.reference(), "holes")


def test_no_candidates_and_empty_batch():
    b = synth.custom_batch([5, 200, 1], prefix=2, n_cand=0, H=2, d=32, seed=3)
    r = FullRun(b)
    assert_close(r.run(), r.reference(), "no candidates")
    # B = 0, T = 0
    q = torch.empty(0, 2, 32, dtype=torch.bfloat16, device=dev())
    off = torch.zeros(1, dtype=torch.int64, device=dev())
    out = jca.attention(q, q, q, off, torch.zeros(0, dtype=torch.int64, device=dev()))
    assert out.shape == (0, 2, 32)


def test_single_key_closed_forms_exact():
    # candidates without any history output their own v (bf16 -> fp32 exactly)
    b = synth.custom_batch([0, 0], prefix=0, n_cand=[5, 130], H=2, d=64, seed=4)
    r = FullRun(b)
    out = r.run(out_fp32=True)
    assert torch.equal(out, r.v.float())


def test_users256_sampled_rows():
    b = synth.users256()
    r = FullRun(b)
    out = r.run(out_fp32=True)
    rows = sample_rows(r.off_np, per_user=2, seed=1)
    ref = r.reference_rows(rows)
    assert_close(out[torch.tensor(rows, device=dev())], ref, "users256 sampled")
    # the 4096-history user completely
    u = 1
    full = r.reference(users=[u])
    s, e = int(r.off_np[u]), int(r.off_np[u + 1])
    assert_close(out[s:e], full[s:e], "users256 user 1 (4096 history)")
    outb = r.run(out_fp32=False)
    assert_close_bf16(outb[torch.tensor(rows, device=dev())], ref, "users256 bf16")


def test_history_outputs_independent_of_candidates():
    b = synth.custom_batch([100, 300], prefix=2, n_cand=[40, 200], H=2, d=128, seed=9)
    r = FullRun(b)
    base = r.run()
    q2, k2, v2 = r.q.clone(), r.k.clone(), r.v.clone()
    g = torch.Generator().manual_seed(1)
    cand = torch.tensor(np.nonzero(r.seg_np == -1)[0], device=dev())
    for t in (q2, k2, v2):
        t[cand] = torch.randn(len(cand), 2, 128, generator=g).to(torch.bfloat16).to(dev())
    out = jca.attention(q2, k2, v2, r.off, r.cs, None, out_fp32=True)
    hist = torch.tensor(np.nonzero(r.seg_np == 1)[0], device=dev())
    assert torch.equal(out[hist], base[hist])


def test_candidate_permutation_invariance():
    b = synth.custom_batch([150], prefix=2, n_cand=90, H=2, d=64, seed=12)
    r = FullRun(b)
    base = r.run()
    cs = int(b.cand_start[0])
    perm = torch.cat([torch.arange(cs), cs + torch.randperm(90, generator=torch.Generator().manual_seed(3))])
    permd = perm.to(dev())
    out = jca.attention(r.q[permd], r.k[permd], r.v[permd], r.off, r.cs, None, out_fp32=True)
    assert_close(out, base[permd].cpu().double().numpy(), "permuted candidates", max_abs=1e-5,
                 rel_l2=1e-6)


def test_data_errors_leave_output_untouched():
    b = synth.tiny()
    r = FullRun(b)
    out = torch.full(r.q.shape, 7.0, dtype=torch.float32, device=dev())
    st = jca.new_status(dev())
    bad_cs = torch.tensor([3, 60, 2], dtype=torch.int64, device=dev())
    jca.jagged_cand_attn_fwd(r.q, r.k, r.v, out, r.off, bad_cs, None, status=st)
    assert int(st.item()) == 3
    assert torch.all(out == 7.0)
    st.zero_()
    bad_off = torch.tensor([0, 6, 5, 20], dtype=torch.int64, device=dev())
    jca.jagged_cand_attn_fwd(r.q, r.k, r.v, out, bad_off, r.cs, None, status=st)
    assert int(st.item()) == 2
    assert torch.all(out == 7.0)


def test_pipeline_wait_timeout_is_recoverable():
    """The failure path without a GPU fault: a bounded wait that nothing completes gives up after
    its limit and records JCA_STATUS_TIMEOUT; the status word then stops later calls that share it,
    and the context keeps working for calls with a fresh status word."""
    st = jca.new_status(dev())
    jca.jca_selftest_wait_timeout(st)
    torch.cuda.synchronize()
    assert int(st.item()) == 16
    assert "timed out" in jca.status_string(16)
    b = synth.tiny()
    r = FullRun(b)
    out = torch.full(b.q.shape, 7.0, dtype=torch.float32, device=dev())
    jca.jagged_cand_attn_fwd(r.q, r.k, r.v, out, r.off, r.cs, r.seg, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 16 and bool((out == 7.0).all())   # nothing written after an error
    assert_close(r.run(out_fp32=True), r.reference(), "after a timeout")
