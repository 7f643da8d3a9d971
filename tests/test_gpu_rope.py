"""GPU parity of the right-anchored RoPE kernels against the oracle (oracle/rope.py): positions
bit-exact, rotated rows within one bf16 ulp, and attention on rotated queries and keys within the
usual attention tolerance, plus the candidate-order invariance the pages state. The fused entry
point (jagged_cand_attn_rope_fwd, tiles rotated inside the attention kernel) is checked against the
oracle under the same bars, and against the pre-pass path: history rows bit-identical (the same
rotated bf16 tiles, the same MMAs), candidate rows within 1e-5 (their own score is summed in
another order)."""

import numpy as np
import pytest
import torch

import oracle
import synth
from candidate_isolated_jagged_b200 import jca
from helpers import CandOnlyRun, FullRun, assert_close, dev

pytestmark = pytest.mark.gpu

IDX = [torch.int32, torch.int64]


def _cases():
    rng = np.random.default_rng(9)
    rl = rng.integers(0, 300, size=64)
    rl[::9] = 0
    cs = np.array([rng.integers(0, L + 1) for L in rl])
    valid = (rng.random(int(rl.sum())) > 0.2).astype(np.uint8)
    n = synth.users256_history_lengths(0)
    return {
        "worked": ([6, 3, 4], [3, 1, 0], None),
        "random_holes": (rl, cs, valid),
        "users256": (n + 4 + 64, n + 4, None),
    }


@pytest.mark.parametrize("idx", IDX)
@pytest.mark.parametrize("name", ["worked", "random_holes", "users256"])
@pytest.mark.parametrize("history_end", [0, 4096, -7])
def test_positions_bit_exact(idx, name, history_end):
    rl, cs, valid = _cases()[name]
    off_np = oracle.offsets_from_lengths(rl)
    seg_np = oracle.segment_ids(off_np, cs, valid)
    ref = oracle.right_anchored_positions(off_np, seg_np, history_end)
    pos = torch.full((seg_np.size,), 12345, dtype=torch.int32, device=dev())
    st = jca.new_status(dev())
    jca.jca_rope_positions(torch.tensor(seg_np, device=dev()), torch.tensor(off_np, dtype=idx,
                           device=dev()), pos, history_end, st)
    jca.check_status(st)
    assert np.array_equal(pos.cpu().numpy().astype(np.int64), ref)


def test_positions_bad_offsets():
    st = jca.new_status(dev())
    seg = torch.ones(6, dtype=torch.int8, device=dev())
    pos = torch.zeros(6, dtype=torch.int32, device=dev())
    jca.jca_rope_positions(seg, torch.tensor([0, 4, 3, 6], device=dev()), pos, 10, st)
    assert int(st.item()) == 2


def _within_one_ulp(got, ref, x):
    # One bf16 ulp of the result, plus the error of the fp32 cosine and sine relative to the
    # inputs' size (which matters only where the two terms of a*cos - b*sin cancel). The kernels
    # compose cos/sin(p theta) from the factors at 128 q and r (p = 128 q + r), each accurate to
    # about 2^-21 (fast intrinsics on an fp64-reduced argument); with the fp32 products of the
    # composition and of the rotation the bound is about 3 * 2^-21, under 2^-19.
    got = got.detach().to("cpu", torch.float64).numpy()
    x = x.to(torch.float64).numpy()
    half = x.shape[-1] // 2
    mag = np.abs(x[..., :half]) + np.abs(x[..., half:])
    mag = np.concatenate([mag, mag], axis=-1)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -126))) - 7)
    return np.abs(got - ref) <= ulp + 2.0 ** -19 * mag


@pytest.mark.parametrize("d", [16, 32, 64, 128])
@pytest.mark.parametrize("inplace", [False, True])
def test_rotation_within_one_ulp(d, inplace):
    g = torch.Generator().manual_seed(d)
    T, H = 1000, 3
    x = torch.randn(T, H, d, generator=g).to(torch.bfloat16)
    pos_np = np.concatenate([np.arange(-20, 480), np.random.default_rng(d).integers(0, 9000, 500)])
    ref = oracle.round_to_bf16(oracle.apply_rope(x, pos_np))
    xg = x.to(dev())
    out = xg if inplace else torch.empty_like(xg)
    jca.jca_apply_rope(xg, out, torch.tensor(pos_np, dtype=torch.int32, device=dev()))
    torch.cuda.synchronize()
    ok = _within_one_ulp(out, ref, x)
    assert ok.mean() == 1.0, f"{(~ok).sum()} elements off by more than one bf16 ulp"


def test_rotation_errors():
    x = torch.zeros(4, 1, 48, dtype=torch.bfloat16, device=dev())
    with pytest.raises(jca.JcaError):
        jca.jca_apply_rope(x, x, torch.zeros(4, dtype=torch.int32, device=dev()))
    x = torch.zeros(4, 1, 64, dtype=torch.bfloat16, device=dev())
    with pytest.raises(jca.JcaError):
        jca.jca_apply_rope(x, x, torch.zeros(4, dtype=torch.int32, device=dev()), base=1.0)


def _rope_full(b, history_end=1000):
    r = FullRun(b)
    pos = torch.empty(r.seg_np.size, dtype=torch.int32, device=dev())
    st = jca.new_status(dev())
    seg = torch.tensor(r.seg_np, device=dev())
    jca.jca_rope_positions(seg, r.off, pos, history_end, st)
    jca.jca_apply_rope(r.q, r.q, pos)
    jca.jca_apply_rope(r.k, r.k, pos)
    jca.check_status(st)
    out = r.run()
    pos_np = oracle.right_anchored_positions(r.off_np, r.seg_np, history_end)
    q = oracle.round_to_bf16(oracle.apply_rope(b.q, pos_np))
    k = oracle.round_to_bf16(oracle.apply_rope(b.k, pos_np))
    ref = oracle.jagged_cand_attn(q, k, b.v, r.off_np, r.seg_np, b.scale)
    return out, ref, r


@pytest.mark.parametrize("d", [32, 128])
def test_attention_with_rope(d):
    b = synth.custom_batch([0, 1, 127, 129, 300, 5], prefix=[0, 1, 2, 0, 4, 1],
                           n_cand=[3, 0, 64, 1, 130, 2], H=2, d=d, seed=d)
    out, ref, _ = _rope_full(b)
    assert_close(out, ref, f"attention with RoPE d={d}")


def test_attention_with_rope_and_padding():
    out, ref, _ = _rope_full(synth.three_users())
    assert_close(out, ref, "three users with RoPE")


def test_candidate_order_invariance_on_gpu():
    # Reversing one user's candidates (their q, k, v rows) reverses their outputs and changes no
    # other row: all candidates share one position and see no other candidate.
    b = synth.custom_batch([40, 200], prefix=2, n_cand=[7, 90], H=2, d=64, seed=11)
    out1, _, r = _rope_full(b)
    s, e = int(r.off_np[1]), int(r.off_np[2])
    cands = np.nonzero(r.seg_np[s:e] == -1)[0] + s
    perm = np.arange(b.q.shape[0])
    perm[cands] = cands[::-1]
    pt = torch.tensor(perm)
    b2 = synth.workloads.Batch(**{**b.__dict__, "q": b.q[pt], "k": b.k[pt], "v": b.v[pt]})
    out2, _, _ = _rope_full(b2)
    assert_close(out2[torch.tensor(perm, device=dev())], out1.cpu().numpy(), "candidate order",
                 max_abs=2e-3, rel_l2=1e-3)


def test_cand_only_with_rope():
    cb = synth.custom_cand_only([5, 140, 0, 33], [2, 150, 4, 1], H=2, d=64, seed=3)
    hend = 500
    hpos_np, cpos_np = oracle.cand_only_positions(oracle.offsets_from_lengths(cb.cand_counts),
                                                  oracle.offsets_from_lengths(cb.hist_lengths),
                                                  None, hend)
    r = CandOnlyRun(cb)
    hpos = torch.empty(cb.Th, dtype=torch.int32, device=dev())
    st = jca.new_status(dev())
    jca.jca_rope_positions(torch.ones(cb.Th, dtype=torch.int8, device=dev()), r.hoff, hpos, hend,
                           st)
    cpos = torch.full((cb.Nc,), hend, dtype=torch.int32, device=dev())
    jca.jca_apply_rope(r.hk, r.hk, hpos)
    jca.jca_apply_rope(r.cq, r.cq, cpos)
    jca.jca_apply_rope(r.ck, r.ck, cpos)
    jca.check_status(st)
    out = r.run()
    rq = oracle.round_to_bf16(oracle.apply_rope(cb.cq, cpos_np))
    rk = oracle.round_to_bf16(oracle.apply_rope(cb.ck, cpos_np))
    rhk = oracle.round_to_bf16(oracle.apply_rope(cb.hk, hpos_np))
    ref = oracle.cand_only_attn(rq, rk, cb.cv, r.coff_np, rhk, cb.hv, r.hoff_np, None, cb.scale)
    assert_close(out, ref, "cand-only with RoPE")


def _fused(b, history_end=1000, idx=torch.int64, out_fp32=True):
    r = FullRun(b, idx=idx)
    out = torch.full(b.q.shape, float("nan"), dtype=torch.float32 if out_fp32 else torch.bfloat16,
                     device=dev())
    st = jca.new_status(dev())
    jca.jagged_cand_attn_rope_fwd(r.q, r.k, r.v, out, r.off, r.cs, r.seg, history_end=history_end,
                                  status=st)
    torch.cuda.synchronize()
    jca.check_status(st, "rope fused")
    return out, r


FUSED = {
    "tiny": lambda: synth.tiny(),
    "holes_d32": lambda: synth.custom_batch([0, 7, 300, 129, 1], prefix=[2, 0, 4, 1, 0],
                                            n_cand=[5, 1, 140, 0, 3], H=3, d=32, seed=4,
                                            pad_hist_to=16),
    "three_users": lambda: synth.three_users(),
    "d128_edges": lambda: synth.custom_batch([0, 1, 127, 128, 129, 255, 300], prefix=[0, 1, 2, 0, 4, 1, 3],
                                             n_cand=[3, 0, 64, 1, 130, 2, 257], H=2, d=128, seed=12),
}


@pytest.mark.parametrize("history_end", [1000, 0, -300])
@pytest.mark.parametrize("name", list(FUSED))
def test_fused_rope_matches_oracle_and_prepass(name, history_end):
    b = FUSED[name]()
    out, r = _fused(b, history_end)
    pos_np = oracle.right_anchored_positions(r.off_np, r.seg_np, history_end)
    q = oracle.round_to_bf16(oracle.apply_rope(b.q, pos_np))
    k = oracle.round_to_bf16(oracle.apply_rope(b.k, pos_np))
    ref = oracle.jagged_cand_attn(q, k, b.v, r.off_np, r.seg_np, b.scale)
    assert_close(out, ref, f"fused rope {name}")
    # the caller's q and k are left unrotated
    assert torch.equal(r.q.cpu(), b.q) and torch.equal(r.k.cpu(), b.k)
    pre, ref2, _ = _rope_full(b, history_end)
    hist = torch.from_numpy(r.seg_np != -1).to(dev())
    assert torch.equal(out[hist], pre[hist])
    assert_close(out, pre.double().cpu().numpy(), f"fused vs pre-pass {name}", max_abs=1e-5,
                 rel_l2=1e-5)


@pytest.mark.parametrize("idx", IDX)
def test_fused_rope_bf16_output_and_index_types(idx):
    b = FUSED["holes_d32"]()
    out, r = _fused(b, 77, idx=idx, out_fp32=False)
    pos_np = oracle.right_anchored_positions(r.off_np, r.seg_np, 77)
    q = oracle.round_to_bf16(oracle.apply_rope(b.q, pos_np))
    k = oracle.round_to_bf16(oracle.apply_rope(b.k, pos_np))
    from helpers import assert_close_bf16
    assert_close_bf16(out, oracle.jagged_cand_attn(q, k, b.v, r.off_np, r.seg_np, b.scale),
                      "fused rope bf16")


def test_fused_rope_users256_sampled():
    """The 256-user workload with in-kernel RoPE (history_end 4096), in the launch configuration
    the benchmark times, checked on every row of eight users (an empty history, the 4096-token
    user, the median, the 200th longest and four more): users never interact, so the oracle runs
    on a batch of just those users."""
    b = synth.users256()
    out, r = _fused(b, 4096)
    order = np.argsort(b.hist_real)
    users = [0, 1, int(order[128]), int(order[200]), 5, 77, 130, 255]
    rows = np.concatenate([np.arange(r.off_np[u], r.off_np[u + 1]) for u in users])
    soff = oracle.offsets_from_lengths(b.row_lengths[users])
    sseg = r.seg_np[rows]
    pos_np = oracle.right_anchored_positions(soff, sseg, 4096)
    rt = torch.from_numpy(rows)
    q = oracle.round_to_bf16(oracle.apply_rope(b.q[rt], pos_np))
    k = oracle.round_to_bf16(oracle.apply_rope(b.k[rt], pos_np))
    ref = oracle.jagged_cand_attn(q, k, b.v[rt], soff, sseg, b.scale)
    assert_close(out[rt.to(dev())], ref, "fused rope users256 sampled")
