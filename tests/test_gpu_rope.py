"""GPU parity of the right-anchored RoPE kernels against the oracle (oracle/rope.py): positions
bit-exact, rotated rows within one bf16 ulp, and attention on rotated queries and keys within the
usual attention tolerance, plus the candidate-order invariance the pages state."""

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
    # One bf16 ulp of the result, plus the fp32 rounding of a*cos - b*sin relative to the
    # inputs' size (which matters only where the two terms cancel).
    got = got.detach().to("cpu", torch.float64).numpy()
    x = x.to(torch.float64).numpy()
    half = x.shape[-1] // 2
    mag = np.abs(x[..., :half]) + np.abs(x[..., half:])
    mag = np.concatenate([mag, mag], axis=-1)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -126))) - 7)
    return np.abs(got - ref) <= ulp + 2.0 ** -22 * mag


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
