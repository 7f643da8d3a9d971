"""GPU parity of UG-Sep's masked cross-attention (ug_masked_cross_attn_fwd) against the oracle
(oracle/ug_sep.py): the first c_u outputs of a sample read only its first n_u inputs, the others
read all T_in inputs, and the residual is added.

Covered: packs of several samples with a ragged last pack, token counts that do not divide 128,
one sample per pack at the 128-token limit, head sizes 16-128, several heads, bf16 and fp32
outputs, with and without a residual; the degenerate cases (no U output, only U outputs, no U
input, no input at all, one token); U outputs bit-identical when the G inputs change; a preset
status word; the residual updated in place; and the 16,384-sample workload the benchmark times,
on sampled samples."""

import numpy as np
import pytest
import torch

import oracle.ug_sep as ou
import synth
from candidate_isolated_jagged_b200 import jca
from helpers import assert_close, assert_close_bf16, dev

pytestmark = pytest.mark.gpu


def _run(b, out_fp32=True, residual=True, status=None):
    out = torch.full(b.q.shape, float("nan"),
                     dtype=torch.float32 if out_fp32 else torch.bfloat16, device=dev())
    st = jca.new_status(dev()) if status is None else status
    res = b.residual.to(dev()) if (residual and b.residual is not None) else None
    jca.ug_masked_cross_attn_fwd(b.q.to(dev()), b.k.to(dev()), b.v.to(dev()), out, b.c_u, b.n_u,
                                 residual=res, status=st)
    torch.cuda.synchronize()
    if status is None:
        jca.check_status(st, "ug_masked_cross_attn_fwd")
    return out


def _ref(b, residual=True, samples=None):
    return ou.ug_cross_attn(b.q, b.k, b.v, b.c_u, b.n_u, b.scale,
                            residual=b.residual if residual else None, samples=samples)


SHAPES = [
    # B, T_out, T_in, c_u, n_u, H, d
    (37, 16, 32, 8, 16, 1, 128),     # 4 samples per pack, last pack holds one sample
    (50, 7, 13, 3, 5, 2, 64),        # 9 per pack: 63 query rows, 117 keys rounded to 128
    (33, 16, 32, 8, 16, 3, 32),
    (20, 5, 9, 2, 4, 2, 16),
    (6, 128, 128, 64, 100, 2, 128),  # one sample per pack, the token limit on both sides
    (5, 100, 24, 30, 10, 1, 64),     # one sample per pack, few keys (trimmed MMA N)
    (9, 1, 1, 1, 1, 1, 16),          # one token in, one out
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_ug_shapes(shape):
    B, To, Ti, cu, nu, H, d = shape
    b = synth.custom_ug(B, To, Ti, cu, nu, H, d, seed=B + To)
    assert_close(_run(b), _ref(b), f"ug {shape}")


@pytest.mark.parametrize("shape", SHAPES[:3], ids=lambda s: "x".join(map(str, s)))
def test_ug_bf16_and_no_residual(shape):
    B, To, Ti, cu, nu, H, d = shape
    b = synth.custom_ug(B, To, Ti, cu, nu, H, d, seed=7 * B)
    assert_close_bf16(_run(b, out_fp32=False), _ref(b), f"ug bf16 {shape}")
    assert_close(_run(b, residual=False), _ref(b, residual=False), f"ug no residual {shape}")


@pytest.mark.parametrize("cu,nu", [(0, 7), (12, 40), (5, 0), (12, 0), (0, 0)])
def test_ug_degenerate_masks(cu, nu):
    b = synth.custom_ug(11, 12, 40, cu, nu, 2, 64, seed=cu * 100 + nu)
    assert_close(_run(b), _ref(b), f"ug c_u={cu} n_u={nu}")


@pytest.mark.parametrize("out_fp32", [True, False])
def test_ug_no_inputs(out_fp32):
    """T_in = 0: every output sees no key, so the output is the residual (or 0)."""
    b = synth.custom_ug(7, 5, 0, 2, 0, 2, 32, seed=3)
    got = _run(b, out_fp32=out_fp32)
    assert torch.equal(got.float().cpu(), b.residual.float())
    got0 = _run(b, out_fp32=out_fp32, residual=False)
    assert torch.count_nonzero(got0).item() == 0


def test_ug_u_outputs_ignore_g_inputs():
    cu, nu = 8, 16
    b = synth.custom_ug(64, 16, 32, cu, nu, 2, 128, seed=21)
    base = _run(b)
    other = synth.custom_ug(64, 16, 32, cu, nu, 2, 128, seed=22)
    b.k[:, nu:] = other.k[:, nu:]
    b.v[:, nu:] = other.v[:, nu:]
    moved = _run(b)
    assert torch.equal(moved[:, :cu], base[:, :cu])
    assert (moved[:, cu:] - base[:, cu:]).abs().max().item() > 1e-3


def test_ug_preset_status_is_a_no_op():
    b = synth.custom_ug(8, 16, 32, 8, 16, 1, 64, seed=5)
    st = jca.new_status(dev())
    st.fill_(3)
    got = _run(b, status=st)
    assert torch.isnan(got).all()
    assert int(st.item()) == 3


@pytest.mark.parametrize("out_fp32", [False, True])
def test_ug_sep16k_sampled(out_fp32):
    """The benchmark's workload (16,384 samples, 32 -> 16 tokens, 16 / 8 U-tokens, one head of
    128), in the launch configuration the benchmark times; 96 samples (the first, the last, the
    edges of the first packs and random ones) are computed by the oracle."""
    b = synth.ug_sep16k()
    got = _run(b, out_fp32=out_fp32)
    rng = np.random.default_rng(0)
    samples = sorted(set([0, 1, 2, 3, 4, 5, 147, 148, b.B - 2, b.B - 1]) |
                     set(rng.choice(b.B, 86, replace=False).tolist()))
    ref = _ref(b, samples=samples)[samples]
    got_s = got[samples]
    if out_fp32:
        assert_close(got_s, ref, "ug_sep16k fp32")
    else:
        assert_close_bf16(got_s, ref, "ug_sep16k bf16")
    assert bool(torch.isfinite(got.float()).all())


def test_ug_in_place_residual():
    """out may be the residual tensor itself (bf16): Y = X + R in place."""
    b = synth.custom_ug(37, 16, 32, 8, 16, 2, 64, seed=31)
    x = b.residual.to(dev()).clone()
    st = jca.new_status(dev())
    jca.ug_masked_cross_attn_fwd(b.q.to(dev()), b.k.to(dev()), b.v.to(dev()), x, b.c_u, b.n_u,
                                 residual=x, status=st)
    torch.cuda.synchronize()
    jca.check_status(st, "ug in place")
    assert_close_bf16(x, _ref(b), "ug in place")
