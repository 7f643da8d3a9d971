"""The FMA-pipe 2^x of the attention kernel (exp2_fma2 in csrc/jca_device.cuh), replayed step by
step in fp32 on the CPU and held to the error bound of its minimax fit, against numpy's exp2."""

import re
from pathlib import Path

import numpy as np
import pytest

SRC = Path(__file__).resolve().parents[1] / "candidate_isolated_jagged_b200" / "csrc" / "jca_device.cuh"


def _coefficients():
    text = SRC.read_text()
    m = re.search(r"kC1 = ([0-9a-fx.p+-]+)f, kC2 = ([0-9a-fx.p+-]+)f, kC3 = ([0-9a-fx.p+-]+)f", text)
    assert m, "exp2_fma2 coefficients not found"
    return [np.float32(float.fromhex(v)) for v in m.groups()]


def _fma32(a, b, c):
    # fp32 fused multiply-add: the product of two fp32 values is exact in fp64, so one rounding
    # of the fp64 sum to fp32 matches the hardware except for rare double-rounding ties.
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_fma2_replay(x):
    """The device steps: clamp, round by adding 1.5 * 2^23, reduce, Horner, add n to exponent."""
    c1, c2, c3 = _coefficients()
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-127.0))
    k = np.float32(1.5 * 2 ** 23)
    t = (x + k).astype(np.float32)
    n = (t - k).astype(np.float32)
    f = _fma32(n, np.float32(-1.0), x)
    p = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    p = _fma32(p, f, np.full_like(f, c1))
    p = _fma32(p, f, np.full_like(f, np.float32(1.0)))
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_coefficients_match_the_fit_error_bound():
    # The source's fp32 coefficients must reach (within rounding) the minimax error of a fresh fit.
    from candidate_isolated_jagged_b200.exp2_poly_fit import fit
    _, err = fit()
    assert err < 1.1e-4
    c1, c2, c3 = (np.float64(c) for c in _coefficients())
    f = np.linspace(-0.5, 0.5, 20001)
    rel = np.abs((1 + f * (c1 + f * (c2 + f * c3))) / np.exp2(f) - 1)
    assert rel.max() < err * 1.02 + 1e-7


def test_relative_error_over_the_softmax_range():
    # Arguments of the softmax: s * scale - m lies in [-inf, 8] (lazy rescaling allows up to +8).
    x = np.concatenate([np.linspace(-126.0, 8.0, 400001, dtype=np.float32),
                        np.float32([0.0, -0.5, 0.5, -1.0, 1.0, 7.999, -125.5])])
    got = exp2_fma2_replay(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1)
    assert rel.max() < 1.2e-4, rel.max()
    assert np.all(got > 0)


def test_exact_values_and_underflow():
    got = exp2_fma2_replay(np.float32([0.0, 1.0, 2.0, -1.0, 8.0]))
    assert got.tolist() == [1.0, 2.0, 4.0, 0.5, 256.0]      # p(0) = 1 exactly
    z = exp2_fma2_replay(np.float32([-np.inf, -127.0, -200.0, -1e30]))
    assert np.all(z == 0.0) and not np.any(np.signbit(z))   # masked keys contribute exactly +0
    tiny = exp2_fma2_replay(np.linspace(-127.0, -126.0, 1001, dtype=np.float32))
    assert np.all(tiny >= 0) and np.all(tiny < 2.0 ** -125)  # never negative, never large


@pytest.mark.parametrize("lo,hi", [(-30.0, 0.0), (-8.0, 8.0)])
def test_monotone_on_dense_grid(lo, hi):
    x = np.linspace(lo, hi, 200001, dtype=np.float32)
    y = exp2_fma2_replay(x)
    # the reduction restarts the polynomial at every half-integer; steps there stay within the
    # error bound, so the sequence is monotone up to that bound
    assert np.all(np.diff(y.astype(np.float64)) >= -2.5e-4 * y[1:].astype(np.float64))
