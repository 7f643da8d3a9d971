"""Pins of UG-Sep's masked cross-attention oracle (oracle/ug_sep.py).

What fixes the oracle, besides its own code (UG-Sep page, section 分离残差连接):
- library routine: with no U output (c_u = 0) it is plain cross-attention, torch's SDPA in fp64;
  a U output equals SDPA over the first n_u inputs only, a G output SDPA over all inputs;
- the page's point: U outputs do not change when the G inputs change (U-token reusability),
  while G outputs do;
- closed forms: n_u = 1 makes every U output equal to the first input's value, n_u = 0 makes it 0
  (plus the residual);
- brute force: a pure-Python triple loop (math.exp) on a tiny case;
- planted mistakes in the mask (an off-by-one at the U/G boundary, the mask on the wrong rows,
  the roles swapped) fail the checks above.
"""

import math

import numpy as np
import pytest
import torch

import oracle.ug_sep as ou
import synth


def _sdpa(q, k, v, scale):
    """fp64 SDPA of one sample: q [Tq, H, d], k/v [Tk, H, d] -> [Tq, H, d]."""
    qh, kh, vh = (t.double().permute(1, 0, 2).unsqueeze(0) for t in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(qh, kh, vh, scale=scale)
    return out[0].permute(1, 0, 2).numpy()


@pytest.mark.parametrize("seed", [0, 1])
def test_no_u_outputs_is_plain_cross_attention(seed):
    b = synth.custom_ug(3, 5, 9, 0, 4, 2, 16, seed=seed, residual=False)
    got = ou.ug_cross_attn(b.q, b.k, b.v, 0, 4, b.scale)
    for s in range(b.B):
        assert np.max(np.abs(got[s] - _sdpa(b.q[s], b.k[s], b.v[s], b.scale))) < 1e-12


@pytest.mark.parametrize("c_u,n_u", [(2, 3), (4, 1), (5, 9), (3, 8)])
def test_u_rows_read_only_u_inputs(c_u, n_u):
    b = synth.custom_ug(2, 5, 9, c_u, n_u, 2, 16, seed=c_u * 10 + n_u, residual=False)
    got = ou.ug_cross_attn(b.q, b.k, b.v, c_u, n_u, b.scale)
    for s in range(b.B):
        ref_u = _sdpa(b.q[s, :c_u], b.k[s, :n_u], b.v[s, :n_u], b.scale)
        assert np.max(np.abs(got[s, :c_u] - ref_u)) < 1e-12
        if c_u < b.T_out:
            ref_g = _sdpa(b.q[s, c_u:], b.k[s], b.v[s], b.scale)
            assert np.max(np.abs(got[s, c_u:] - ref_g)) < 1e-12


def test_u_outputs_ignore_g_inputs():
    c_u, n_u = 3, 4
    b = synth.custom_ug(4, 6, 10, c_u, n_u, 2, 16, seed=5, residual=False)
    base = ou.ug_cross_attn(b.q, b.k, b.v, c_u, n_u, b.scale)
    other = synth.custom_ug(4, 6, 10, c_u, n_u, 2, 16, seed=6, residual=False)
    k2, v2 = b.k.clone(), b.v.clone()
    k2[:, n_u:] = other.k[:, n_u:]
    v2[:, n_u:] = other.v[:, n_u:]
    moved = ou.ug_cross_attn(b.q, k2, v2, c_u, n_u, b.scale)
    assert np.array_equal(moved[:, :c_u], base[:, :c_u])
    assert np.max(np.abs(moved[:, c_u:] - base[:, c_u:])) > 1e-3


def test_closed_forms():
    b = synth.custom_ug(3, 4, 7, 2, 1, 2, 16, seed=9)
    got = ou.ug_cross_attn(b.q, b.k, b.v, 2, 1, b.scale)
    v0 = b.v[:, 0].double().numpy()
    for i in range(2):
        assert np.array_equal(got[:, i], v0)      # one U input: its value, exactly
    got0 = ou.ug_cross_attn(b.q, b.k, b.v, 2, 0, b.scale, residual=b.residual)
    res = b.residual.double().numpy()
    assert np.array_equal(got0[:, :2], res[:, :2])  # no U input: 0, plus the residual
    plain = ou.ug_cross_attn(b.q, b.k, b.v, 2, 0, b.scale)
    assert np.array_equal(got0[:, 2:], plain[:, 2:] + res[:, 2:])


def test_matches_brute_force():
    c_u, n_u = 2, 3
    b = synth.custom_ug(2, 4, 5, c_u, n_u, 2, 8, seed=3)
    got = ou.ug_cross_attn(b.q, b.k, b.v, c_u, n_u, b.scale, residual=b.residual)
    q, k, v, r = (t.double().tolist() for t in (b.q, b.k, b.v, b.residual))
    for s in range(b.B):
        for i in range(b.T_out):
            keys = range(n_u) if i < c_u else range(b.T_in)
            for h in range(b.H):
                sc = [b.scale * math.fsum(x * y for x, y in zip(q[s][i][h], k[s][j][h]))
                      for j in keys]
                top = max(sc)
                w = [math.exp(x - top) for x in sc]
                tot = math.fsum(w)
                for c in range(b.d):
                    ref = math.fsum(wj / tot * v[s][j][h][c] for wj, j in zip(w, keys))
                    assert abs(got[s, i, h, c] - (ref + r[s][i][h][c])) < 1e-12


def test_pair_count():
    assert ou.ug_pairs(16, 32, 8, 16) == int(ou.ug_mask(16, 32, 8, 16).sum()) == 8 * 16 + 8 * 32
    assert ou.ug_pairs(5, 9, 0, 4) == 45
    assert ou.ug_pairs(5, 9, 5, 0) == 0


def test_planted_mask_mistakes_are_caught():
    c_u, n_u = 3, 4
    b = synth.custom_ug(2, 6, 9, c_u, n_u, 2, 16, seed=12, residual=False)
    good = ou.ug_cross_attn(b.q, b.k, b.v, c_u, n_u, b.scale)
    ref_u = np.stack([_sdpa(b.q[s, :c_u], b.k[s, :n_u], b.v[s, :n_u], b.scale)
                      for s in range(b.B)])
    assert np.max(np.abs(good[:, :c_u] - ref_u)) < 1e-12
    orig = ou.ug_mask
    bad_masks = (
        lambda To, Ti, cu, nu: ~((np.arange(To)[:, None] < cu) & (np.arange(Ti)[None, :] > nu)),
        lambda To, Ti, cu, nu: ~((np.arange(To)[:, None] >= cu) & (np.arange(Ti)[None, :] >= nu)),
        lambda To, Ti, cu, nu: ~((np.arange(To)[:, None] < cu) & (np.arange(Ti)[None, :] < nu)),
    )
    for bad in bad_masks:
        ou.ug_mask = bad
        try:
            wrong = ou.ug_cross_attn(b.q, b.k, b.v, c_u, n_u, b.scale)
        finally:
            ou.ug_mask = orig
        assert np.max(np.abs(wrong - good)) > 1e-6


def _brute(b, c_u, n_u):
    """Pure-Python restatement (math.exp): output i of a sample reads inputs [0, n_u) if i < c_u,
    else all inputs; no key -> 0; plus the residual."""
    q, k, v, r = (t.double().tolist() for t in (b.q, b.k, b.v, b.residual))
    out = np.zeros((b.B, b.T_out, b.H, b.d))
    for s in range(b.B):
        for i in range(b.T_out):
            keys = list(range(min(n_u, b.T_in) if i < c_u else b.T_in))
            for h in range(b.H):
                row = [0.0] * b.d
                if keys:
                    sc = [b.scale * math.fsum(x * y for x, y in zip(q[s][i][h], k[s][j][h]))
                          for j in keys]
                    top = max(sc)
                    w = [math.exp(x - top) for x in sc]
                    tot = math.fsum(w)
                    row = [math.fsum(wj / tot * v[s][j][h][c] for wj, j in zip(w, keys))
                           for c in range(b.d)]
                for c in range(b.d):
                    out[s, i, h, c] = row[c] + r[s][i][h][c]
    return out


def test_matches_brute_force_random_shapes():
    rng = np.random.default_rng(123)
    for case in range(24):
        B = int(rng.integers(1, 4))
        T_out = int(rng.integers(1, 6))
        T_in = int(rng.integers(1, 7))
        c_u = int(rng.integers(0, T_out + 1))
        n_u = int(rng.integers(0, T_in + 1))
        H = int(rng.integers(1, 3))
        d = int(rng.choice([4, 8]))
        b = synth.custom_ug(B, T_out, T_in, c_u, n_u, H, d, seed=1000 + case)
        got = ou.ug_cross_attn(b.q, b.k, b.v, c_u, n_u, b.scale, residual=b.residual)
        assert np.max(np.abs(got - _brute(b, c_u, n_u))) < 1e-12, (B, T_out, T_in, c_u, n_u)
