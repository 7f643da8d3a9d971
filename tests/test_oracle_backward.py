"""Pins of the backward oracle (oracle/backward.py) against things other than itself: torch's own
autograd through its scaled-dot-product attention (fp64, explicit boolean mask), central finite
differences of the forward oracle, the isolation properties the mask implies for gradients, closed
forms, and a library log-sum-exp; planted mistakes in a copy of the gradient formulas must fail."""

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

import oracle
import oracle.backward as ob
import synth


def _batch(seed=0, **kw):
    args = dict(hist_lengths=[3, 0, 9, 5], prefix=[1, 2, 0, 1], n_cand=[2, 3, 4, 0], H=2, d=16,
                seed=seed, pad_hist_to=4)
    args.update(kw)
    return synth.custom_batch(**args)


def _layout(b):
    off = oracle.offsets_from_lengths(b.row_lengths)
    return off, oracle.segment_ids(off, b.cand_start, b.valid)


def _dout(b, seed=7):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(b.q.shape, generator=g, dtype=torch.float64)


def _autograd_grads(b, off, seg, dout):
    """Gradients through torch's SDPA (float64, CPU) per user, over the user's non-padding rows only
    (SDPA gives NaN for a row with no visible key; padding keys are never visible, so dropping the
    padding rows is exact). Padding rows keep zero gradients."""
    T, H, d = b.q.shape
    dq, dk, dv = (np.zeros((T, H, d)) for _ in range(3))
    for u in range(b.B):
        s, e = int(off[u]), int(off[u + 1])
        rows = np.arange(s, e)[seg[s:e] != 0]
        if rows.size == 0:
            continue
        mask = torch.from_numpy(oracle.history_candidate_mask(seg[rows]))
        q, k, v = (t[rows].double().permute(1, 0, 2).unsqueeze(0).requires_grad_(True)
                   for t in (b.q, b.k, b.v))
        o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask,
                                                             scale=b.scale)
        o.backward(dout[rows].permute(1, 0, 2).unsqueeze(0))
        for dst, t in ((dq, q), (dk, k), (dv, v)):
            dst[rows] = t.grad[0].permute(1, 0, 2).numpy()
    return dq, dk, dv


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_matches_autograd_of_sdpa(seed):
    b = _batch(seed)
    off, seg = _layout(b)
    dout = _dout(b, seed + 10)
    got = ob.jagged_cand_attn_bwd(b.q, b.k, b.v, dout.numpy(), off, seg, b.scale)
    ref = _autograd_grads(b, off, seg, dout)
    for g, r in zip(got, ref):
        assert np.max(np.abs(g - r)) < 1e-12
    for g in got:
        assert np.all(g[seg == 0] == 0.0)    # padding rows: no gradient


def test_finite_differences():
    b = _batch(3, hist_lengths=[2, 3], prefix=[1, 0], n_cand=[2, 1], H=1, d=4, pad_hist_to=None)
    off, seg = _layout(b)
    dout = _dout(b, 3).numpy()
    q, k, v = (t.double().numpy() for t in (b.q, b.k, b.v))

    def loss(q_, k_, v_):
        return float(np.sum(dout * oracle.jagged_cand_attn(q_, k_, v_, off, seg, b.scale)))

    grads = ob.jagged_cand_attn_bwd(q, k, v, dout, off, seg, b.scale)
    rng = np.random.default_rng(0)
    h = 1e-5
    for which in range(3):
        for _ in range(12):
            idx = tuple(int(rng.integers(0, n)) for n in q.shape)
            args = [q.copy(), k.copy(), v.copy()]
            args[which][idx] += h
            up = loss(*args)
            args[which][idx] -= 2 * h
            dn = loss(*args)
            assert abs((up - dn) / (2 * h) - grads[which][idx]) < 1e-7


def test_candidate_gradient_isolation():
    # The upstream gradient of one candidate's output reaches only that candidate's own q, k, v
    # and its user's history rows: every other candidate's gradients are exactly 0.
    b = _batch(4)
    off, seg = _layout(b)
    cands = np.nonzero(seg == -1)[0]
    i = int(cands[2])
    dout = np.zeros(b.q.shape)
    dout[i] = _dout(b, 1).numpy()[i]
    dq, dk, dv = ob.jagged_cand_attn_bwd(b.q, b.k, b.v, dout, off, seg, b.scale)
    others = np.setdiff1d(cands, [i])
    for g in (dq, dk, dv):
        assert np.all(g[others] == 0.0)
    assert np.any(dv[i] != 0.0) and np.any(dq[i] != 0.0)
    user = np.searchsorted(off, i, side="right") - 1
    outside = np.r_[0:off[user], off[user + 1]:len(seg)]
    for g in (dq, dk, dv):
        assert np.all(g[outside] == 0.0)


def test_history_loss_gives_no_candidate_gradient():
    # History outputs never read candidates, so a loss on history rows only leaves every
    # candidate's q, k and v without gradient.
    b = _batch(5)
    off, seg = _layout(b)
    dout = _dout(b, 2).numpy()
    dout[seg != 1] = 0.0
    dq, dk, dv = ob.jagged_cand_attn_bwd(b.q, b.k, b.v, dout, off, seg, b.scale)
    for g in (dq, dk, dv):
        assert np.all(g[seg == -1] == 0.0)
    assert np.any(dk[seg == 1] != 0.0)


def test_lone_candidate_closed_form():
    # A candidate with no prefix and no history sees only itself: out = v, so dv = dout and
    # dq = dk = 0.
    b = synth.custom_batch([0], prefix=0, n_cand=1, H=2, d=8, seed=1)
    off, seg = _layout(b)
    dout = _dout(b, 5).numpy()
    dq, dk, dv = ob.jagged_cand_attn_bwd(b.q, b.k, b.v, dout, off, seg, b.scale)
    assert np.array_equal(dv, dout)
    assert np.all(dq == 0.0) and np.all(dk == 0.0)


def test_log_sum_exp():
    b = _batch(6)
    off, seg = _layout(b)
    lse = ob.log_sum_exp(b.q, b.k, off, seg, b.scale)
    q, k = b.q.double().numpy(), b.k.double().numpy()
    for u in range(b.B):
        s, e = int(off[u]), int(off[u + 1])
        mask = oracle.history_candidate_mask(seg[s:e])
        for r in range(e - s):
            for h in range(b.H):
                keys = np.nonzero(mask[r])[0]
                if keys.size == 0:
                    assert lse[s + r, h] == -np.inf
                    continue
                ref = logsumexp(b.scale * (k[s + keys, h, :] @ q[s + r, h, :]))
                assert abs(lse[s + r, h] - ref) < 1e-12
    # A lone candidate's only key is itself: lse = scale q.k.
    one = synth.custom_batch([0], prefix=0, n_cand=1, H=1, d=8, seed=2)
    o_off, o_seg = _layout(one)
    val = ob.log_sum_exp(one.q, one.k, o_off, o_seg, one.scale)[0, 0]
    qq, kk = one.q.double().numpy()[0, 0], one.k.double().numpy()[0, 0]
    assert abs(val - one.scale * float(qq @ kk)) < 1e-12


def test_planted_gradient_mistakes_are_caught(monkeypatch):
    b = _batch(8)
    off, seg = _layout(b)
    dout = _dout(b, 8)
    ref = _autograd_grads(b, off, seg, dout)
    orig = ob.masked_softmax_attention_bwd

    def no_centering(q, k, v, dO, mask, scale):
        # A copy of the gradient formulas with dS = P * dP (the rowsum term dropped).
        q, k, v, dO = (ob._as_f64(t) for t in (q, k, v, dO))
        dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
        has_key = mask.any(axis=1)
        for h in range(q.shape[1]):
            S = np.where(mask, scale * (q[:, h] @ k[:, h].T), -np.inf)
            m = np.where(has_key, S.max(axis=1, initial=-np.inf), 0.0)
            E = np.where(mask, np.exp(S - m[:, None]), 0.0)
            P = E / np.where(has_key, E.sum(axis=1), 1.0)[:, None]
            dv[:, h] = P.T @ dO[:, h]
            dS = P * (dO[:, h] @ v[:, h].T)
            dq[:, h] = scale * (dS @ k[:, h])
            dk[:, h] = scale * (dS.T @ q[:, h])
        return dq, dk, dv

    def swapped_grads(q, k, v, dO, mask, scale):
        dq, dk, dv = orig(q, k, v, dO, mask, scale)
        return dk, dq, dv

    def no_scale(q, k, v, dO, mask, scale):
        dq, dk, dv = orig(q, k, v, dO, mask, 1.0)
        return dq, dk, dv

    def transposed_mask(q, k, v, dO, mask, scale):
        return orig(q, k, v, dO, mask.T, scale)

    for bad in (no_centering, swapped_grads, no_scale, transposed_mask):
        monkeypatch.setattr(ob, "masked_softmax_attention_bwd", bad)
        got = ob.jagged_cand_attn_bwd(b.q, b.k, b.v, dout.numpy(), off, seg, b.scale)
        assert max(float(np.max(np.abs(g - r))) for g, r in zip(got, ref)) > 1e-6
    monkeypatch.setattr(ob, "masked_softmax_attention_bwd", orig)
