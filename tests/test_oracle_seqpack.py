"""Pins of the candidate-packing oracle (oracle/seqpack.py) on the CPU.

Training packs users' sequences into one matrix, and with candidate packing the candidates are
stored apart in one block and read back by candidate_positions (候选隔离注意力掩码, section
训练时的序列打包); packing must not change what any row computes. Pinned by: a hand-worked layout
on the worked offsets example, exact equality with the serving-layout oracle on the same rows
rearranged (forward, log-sum-exp and gradients), central finite differences of the packed forward,
and planted mistakes in the layout that the equality catches.
"""

import numpy as np
import pytest

import oracle
import oracle.backward as ob
import oracle.seqpack as osp
import synth
from helpers import seqpack_layout


def test_hand_worked_layout():
    # histories of 2, 5 and 1 rows (offsets [0, 2, 7, 8], the worked offsets example) and 3, 0, 2
    # candidates: the candidate block starts at row 8.
    hoff, coff = np.array([0, 2, 7, 8]), np.array([0, 3, 3, 5])
    assert osp.candidate_positions(hoff, coff).tolist() == [8, 9, 10, 11, 12]
    assert osp.user_rows(hoff, coff, 0).tolist() == [0, 1, 8, 9, 10]
    assert osp.user_rows(hoff, coff, 1).tolist() == [2, 3, 4, 5, 6]
    assert osp.user_rows(hoff, coff, 2).tolist() == [7, 11, 12]
    assert osp.segment_ids(hoff, coff).tolist() == [1] * 8 + [-1] * 5
    assert osp.segment_ids(hoff, coff, [1, 1, 1, 0, 1, 1, 1, 1])[3] == 0


def _batches():
    return [synth.tiny(),
            synth.custom_batch([0, 7, 30, 12, 1], prefix=[2, 0, 4, 1, 0], n_cand=[5, 1, 14, 0, 3],
                               H=3, d=8, seed=4, pad_hist_to=8)]


@pytest.mark.parametrize("i", [0, 1])
def test_forward_and_lse_equal_the_serving_layout(i):
    b = _batches()[i]
    off = oracle.offsets_from_lengths(b.row_lengths)
    seg = oracle.segment_ids(off, b.cand_start, b.valid)
    perm, hoff, coff = seqpack_layout(b)
    sseg = seg[perm]
    got = osp.seqpack_attn(b.q[perm], b.k[perm], b.v[perm], hoff, coff, sseg, b.scale)
    ref = oracle.jagged_cand_attn(b.q, b.k, b.v, off, seg, b.scale)[perm]
    assert np.array_equal(got, ref)
    lse = osp.seqpack_log_sum_exp(b.q[perm], b.k[perm], hoff, coff, sseg, b.scale)
    assert np.array_equal(lse, ob.log_sum_exp(b.q, b.k, off, seg, b.scale)[perm])


@pytest.mark.parametrize("i", [0, 1])
def test_gradients_equal_the_serving_layout(i):
    b = _batches()[i]
    off = oracle.offsets_from_lengths(b.row_lengths)
    seg = oracle.segment_ids(off, b.cand_start, b.valid)
    perm, hoff, coff = seqpack_layout(b)
    dout = synth.upstream_grad(b.q.shape, 3).double().numpy()
    got = osp.seqpack_attn_bwd(b.q[perm], b.k[perm], b.v[perm], dout[perm], hoff, coff, seg[perm],
                               b.scale)
    ref = ob.jagged_cand_attn_bwd(b.q, b.k, b.v, dout, off, seg, b.scale)
    for g, r in zip(got, ref):
        assert np.array_equal(g, r[perm])


def test_gradients_by_finite_differences():
    # Packed forward differentiated numerically, independent of the gradient formulas.
    b = synth.custom_batch([3, 0, 2], prefix=1, n_cand=[2, 2, 1], H=1, d=4, seed=8)
    off = oracle.offsets_from_lengths(b.row_lengths)
    perm, hoff, coff = seqpack_layout(b)
    seg = oracle.segment_ids(off, b.cand_start)[perm]
    q, k, v = (t.double().numpy()[perm] for t in (b.q, b.k, b.v))
    rng = np.random.default_rng(0)
    dout = rng.standard_normal(q.shape)
    dq, dk, dv = osp.seqpack_attn_bwd(q, k, v, dout, hoff, coff, seg, b.scale)
    eps = 1e-6

    def loss(qq, kk, vv):
        return float(np.sum(osp.seqpack_attn(qq, kk, vv, hoff, coff, seg, b.scale) * dout))

    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - g[idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, g[idx])


def test_planted_layout_mistakes_are_caught(monkeypatch):
    b = _batches()[1]
    off = oracle.offsets_from_lengths(b.row_lengths)
    seg = oracle.segment_ids(off, b.cand_start, b.valid)
    perm, hoff, coff = seqpack_layout(b)
    ref = oracle.jagged_cand_attn(b.q, b.k, b.v, off, seg, b.scale)[perm]

    def run():
        return osp.seqpack_attn(b.q[perm], b.k[perm], b.v[perm], hoff, coff, seg[perm], b.scale)

    # candidate rows counted from 0 instead of from the end of the history block
    monkeypatch.setattr(osp, "candidate_positions",
                        lambda h, c: np.arange(int(np.asarray(c)[-1]), dtype=np.int64))
    assert not np.allclose(run(), ref)
    monkeypatch.undo()
    # the whole candidate block treated as every user's candidates
    monkeypatch.setattr(osp, "user_rows", lambda h, c, u: np.concatenate(
        [np.arange(int(h[u]), int(h[u + 1])), int(h[-1]) + np.arange(int(c[-1]))]))
    assert not np.allclose(run(), ref)
    monkeypatch.undo()
    assert np.array_equal(run(), ref)
