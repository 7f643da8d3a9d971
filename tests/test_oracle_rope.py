"""Pins of the right-anchored RoPE oracle (oracle/rope.py) against the pages' rule, closed forms and
invariants, so that a dropped term, a flipped sign or a wrong index in it fails here."""

import json
from pathlib import Path

import numpy as np
import pytest

import oracle

GOLDEN = Path(__file__).parent / "golden"


def test_positions_worked_example():
    g = json.loads((GOLDEN / "rope_positions.json").read_text())
    off = oracle.offsets_from_lengths(g["lengths"])
    pos = oracle.right_anchored_positions(off, np.array(g["seg"], dtype=np.int8), g["history_end"])
    assert pos.tolist() == g["positions"]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_newest_history_at_history_end_minus_one(seed):
    rng = np.random.default_rng(seed)
    lengths, segs = [], []
    for _ in range(20):
        n_hist, n_pad, n_cand = (int(x) for x in rng.integers(0, 9, size=3))
        row = np.array([1] * n_hist + [0] * n_pad + [-1] * n_cand, dtype=np.int8)
        rng.shuffle(row[: n_hist + n_pad])          # padding anywhere inside the history
        lengths.append(row.size)
        segs.append(row)
    off = oracle.offsets_from_lengths(lengths)
    seg = np.concatenate(segs) if segs else np.zeros(0, np.int8)
    pos = oracle.right_anchored_positions(off, seg, 1000)
    for b, row in enumerate(segs):
        p = pos[off[b]:off[b + 1]]
        hist = p[row == 1]
        if hist.size:
            assert hist[-1] == 999 and np.all(np.diff(hist) == 1)    # contiguous, right-aligned
        assert np.all(p[row == -1] == 1000)                          # one shared position


def test_inverse_frequencies_closed_form():
    inv = oracle.rope_inverse_frequencies(4, base=10000.0)
    assert inv.tolist() == [1.0, 0.01]                               # 10000^0, 10000^(-2/4)
    assert oracle.rope_inverse_frequencies(128)[64 - 1] == pytest.approx(10000.0 ** (-126 / 128))


def test_two_dims_is_complex_rotation():
    # d = 2: (a, b) -> (a + ib) e^{i p theta_0} with theta_0 = 1
    rng = np.random.default_rng(5)
    x = rng.standard_normal((7, 3, 2))
    pos = np.arange(7) * 3 - 5
    y = oracle.apply_rope(x, pos)
    z = (x[..., 0] + 1j * x[..., 1]) * np.exp(1j * pos)[:, None]
    assert np.allclose(y[..., 0], z.real, atol=1e-12) and np.allclose(y[..., 1], z.imag, atol=1e-12)


def test_rotation_preserves_norm_and_position_zero_is_identity():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((11, 2, 16))
    pos = rng.integers(-50, 5000, size=11)
    y = oracle.apply_rope(x, pos)
    assert np.allclose(np.linalg.norm(y, axis=2), np.linalg.norm(x, axis=2), rtol=1e-12)
    assert np.array_equal(oracle.apply_rope(x, np.zeros(11, np.int64)), x)


def test_scores_depend_only_on_position_difference():
    # <rope(q, p + c), rope(k, r + c)> == <rope(q, p), rope(k, r)> for any shift c
    rng = np.random.default_rng(7)
    q = rng.standard_normal((5, 1, 32))
    k = rng.standard_normal((5, 1, 32))
    p = rng.integers(0, 300, size=5)
    r = rng.integers(0, 300, size=5)
    s0 = np.einsum("ihd,ihd->i", oracle.apply_rope(q, p), oracle.apply_rope(k, r))
    s1 = np.einsum("ihd,ihd->i", oracle.apply_rope(q, p + 777), oracle.apply_rope(k, r + 777))
    assert np.allclose(s0, s1, atol=1e-10)


def _rope_attention(b, history_end):
    seg = oracle.segment_ids(oracle.offsets_from_lengths(b.row_lengths), b.cand_start, b.valid)
    off = oracle.offsets_from_lengths(b.row_lengths)
    pos = oracle.right_anchored_positions(off, seg, history_end)
    q = oracle.apply_rope(b.q, pos)
    k = oracle.apply_rope(b.k, pos)
    return oracle.jagged_cand_attn(q, k, b.v, off, seg, b.scale), off, seg


def test_attention_independent_of_history_end():
    import synth
    b = synth.custom_batch([5, 0, 9], prefix=1, n_cand=4, H=2, d=16, seed=3)
    o1, _, _ = _rope_attention(b, 0)
    o2, _, _ = _rope_attention(b, 4096)
    assert np.allclose(o1, o2, atol=1e-10)


def test_candidate_order_does_not_change_scores():
    # Candidates share one position, so with the isolation mask a permutation of a user's
    # candidates permutes their outputs and leaves every other row unchanged.
    import synth
    import torch
    b = synth.custom_batch([6, 3], prefix=2, n_cand=5, H=2, d=16, seed=4)
    o1, off, seg = _rope_attention(b, 100)
    s, e = int(off[0]), int(off[1])
    cands = np.nonzero(seg[s:e] == -1)[0] + s
    perm = np.arange(b.q.shape[0])
    perm[cands] = cands[::-1]
    b2 = synth.workloads.Batch(**{**b.__dict__, "q": b.q[torch.tensor(perm)],
                                  "k": b.k[torch.tensor(perm)], "v": b.v[torch.tensor(perm)]})
    o2, _, _ = _rope_attention(b2, 100)
    assert np.allclose(o2[perm], o1, atol=1e-12)


def test_cand_only_positions():
    hpos, cpos = oracle.cand_only_positions([0, 3, 5], [0, 4, 6], None, 50)
    assert hpos.tolist() == [46, 47, 48, 49, 48, 49] and cpos.tolist() == [50] * 5


def test_round_to_bf16_ties_to_even():
    x = np.array([1.0, 1 + 2 ** -8, 1 + 3 * 2 ** -9, 1 + 2 ** -7 + 2 ** -8, -2.0 ** -130])
    assert oracle.round_to_bf16(x).tolist() == [1.0, 1.0, 1 + 2 ** -7, 1 + 2 ** -6, -2.0 ** -130]


def test_rotate_half_pairing_d4():
    # d = 4: element j pairs with element j + 2, frequencies (1, 1/100)
    x = np.array([[[1.0, 2.0, 3.0, 4.0]]])
    p = 0.7
    y = oracle.apply_rope(x, np.array([p]))[0, 0]
    c0, s0, c1, s1 = np.cos(p), np.sin(p), np.cos(p / 100), np.sin(p / 100)
    assert np.allclose(y, [1 * c0 - 3 * s0, 2 * c1 - 4 * s1, 1 * s0 + 3 * c0, 2 * s1 + 4 * c1],
                       atol=1e-14)
