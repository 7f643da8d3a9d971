"""Pins of the causal-variant oracle (oracle/variants.py): torch's SDPA with is_causal per user
(fp64, a library routine), the pure-Python brute force with a lower-triangular mask, closed forms
(the first position of a user sees only itself; a one-token user outputs its v), the pair count,
and planted mistakes (strict triangle, upper triangle, a mask crossing users)."""

import numpy as np
import pytest
import torch

import oracle
import oracle.variants as ov
import synth


def _batch(seed=0, lengths=(1, 5, 0, 17, 64)):
    return synth.custom_batch(list(lengths), prefix=0, n_cand=0, H=2, d=16, seed=seed)


@pytest.mark.parametrize("seed", [0, 1])
def test_matches_sdpa_is_causal(seed):
    b = _batch(seed)
    off = oracle.offsets_from_lengths(b.row_lengths)
    got = ov.jagged_causal_attn(b.q, b.k, b.v, off, b.scale)
    for u in range(b.B):
        s, e = int(off[u]), int(off[u + 1])
        if e == s:
            continue
        q, k, v = (t[s:e].double().permute(1, 0, 2).unsqueeze(0) for t in (b.q, b.k, b.v))
        ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True,
                                                               scale=b.scale)
        assert np.max(np.abs(got[s:e] - ref[0].permute(1, 0, 2).numpy())) < 1e-12


def test_matches_brute_force():
    # Pure-Python triple loop (math.exp, no numpy): position i sees positions 0..i of its user.
    import math
    b = _batch(3, lengths=(3, 1, 6))
    off = oracle.offsets_from_lengths(b.row_lengths)
    got = ov.jagged_causal_attn(b.q, b.k, b.v, off, b.scale)
    q, k, v = (t.double().tolist() for t in (b.q, b.k, b.v))
    for u in range(b.B):
        s, e = int(off[u]), int(off[u + 1])
        for i in range(s, e):
            for h in range(b.H):
                sc = [b.scale * math.fsum(x * y for x, y in zip(q[i][h], k[j][h]))
                      for j in range(s, i + 1)]
                top = max(sc)
                w = [math.exp(x - top) for x in sc]
                tot = math.fsum(w)
                for c in range(b.d):
                    ref = math.fsum(w[j - s] / tot * v[j][h][c] for j in range(s, i + 1))
                    assert abs(got[i, h, c] - ref) < 1e-12


def test_closed_forms():
    b = _batch(4)
    off = oracle.offsets_from_lengths(b.row_lengths)
    got = ov.jagged_causal_attn(b.q, b.k, b.v, off, b.scale)
    v = b.v.double().numpy()
    for u in range(b.B):
        s, e = int(off[u]), int(off[u + 1])
        if e > s:
            assert np.array_equal(got[s], v[s])      # the first position sees only itself


def test_pair_count():
    lengths = [1, 5, 0, 17, 64]
    off = oracle.offsets_from_lengths(lengths)
    total = sum(int(ov.causal_mask(e - s).sum()) for s, e in zip(off[:-1], off[1:]))
    assert ov.causal_pairs(lengths) == total == 1 + 15 + 0 + 153 + 2080


def test_planted_mask_mistakes_are_caught():
    b = _batch(5)
    off = oracle.offsets_from_lengths(b.row_lengths)
    good = ov.jagged_causal_attn(b.q, b.k, b.v, off, b.scale)
    orig = ov.causal_mask
    for bad in (lambda L: np.tril(np.ones((L, L), bool), -1) | (np.arange(L)[:, None] == 0) &
                (np.arange(L)[None, :] == 0),          # strict triangle (row 0 kept non-empty)
                lambda L: np.triu(np.ones((L, L), bool))):  # upper triangle
        ov.causal_mask = bad
        try:
            assert np.max(np.abs(ov.jagged_causal_attn(b.q, b.k, b.v, off, b.scale) - good)) > 1e-6
        finally:
            ov.causal_mask = orig
    # A mask that crosses users: attention over the whole packed batch at once.
    T = int(off[-1])
    whole = oracle.masked_softmax_attention(b.q, b.k, b.v, ov.causal_mask(T), b.scale)
    assert np.max(np.abs(whole - good)) > 1e-6
