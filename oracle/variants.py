"""CPU oracle of the per-user causal variant of jagged attention (numpy, fp64).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only the tests, the smoke check and the
benchmark's CPU baseline may import it, and it imports nothing from the CUDA package.

The candidate-isolation page's FAQ notes that the early demo ranker built a lower-triangular mask
over the user's sequence (jnp.tril) before production moved to bidirectional prefix/history
attention; the contest repository's inference path runs the same kind of mask over packed users
(a block-diagonal causal varlen attention split at cu_seqlens). The variant computed here is that
mask on the packed layout: position i of user b attends to the positions j <= i of the same user,
and nothing else. Written out per user with an explicit [L, L] lower-triangular mask and the same
masked softmax as the main oracle.
"""

from __future__ import annotations

import numpy as np

from .jagged_oracle import masked_softmax_attention


def causal_mask(L: int) -> np.ndarray:
    """mask[q, kv] = kv <= q: the lower triangle, diagonal included."""
    q = np.arange(int(L))[:, None]
    kv = np.arange(int(L))[None, :]
    return kv <= q


def jagged_causal_attn(q, k, v, offsets, scale: float, users=None) -> np.ndarray:
    """Per-user causal attention over a packed batch (fp64 [T, H, d]); ``users`` restricts the
    computation to a subset (other rows stay 0)."""
    offsets = np.asarray(offsets, dtype=np.int64)
    T = int(offsets[-1])
    out = np.zeros((T, q.shape[1], v.shape[2]), dtype=np.float64)
    for b in (range(offsets.shape[0] - 1) if users is None else users):
        s, e = int(offsets[b]), int(offsets[b + 1])
        if e > s:
            out[s:e] = masked_softmax_attention(q[s:e], k[s:e], v[s:e], causal_mask(e - s), scale)
    return out


def causal_pairs(lengths) -> int:
    """Allowed (query, key) pairs of the causal variant: L (L + 1) / 2 per user."""
    n = np.asarray(lengths, dtype=np.int64)
    return int((n * (n + 1) // 2).sum())
