"""CPU oracle for right-anchored rotary position embedding (numpy, fp64).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only the tests, the smoke check and the
benchmark's CPU baseline may import it, and it imports nothing from the CUDA package.

What the pages fix (候选隔离注意力掩码, section 位置编码：候选共用一个位置): the history is right-aligned,
so that the newest history record always sits at position ``history_end - 1`` whatever the
history's length, and every candidate sits at ``history_end``. Candidates therefore carry no order
information, and together with the mask isolation, reordering candidates does not change any score.

Readings (the pages are silent on these):

* Segment-1 tokens (user prefix and history) form one right-aligned run: the k-th segment-1 token
  of a user with n segment-1 tokens gets ``history_end - n + k``. Padding tokens (segment 0) get
  the position the next segment-1 token would get, ``history_end - n + (segment-1 tokens before
  it)``; no score ever reads it (padding is never a visible key, and a padding query outputs 0).
* ``history_end`` is one constant for the batch. Rotary scores depend only on position
  differences, so its value never changes an attention output (pinned in the tests).
* Rotation: the rotate-half pairing (element j with element j + d/2) with frequencies
  ``base ** (-2 j / d)``, base 10000, applied to queries and keys of every head alike.
"""

from __future__ import annotations

import numpy as np

from .jagged_oracle import SEG_CANDIDATE, SEG_HISTORY


def right_anchored_positions(offsets, seg, history_end: int) -> np.ndarray:
    """Position of every packed token under the right-anchored rule (int64 [T])."""
    offsets = np.asarray(offsets, dtype=np.int64)
    seg = np.asarray(seg)
    pos = np.zeros(seg.shape[0], dtype=np.int64)
    for b in range(len(offsets) - 1):
        s, e = int(offsets[b]), int(offsets[b + 1])
        n = int(np.sum(seg[s:e] == SEG_HISTORY))
        before = 0                                # segment-1 tokens seen so far in the row
        for i in range(s, e):
            if seg[i] == SEG_CANDIDATE:
                pos[i] = history_end
            else:
                pos[i] = history_end - n + before
                if seg[i] == SEG_HISTORY:
                    before += 1
    return pos


def rope_inverse_frequencies(d: int, base: float = 10000.0) -> np.ndarray:
    """theta_j = base ** (-2 j / d) for j = 0 .. d/2 - 1 (float64)."""
    j = np.arange(d // 2, dtype=np.float64)
    return base ** (-2.0 * j / d)


def apply_rope(x, pos, base: float = 10000.0) -> np.ndarray:
    """Rotate [T, H, d] rows by their positions: for each pair (j, j + d/2),
    (a, b) -> (a cos(p theta_j) - b sin(p theta_j), a sin(p theta_j) + b cos(p theta_j))."""
    x = np.asarray(x.float().numpy() if hasattr(x, "float") else x, dtype=np.float64)
    T, H, d = x.shape
    half = d // 2
    ang = np.asarray(pos, dtype=np.float64)[:, None] * rope_inverse_frequencies(d, base)[None, :]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    a, b = x[..., :half], x[..., half:]
    out = np.empty_like(x)
    out[..., :half] = a * c - b * s
    out[..., half:] = a * s + b * c
    return out


def cand_only_positions(cand_offsets, hist_offsets, hist_seg, history_end: int):
    """Positions for the candidate-only layer: the frozen history K/V keep their right-anchored
    positions (segment-1 history rows; hist_seg None means all valid), every candidate sits at
    history_end. Returns (history positions [Th], candidate positions [Nc])."""
    hist_offsets = np.asarray(hist_offsets, dtype=np.int64)
    Th = int(hist_offsets[-1])
    hseg = np.ones(Th, dtype=np.int8) if hist_seg is None else np.asarray(hist_seg)
    hpos = right_anchored_positions(hist_offsets, hseg, history_end)
    Nc = int(np.asarray(cand_offsets)[-1])
    return hpos, np.full(Nc, history_end, dtype=np.int64)


def round_to_bf16(x) -> np.ndarray:
    """Round to bfloat16 as a bf16 tensor stores it: to fp32 first, then to the nearest bf16 (ties
    to even). Returns the rounded values as float64."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    bits = f.view(np.uint32).astype(np.uint64)
    rounded = ((bits + 0x7FFF + ((bits >> 16) & 1)) >> 16) << 16
    return (rounded & 0xFFFFFFFF).astype(np.uint32).view(np.float32).astype(np.float64)
