"""Second, independent restatement of the attention definition, in pure Python (lists + math).

TEST INFRASTRUCTURE ONLY: used to pin the numpy oracle on tiny inputs. It shares no code with the
numpy oracle, and states visibility in an equivalent but differently written form of the rule in
候选隔离注意力掩码 (section 段 ID：掩码的表达方式): a key j is visible to a query i of the same user
when j has segment 1 and i is not padding, or when i == j and i is a candidate.
"""

from __future__ import annotations

import math


def visible(seg_row, i, j) -> bool:
    if seg_row[j] == 1 and seg_row[i] != 0:
        return True
    return i == j and seg_row[i] == -1


def attention_row(qi, keys, values, seg_row, i, scale):
    """One query row of one head: qi [d], keys/values [L][d] lists of floats."""
    scores = []
    for j in range(len(keys)):
        if visible(seg_row, i, j):
            s = 0.0
            for a, b in zip(qi, keys[j]):
                s += a * b
            scores.append((j, scale * s))
    if not scores:
        return [0.0] * len(values[0]) if values else []
    top = max(s for _, s in scores)
    weights = [(j, math.exp(s - top)) for j, s in scores]
    total = math.fsum(w for _, w in weights)
    out = [0.0] * len(values[0])
    for j, w in weights:
        for c in range(len(out)):
            out[c] += (w / total) * values[j][c]
    return out


def jagged_attention(q, k, v, row_lengths, seg, scale):
    """q, k, v: nested lists [T][H][d]; row_lengths: per-user row lengths; seg: list [T]."""
    T = len(q)
    H = len(q[0]) if T else 0
    out = [[None] * H for _ in range(T)]
    start = 0
    for L in row_lengths:
        seg_row = seg[start:start + L]
        for h in range(H):
            keys = [k[start + j][h] for j in range(L)]
            values = [v[start + j][h] for j in range(L)]
            for i in range(L):
                out[start + i][h] = attention_row(q[start + i][h], keys, values, seg_row, i, scale)
        start += L
    return out
