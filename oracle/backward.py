"""CPU oracle of the backward pass of jagged candidate-isolated attention (numpy, fp64).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only the tests, the smoke check and the
benchmark's CPU baseline may import it, and it imports nothing from the CUDA package.

The pages train on the same packed layout they serve (候选隔离注意力掩码, section 训练时的序列打包:
several users' sequences share one packed matrix and the attention splits them at cu_seqlens,
i.e. the values + offsets of the forward), with the same mask. The backward pass is therefore the
gradient of the forward's masked softmax attention, per user and head. Written out from the
definitions, with S = scale Q K^T (masked entries -inf), P the row softmax of S and O = P V, for an
upstream gradient dO:

    dV = P^T dO
    dP = dO V^T
    dS = P * (dP - rowsum(P * dP))          (rowsum(P * dP) = rowsum(dO * O))
    dQ = scale dS K
    dK = scale dS^T Q

Rows that see no key (padding queries) output the constant 0, so no gradient flows through them;
padding keys are never visible, so their dK and dV are 0 as well.

``log_sum_exp`` is the statistic a tiled backward keeps from its forward: per row and head,
log sum_j exp(scale q.k_j) over the visible keys j (natural log; -inf for a row with no key).
"""

from __future__ import annotations

import numpy as np

from .jagged_oracle import _as_f64, history_candidate_mask


def masked_softmax_attention_bwd(q, k, v, dout, mask, scale: float):
    """Gradients (dq, dk, dv) of one user's masked softmax attention for the upstream gradient
    ``dout``; q, k, v, dout: [L, H, d], mask: [L, L] bool."""
    q, k, v, dout = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(dout)
    L, H, d = q.shape
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    if L == 0:
        return dq, dk, dv
    has_key = mask.any(axis=1)
    for h in range(H):
        S = scale * (q[:, h, :] @ k[:, h, :].T)
        S = np.where(mask, S, -np.inf)
        m = np.where(has_key, S.max(axis=1, initial=-np.inf), 0.0)
        E = np.where(mask, np.exp(S - m[:, None]), 0.0)
        P = E / np.where(has_key, E.sum(axis=1), 1.0)[:, None]
        dO = dout[:, h, :]
        dv[:, h, :] = P.T @ dO
        dP = dO @ v[:, h, :].T
        dS = P * (dP - (P * dP).sum(axis=1)[:, None])
        dq[:, h, :] = scale * (dS @ k[:, h, :])
        dk[:, h, :] = scale * (dS.T @ q[:, h, :])
    return dq, dk, dv


def jagged_cand_attn_bwd(q, k, v, dout, offsets, seg, scale: float,
                         mask_fn=history_candidate_mask, users=None):
    """Gradients (dq, dk, dv), each fp64 [T, H, d], of ``jagged_cand_attn`` for the upstream
    gradient ``dout``: per user row [offsets[b], offsets[b+1]) with the explicit mask of its
    segment IDs; no gradient crosses a user boundary. ``users`` restricts the work (other rows 0)."""
    offsets = np.asarray(offsets, dtype=np.int64)
    seg = np.asarray(seg)
    T = int(offsets[-1])
    shape = (T, q.shape[1], q.shape[2])
    dq, dk, dv = np.zeros(shape), np.zeros(shape), np.zeros((T, v.shape[1], v.shape[2]))
    for b in (range(offsets.shape[0] - 1) if users is None else users):
        s, e = int(offsets[b]), int(offsets[b + 1])
        if e == s:
            continue
        g = masked_softmax_attention_bwd(q[s:e], k[s:e], v[s:e], dout[s:e], mask_fn(seg[s:e]),
                                         scale)
        dq[s:e], dk[s:e], dv[s:e] = g
    return dq, dk, dv


def log_sum_exp(q, k, offsets, seg, scale: float, mask_fn=history_candidate_mask):
    """Per row and head, log sum_j exp(scale q.k_j) over the keys the mask lets the row see
    (fp64 [T, H]; -inf for rows that see no key)."""
    q, k = _as_f64(q), _as_f64(k)
    offsets = np.asarray(offsets, dtype=np.int64)
    seg = np.asarray(seg)
    T, H, _ = q.shape
    out = np.full((T, H), -np.inf)
    for b in range(offsets.shape[0] - 1):
        s, e = int(offsets[b]), int(offsets[b + 1])
        if e == s:
            continue
        mask = mask_fn(seg[s:e])
        for h in range(H):
            S = scale * (q[s:e, h, :] @ k[s:e, h, :].T)
            S = np.where(mask, S, -np.inf)
            m = S.max(axis=1, initial=-np.inf)
            ok = np.isfinite(m)
            lse = np.full(e - s, -np.inf)
            lse[ok] = m[ok] + np.log(np.exp(S[ok] - m[ok, None]).sum(axis=1))
            out[s:e, h] = lse
    return out
