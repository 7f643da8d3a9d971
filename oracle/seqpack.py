"""CPU oracle of training with candidate packing (numpy, fp64).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only the tests, the smoke check and the
benchmark's CPU baseline may import it, and it imports nothing from the CUDA package.

What the pages fix (候选隔离注意力掩码, section 训练时的序列打包): training packs several users'
sequences into one matrix and the variable-length attention splits them at cu_seqlens; with
candidate packing on, the candidates are stored apart, all in one place, and each candidate's
representation is then taken out at its candidate_positions entry. Packing changes where rows sit,
not what they compute: the serving contract (the mask of section 段 ID：掩码的表达方式) holds.

Reading of the layout (the pages name it, they do not draw it): one packed matrix of T = Th + Nc
rows. Rows [0, Th) hold every user's prefix + history back to back, split at ``hist_offsets``
(the cu_seqlens, [B+1], hist_offsets[B] = Th). Rows [Th, T) hold every user's candidates back to
back, split at ``cand_offsets`` ([B+1], relative to Th, cand_offsets[B] = Nc). Candidate c (in
that order) sits at row candidate_positions[c] = Th + c. Segment IDs per row keep their meaning:
1 for a history row, 0 for padding, -1 for a candidate. User b's rows are its history run followed
by its candidate run; the explicit mask of those rows, in that order, is the serving rule.
"""

from __future__ import annotations

import numpy as np

from .backward import masked_softmax_attention_bwd
from .jagged_oracle import (SEG_CANDIDATE, SEG_HISTORY, _as_f64, history_candidate_mask,
                            masked_softmax_attention)


def candidate_positions(hist_offsets, cand_offsets) -> np.ndarray:
    """Row of each candidate in the packed matrix: the candidate block starts after the last
    history row."""
    Th = int(np.asarray(hist_offsets)[-1])
    Nc = int(np.asarray(cand_offsets)[-1])
    return Th + np.arange(Nc, dtype=np.int64)


def user_rows(hist_offsets, cand_offsets, b: int) -> np.ndarray:
    """Packed rows of user b: its history run, then its candidate run."""
    hoff = np.asarray(hist_offsets, dtype=np.int64)
    coff = np.asarray(cand_offsets, dtype=np.int64)
    pos = candidate_positions(hoff, coff)
    return np.concatenate([np.arange(int(hoff[b]), int(hoff[b + 1])),
                           pos[int(coff[b]):int(coff[b + 1])]]).astype(np.int64)


def segment_ids(hist_offsets, cand_offsets, hist_valid=None) -> np.ndarray:
    """Segment IDs of the packed matrix: history rows 1 (0 where ``hist_valid`` marks padding),
    candidate rows -1."""
    Th = int(np.asarray(hist_offsets)[-1])
    Nc = int(np.asarray(cand_offsets)[-1])
    seg = np.empty(Th + Nc, dtype=np.int8)
    seg[:Th] = SEG_HISTORY if hist_valid is None else np.where(
        np.asarray(hist_valid).astype(bool), SEG_HISTORY, 0)
    seg[Th:] = SEG_CANDIDATE
    return seg


def seqpack_attn(q, k, v, hist_offsets, cand_offsets, seg, scale: float,
                 mask_fn=history_candidate_mask) -> np.ndarray:
    """Forward over the packed matrix (fp64 [T, H, d]): per user, masked softmax attention over
    its rows under the explicit mask of their segment IDs."""
    seg = np.asarray(seg)
    B = np.asarray(hist_offsets).shape[0] - 1
    T = seg.shape[0]
    out = np.zeros((T, q.shape[1], v.shape[2]), dtype=np.float64)
    for b in range(B):
        rows = user_rows(hist_offsets, cand_offsets, b)
        if rows.size == 0:
            continue
        out[rows] = masked_softmax_attention(_as_f64(q)[rows], _as_f64(k)[rows], _as_f64(v)[rows],
                                             mask_fn(seg[rows]), scale)
    return out


def seqpack_log_sum_exp(q, k, hist_offsets, cand_offsets, seg, scale: float) -> np.ndarray:
    """Per row and head, log sum_j exp(scale q.k_j) over the keys the mask lets the row see
    (natural log, fp64 [T, H]; -inf for a row that sees no key)."""
    q, k = _as_f64(q), _as_f64(k)
    seg = np.asarray(seg)
    B = np.asarray(hist_offsets).shape[0] - 1
    T, H, _ = q.shape
    out = np.full((T, H), -np.inf)
    for b in range(B):
        rows = user_rows(hist_offsets, cand_offsets, b)
        if rows.size == 0:
            continue
        mask = history_candidate_mask(seg[rows])
        for h in range(H):
            S = np.where(mask, scale * (q[rows, h, :] @ k[rows, h, :].T), -np.inf)
            m = S.max(axis=1, initial=-np.inf)
            ok = np.isfinite(m)
            lse = np.full(rows.size, -np.inf)
            lse[ok] = m[ok] + np.log(np.exp(S[ok] - m[ok, None]).sum(axis=1))
            out[rows, h] = lse
    return out


def seqpack_attn_bwd(q, k, v, dout, hist_offsets, cand_offsets, seg, scale: float,
                     users=None):
    """Gradients (dq, dk, dv), fp64 [T, H, d], of ``seqpack_attn`` for the upstream gradient
    ``dout``, per user over its rows; ``users`` restricts the work (other rows stay 0)."""
    seg = np.asarray(seg)
    B = np.asarray(hist_offsets).shape[0] - 1
    T = seg.shape[0]
    shape = (T, q.shape[1], q.shape[2])
    dq, dk, dv = np.zeros(shape), np.zeros(shape), np.zeros((T, v.shape[1], v.shape[2]))
    q, k, v, dout = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(dout)
    for b in (range(B) if users is None else users):
        rows = user_rows(hist_offsets, cand_offsets, b)
        if rows.size == 0:
            continue
        g = masked_softmax_attention_bwd(q[rows], k[rows], v[rows], dout[rows],
                                         history_candidate_mask(seg[rows]), scale)
        dq[rows], dk[rows], dv[rows] = g
    return dq, dk, dv
