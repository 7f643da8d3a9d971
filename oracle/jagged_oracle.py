"""CPU oracle for jagged, candidate-isolated softmax attention (numpy, fp64).

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg may import this module. The product path never calls it, and it imports nothing from
the CUDA package: the two share no code.

Every function restates one rule of the source pages, in the pages' order and notation:

* Packed storage: values + offsets, where sequence i is ``values[offsets[i]:offsets[i+1]]``
  ('HSTU scale' tutorial, section 手算 padding 的浪费与 offset).
* Segment IDs per position: 1 = user prefix / history, -1 = candidate, 0 = padding
  (候选隔离注意力掩码, section 段 ID：掩码的表达方式).
* ``bounds_from_segment_ids``: per row, the history interval and the candidate interval
  (same section). The empty-interval convention is not on the pages; the reading taken is
  hist_lo = hist_hi = row start, cand_lo = cand_hi = row end (parity unpinned by the pages;
  pinned by our own unit tests only).
* ``history_candidate_mask``: key is visible when it is history and the query is history or a
  candidate, or when query and key are the same candidate position (same section).
* Masked softmax attention with an explicit [L, L] mask per user, which the GPU path deliberately
  never builds (候选隔离注意力掩码, section 设计决策). Query rows with no visible key (padding rows)
  output 0 (reading: the pages are silent).
* Candidate-only layer: candidate queries attend to frozen history K/V and their own K/V
  (section 只更新候选的末尾层). The oracle evaluates it through the fallback the same section gives:
  run the full mask over [history | candidates] and keep the candidate rows.
"""

from __future__ import annotations

import numpy as np

SEG_HISTORY = 1
SEG_CANDIDATE = -1
SEG_PADDING = 0


# ------------------------------------------------------------------------------------------------
# Storage: values + offsets ('HSTU scale', section 手算 padding 的浪费与 offset)
# ------------------------------------------------------------------------------------------------

def offsets_from_lengths(lengths) -> np.ndarray:
    """Offsets of a ragged batch: start at 0, and every sequence appends its length to the end
    of the previous one. Returns int64 [B+1]."""
    offsets = [0]
    for n in lengths:
        n = int(n)
        if n < 0:
            raise ValueError("negative sequence length")
        offsets.append(offsets[-1] + n)
    return np.asarray(offsets, dtype=np.int64)


def split_by_offsets(values, offsets):
    """Sequence i is values[offsets[i]:offsets[i+1]]."""
    return [values[int(offsets[i]):int(offsets[i + 1])] for i in range(len(offsets) - 1)]


def packing_counts(lengths):
    """Token positions when every sequence is padded to the longest one, token positions when the
    sequences are stored ragged, and the dense/ragged pair-work ratio B*max(n)^2 / sum(n^2)
    ('HSTU scale', section 不同长度不是边角问题)."""
    lengths = [int(n) for n in lengths]
    padded = len(lengths) * max(lengths)
    ragged = sum(lengths)
    pair_ratio = len(lengths) * max(lengths) ** 2 / sum(n * n for n in lengths)
    return padded, ragged, pair_ratio


# ------------------------------------------------------------------------------------------------
# Segment IDs (候选隔离注意力掩码, section 段 ID：掩码的表达方式)
# ------------------------------------------------------------------------------------------------

def attention_segment_ids(row_len: int, candidate_start_offset: int, padding_mask=None,
                          attend_padded_history: bool = False) -> np.ndarray:
    """Segment IDs of one row.

    is_candidate = idx >= candidate_start_offset; valid = padding_mask, or padding_mask OR NOT
    is_candidate when attend_padded_history; segment = valid ? (is_candidate ? -1 : 1) : 0.
    ``padding_mask`` is True for real tokens; None means every token is real.
    """
    idx = np.arange(int(row_len))
    is_candidate = idx >= int(candidate_start_offset)
    if padding_mask is None:
        valid = np.ones(int(row_len), dtype=bool)
    else:
        valid = np.asarray(padding_mask).astype(bool)
    if attend_padded_history:
        valid = np.logical_or(valid, np.logical_not(is_candidate))
    return np.where(valid, np.where(is_candidate, SEG_CANDIDATE, SEG_HISTORY),
                    SEG_PADDING).astype(np.int8)


def segment_ids(offsets, cand_start, valid=None, attend_padded_history: bool = False) -> np.ndarray:
    """Segment IDs of a packed batch: the per-row rule applied to each user's row
    [offsets[b], offsets[b+1]) with its row-relative candidate start."""
    offsets = np.asarray(offsets, dtype=np.int64)
    B = offsets.shape[0] - 1
    T = int(offsets[-1])
    out = np.zeros(T, dtype=np.int8)
    for b in range(B):
        s, e = int(offsets[b]), int(offsets[b + 1])
        pm = None if valid is None else np.asarray(valid[s:e]).astype(bool)
        out[s:e] = attention_segment_ids(e - s, int(cand_start[b]), pm, attend_padded_history)
    return out


# ------------------------------------------------------------------------------------------------
# Bounds (候选隔离注意力掩码, section 段 ID：掩码的表达方式)
# ------------------------------------------------------------------------------------------------

def bounds_from_segment_ids(seg, offsets):
    """Per user b: [hist_lo, hist_hi) spans the positions with segment 1 and [cand_lo, cand_hi)
    the positions with segment -1, as absolute packed indices.

    Empty sets: hist_lo = hist_hi = offsets[b]; cand_lo = cand_hi = offsets[b+1].
    Also returns ``layout_ok[b]``: False when a history position follows a candidate position in
    the row, which breaks the [prefix | history | candidates] order.
    """
    seg = np.asarray(seg)
    offsets = np.asarray(offsets, dtype=np.int64)
    B = offsets.shape[0] - 1
    hist_lo = np.zeros(B, dtype=np.int64)
    hist_hi = np.zeros(B, dtype=np.int64)
    cand_lo = np.zeros(B, dtype=np.int64)
    cand_hi = np.zeros(B, dtype=np.int64)
    layout_ok = np.ones(B, dtype=bool)
    for b in range(B):
        s, e = int(offsets[b]), int(offsets[b + 1])
        row = seg[s:e]
        h = np.nonzero(row == SEG_HISTORY)[0]
        c = np.nonzero(row == SEG_CANDIDATE)[0]
        if h.size:
            hist_lo[b], hist_hi[b] = s + h[0], s + h[-1] + 1
        else:
            hist_lo[b] = hist_hi[b] = s
        if c.size:
            cand_lo[b], cand_hi[b] = s + c[0], s + c[-1] + 1
        else:
            cand_lo[b] = cand_hi[b] = e
        if h.size and c.size and h[-1] > c[0]:
            layout_ok[b] = False
    return hist_lo, hist_hi, cand_lo, cand_hi, layout_ok


# ------------------------------------------------------------------------------------------------
# Mask (候选隔离注意力掩码, sections 段 ID：掩码的表达方式 and 掩码长什么样)
# ------------------------------------------------------------------------------------------------

def history_candidate_mask(seg_row) -> np.ndarray:
    """Explicit [L, L] boolean mask of one user's row: mask[q, kv] is True when q may attend kv.

    history_mask        = kv_is_history & (q_is_history | q_is_candidate)
    candidate_self_mask = q_is_candidate & kv_is_candidate & (q_pos == kv_pos)
    mask                = history_mask | candidate_self_mask
    """
    seg_row = np.asarray(seg_row)
    L = seg_row.shape[0]
    q_is_history = (seg_row == SEG_HISTORY)[:, None]
    q_is_candidate = (seg_row == SEG_CANDIDATE)[:, None]
    kv_is_history = (seg_row == SEG_HISTORY)[None, :]
    kv_is_candidate = (seg_row == SEG_CANDIDATE)[None, :]
    q_pos = np.arange(L)[:, None]
    kv_pos = np.arange(L)[None, :]
    history_mask = kv_is_history & (q_is_history | q_is_candidate)
    candidate_self_mask = q_is_candidate & kv_is_candidate & (q_pos == kv_pos)
    return history_mask | candidate_self_mask


# ------------------------------------------------------------------------------------------------
# Attention
# ------------------------------------------------------------------------------------------------

def _as_f64(x) -> np.ndarray:
    """bf16/fp32 torch tensor or array -> fp64 numpy (exact upcast)."""
    try:
        import torch  # local import: the oracle only needs torch to read tensors
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def masked_softmax_attention(q, k, v, mask, scale: float) -> np.ndarray:
    """Softmax attention of one user's row under an explicit mask.

    q, k, v: [L, H, d]; mask: [L, L] bool. For each head: S = scale * Q K^T, masked entries set to
    -inf, row-wise max-subtracted softmax, O = P V. Rows without any visible key output 0.
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    L, H, d = q.shape
    out = np.zeros((L, H, v.shape[2]), dtype=np.float64)
    if L == 0:
        return out
    has_key = mask.any(axis=1)
    for h in range(H):
        S = scale * (q[:, h, :] @ k[:, h, :].T)
        S = np.where(mask, S, -np.inf)
        m = np.where(has_key, S.max(axis=1, initial=-np.inf), 0.0)
        P = np.where(mask, np.exp(S - m[:, None]), 0.0)
        denom = P.sum(axis=1)
        P = P / np.where(has_key, denom, 1.0)[:, None]
        out[:, h, :] = P @ v[:, h, :]
    out[~has_key] = 0.0
    return out


def jagged_cand_attn(q, k, v, offsets, seg, scale: float, mask_fn=history_candidate_mask,
                     users=None) -> np.ndarray:
    """Jagged candidate-isolated attention over a packed batch (fp64 result [T, H, d]).

    For each user b with row [offsets[b], offsets[b+1]), build the explicit mask from the row's
    segment IDs and run masked softmax attention; no position reads across a user boundary.
    ``users`` restricts the computation to a subset of users (other rows stay 0).
    """
    offsets = np.asarray(offsets, dtype=np.int64)
    seg = np.asarray(seg)
    T = int(offsets[-1])
    out = np.zeros((T, q.shape[1], v.shape[2]), dtype=np.float64)
    B = offsets.shape[0] - 1
    for b in (range(B) if users is None else users):
        s, e = int(offsets[b]), int(offsets[b + 1])
        if e == s:
            continue
        mask = mask_fn(seg[s:e])
        out[s:e] = masked_softmax_attention(q[s:e], k[s:e], v[s:e], mask, scale)
    return out


def jagged_cand_attn_rows(q, k, v, offsets, seg, scale: float, rows) -> np.ndarray:
    """Output rows ``rows`` (absolute packed indices) of ``jagged_cand_attn``, computed one by one
    from each row's own user (for sampling outputs of workloads too large to compute whole)."""
    offsets = np.asarray(offsets, dtype=np.int64)
    seg = np.asarray(seg)
    rows = np.asarray(rows, dtype=np.int64)
    H, dv = q.shape[1], v.shape[2]
    out = np.zeros((rows.shape[0], H, dv), dtype=np.float64)
    users = np.searchsorted(offsets, rows, side="right") - 1
    for b in np.unique(users):
        s, e = int(offsets[b]), int(offsets[b + 1])
        sel = np.nonzero(users == b)[0]
        rel = rows[sel] - s
        mask = history_candidate_mask(seg[s:e])[rel]
        out[sel] = masked_softmax_attention(q[rows[sel]], k[s:e], v[s:e], mask, scale)
    return out


def cand_only_attn(cq, ck, cv, cand_offsets, hk, hv, hist_offsets, hist_seg, scale: float,
                   mask_fn=history_candidate_mask, users=None, cand_rows=None) -> np.ndarray:
    """Candidate-only layer: candidate queries over frozen history K/V plus their own K/V.

    Evaluated through the full-layer fallback (候选隔离注意力掩码, section 只更新候选的末尾层):
    each user's row is [history | candidates], with history segments taken from ``hist_seg``
    (1 = valid, 0 = padding; None = all valid) and candidates marked -1; the full mask runs over
    the row and only the candidate rows are kept.

    ``cand_rows`` (absolute candidate indices) returns only those rows, in that order; the row of
    user b is then [history | the requested candidates of b]. This relies on candidate isolation
    (a candidate's output does not depend on the other candidates), which the oracle's own pins
    check by adding and removing candidates.
    """
    coff = np.asarray(cand_offsets, dtype=np.int64)
    hoff = np.asarray(hist_offsets, dtype=np.int64)
    B = coff.shape[0] - 1
    Th = int(hoff[-1])
    hseg = (np.ones(Th, dtype=np.int8) if hist_seg is None
            else np.asarray(hist_seg).astype(np.int8))
    H, dv = cq.shape[1], cv.shape[2]
    if cand_rows is not None:
        cand_rows = np.asarray(cand_rows, dtype=np.int64)
        groups = {}
        users_of = np.searchsorted(coff, cand_rows, side="right") - 1
        for i, b in enumerate(users_of):
            groups.setdefault(int(b), []).append(i)
        out = np.zeros((cand_rows.shape[0], H, dv), dtype=np.float64)
    else:
        groups = {b: None for b in (range(B) if users is None else users)}
        out = np.zeros((int(coff[-1]), H, dv), dtype=np.float64)
    for b, sel in groups.items():
        hs, he = int(hoff[b]), int(hoff[b + 1])
        if sel is None:
            rows = np.arange(int(coff[b]), int(coff[b + 1]))
            dst = rows
        else:
            rows = cand_rows[sel]
            dst = np.asarray(sel)
        if rows.size == 0:
            continue
        n_h = he - hs
        k_cat = np.concatenate([_as_f64(hk[hs:he]), _as_f64(ck[rows])], axis=0)
        v_cat = np.concatenate([_as_f64(hv[hs:he]), _as_f64(cv[rows])], axis=0)
        seg_cat = np.concatenate([hseg[hs:he], np.full(rows.size, SEG_CANDIDATE, np.int8)])
        mask = mask_fn(seg_cat)
        q_rows = _as_f64(cq[rows])
        out[dst] = masked_softmax_attention(q_rows, k_cat, v_cat, mask[n_h:], scale)
    return out


# ------------------------------------------------------------------------------------------------
# Work counting
# ------------------------------------------------------------------------------------------------

def allowed_pairs(offsets, seg, mask_fn=history_candidate_mask) -> int:
    """Number of (query, key) pairs the mask allows, summed over users (counted from the explicit
    mask). Effective attention FLOPs are 4 * d * H times this count (2 for QK^T, 2 for PV)."""
    offsets = np.asarray(offsets, dtype=np.int64)
    total = 0
    for b in range(offsets.shape[0] - 1):
        s, e = int(offsets[b]), int(offsets[b + 1])
        if e > s:
            total += int(mask_fn(np.asarray(seg)[s:e]).sum())
    return total


def work_items(offsets, seg, H: int, tile_m: int = 256, tile_n: int = 128):
    """The set of (user, head, query block) items a tiled kernel must process, with each item's
    cost in key tiles over the user's history interval. Used to check the GPU work queue holds
    exactly these items (any order of equal costs, non-increasing cost)."""
    hist_lo, hist_hi, _, _, _ = bounds_from_segment_ids(seg, offsets)
    offsets = np.asarray(offsets, dtype=np.int64)
    items = []
    for b in range(offsets.shape[0] - 1):
        L = int(offsets[b + 1] - offsets[b])
        n_q = -(-L // tile_m)
        n_kv = -(-int(hist_hi[b] - hist_lo[b]) // tile_n)
        for h in range(H):
            for t in range(n_q):
                items.append((b, h, t, n_kv))
    return items
