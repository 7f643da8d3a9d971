"""CPU oracle of the ranker's layer stack with candidate-only tail layers (numpy, fp64).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only the tests, the smoke check and the
benchmark's CPU baseline may import it, and it imports nothing from the CUDA package.

What the pages fix (候选隔离注意力掩码, section 只更新候选的末尾层 and its flowchart): the stack runs its
first ``num_layers - N`` layers over whole rows [prefix | history | candidates] under the isolation
mask; the hidden states are then split into history and candidates, the history (prefix included)
is frozen, and the last N layers compute only the candidates, whose queries attend to the frozen
history K/V and to their own K/V. The flagship setting has 8 layers with N = 2. Because history
never attends to candidates (section 掩码长什么样), a history state does not depend on the candidates
at any layer. The fallback the same section gives (standard layers over the whole sequence, with
the non-candidate outputs then replaced by the frozen history states) yields the same candidate
outputs; the tests pin one against the other.

Readings (the pages describe only the attention part of a layer):

* A layer is ``x <- x + Attn(x Wq, x Wk, x Wv) Wo`` with square weights (D = H d, no bias) and,
  when a ``history_end`` is given, right-anchored RoPE on the queries and keys (section
  位置编码：候选共用一个位置); no normalisation or feed-forward block is described, so none is applied.
* ``update_user_token`` keeps the pages' default (False): prefix tokens freeze with the history.
* With ``bf16=True`` activations are rounded to bf16 where the model stores them: each projection
  output, each RoPE output, the attention output, and the residual sum ``x + a Wo`` (rounded once,
  as a GEMM with a fused residual does). With ``bf16=False`` nothing is rounded (exact fp64).
* Padding rows (segment 0) have zero attention output, so their states never change; they are not
  part of the frozen history K/V (the candidate-only layer never sees them).
"""

from __future__ import annotations

import numpy as np

from .jagged_oracle import SEG_CANDIDATE, SEG_HISTORY, _as_f64, cand_only_attn, jagged_cand_attn
from .rope import apply_rope, right_anchored_positions, round_to_bf16


def _rounder(bf16: bool):
    return round_to_bf16 if bf16 else (lambda a: np.asarray(a, dtype=np.float64))


def split_history_and_candidates(offsets, seg):
    """Split a packed batch into per-user history (segment 1) and candidate (segment -1) rows.

    Returns (hist_rows, cand_rows, hist_offsets, cand_offsets): absolute row indices in row order,
    and the offsets of each user's run in the two compact lists. Padding rows go to neither."""
    offsets = np.asarray(offsets, dtype=np.int64)
    seg = np.asarray(seg)
    hist, cand, nh, nc = [], [], [0], [0]
    for b in range(len(offsets) - 1):
        for i in range(int(offsets[b]), int(offsets[b + 1])):
            if seg[i] == SEG_HISTORY:
                hist.append(i)
            elif seg[i] == SEG_CANDIDATE:
                cand.append(i)
        nh.append(len(hist))
        nc.append(len(cand))
    return (np.asarray(hist, dtype=np.int64), np.asarray(cand, dtype=np.int64),
            np.asarray(nh, dtype=np.int64), np.asarray(nc, dtype=np.int64))


def full_layer(x, w, offsets, seg, H: int, scale: float, pos=None, bf16: bool = True):
    """One layer over whole rows; x [T, D], w = (Wq, Wk, Wv, Wo) [D, D] each."""
    r = _rounder(bf16)
    wq, wk, wv, wo = w
    T, D = x.shape
    d = D // H
    q = r(x @ wq).reshape(T, H, d)
    k = r(x @ wk).reshape(T, H, d)
    v = r(x @ wv).reshape(T, H, d)
    if pos is not None:
        q, k = r(apply_rope(q, pos)), r(apply_rope(k, pos))
    a = r(jagged_cand_attn(q, k, v, offsets, seg, scale)).reshape(T, D)
    return r(x + a @ wo)


def candidate_only_layer(xc, xh, w, cand_offsets, hist_offsets, H: int, scale: float,
                         cpos=None, hpos=None, bf16: bool = True):
    """One candidate-only layer: candidate states xc [Nc, D] over frozen history states
    xh [Th, D] (K/V = xh Wk, xh Wv); returns the new candidate states."""
    r = _rounder(bf16)
    wq, wk, wv, wo = w
    D = xc.shape[1]
    d = D // H
    cq = r(xc @ wq).reshape(-1, H, d)
    ck = r(xc @ wk).reshape(-1, H, d)
    cv = r(xc @ wv).reshape(-1, H, d)
    hk = r(xh @ wk).reshape(-1, H, d)
    hv = r(xh @ wv).reshape(-1, H, d)
    if cpos is not None:
        cq, ck = r(apply_rope(cq, cpos)), r(apply_rope(ck, cpos))
        hk = r(apply_rope(hk, hpos))
    a = r(cand_only_attn(cq, ck, cv, cand_offsets, hk, hv, hist_offsets, None, scale))
    return r(xc + a.reshape(-1, D) @ wo)


def stack_forward(x, weights, offsets, seg, H: int, n_cand_only: int, scale: float,
                  history_end=None, fallback: bool = False, bf16: bool = True):
    """The whole stack; returns the final states [T, D] (history and padding rows hold the states
    they had at the split).

    ``weights``: one (Wq, Wk, Wv, Wo) per layer; the last ``n_cand_only`` layers update only the
    candidates. ``fallback`` runs those layers as whole-row layers and restores the frozen
    non-candidate states after each, as the pages' fallback does. ``history_end`` not None turns on
    right-anchored RoPE."""
    r = _rounder(bf16)
    x = r(_as_f64(x))
    w64 = [tuple(_as_f64(m) for m in w) for w in weights]
    offsets = np.asarray(offsets, dtype=np.int64)
    seg = np.asarray(seg)
    n_layers = len(w64)
    pos = None if history_end is None else right_anchored_positions(offsets, seg, history_end)
    for layer in range(n_layers - n_cand_only):
        x = full_layer(x, w64[layer], offsets, seg, H, scale, pos, bf16)
    hist, cand, hoff, coff = split_history_and_candidates(offsets, seg)
    frozen = x.copy()
    keep = seg != SEG_CANDIDATE
    xc, xh = x[cand], frozen[hist]
    for layer in range(n_layers - n_cand_only, n_layers):
        if fallback:
            x = full_layer(x, w64[layer], offsets, seg, H, scale, pos, bf16)
            x[keep] = frozen[keep]
        else:
            xc = candidate_only_layer(xc, xh, w64[layer], coff, hoff, H, scale,
                                      None if pos is None else pos[cand],
                                      None if pos is None else pos[hist], bf16)
    if not fallback:
        x = frozen.copy()
        x[cand] = xc
    return x
