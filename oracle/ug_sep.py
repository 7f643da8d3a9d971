"""CPU oracle of UG-Sep's masked cross-attention (the separated residual), numpy fp64.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only the tests, the smoke check and the
benchmark's CPU baseline may import it, and it imports nothing from the CUDA package.

Source: the UG-Sep page ("Compute Only Once: UG-Separated TokenMixer"), sections 分离残差连接
(separated residual connection) and UG-Separated Mixup 与 mask. In a pyramid TokenMixer the layer
output has fewer tokens than its input, so the residual is carried by a cross-attention: the
Mixup + PFFN output (T_out tokens) gives the queries, the layer input (T_in tokens) gives the keys
and values, and the mask M_UG in {0,1}^{T_out x T_in} keeps every U output position from attending
to a G input position. U tokens come first on both sides: the first c_u outputs are U-tokens (the
page's assumption after Mixup) and the first n inputs are the user-side tokens x_u (T = n + m).

The page's formulas for R and Y were lost in extraction; the reading taken here is the plain one
its variable list supports: R = softmax(scale * Q K^T restricted by M_UG) V, per sample and per
head, and Y = X_out + R when a residual is given. A U output with no U input to read (n = 0) sees
no key and outputs 0, the same reading as a padding query of the jagged path.
"""

from __future__ import annotations

import numpy as np

from .jagged_oracle import masked_softmax_attention


def ug_mask(T_out: int, T_in: int, c_u: int, n_u: int) -> np.ndarray:
    """M_UG[i, j] = not (output i is a U-token and input j is a G-token)."""
    i = np.arange(int(T_out))[:, None]
    j = np.arange(int(T_in))[None, :]
    return ~((i < int(c_u)) & (j >= int(n_u)))


def ug_cross_attn(q, k, v, c_u: int, n_u: int, scale: float, residual=None,
                  samples=None) -> np.ndarray:
    """Masked cross-attention of every sample (fp64 [B, T_out, H, d]).

    q: [B, T_out, H, d]; k, v: [B, T_in, H, d]; residual (optional): [B, T_out, H, d], added to
    the attention output. ``samples`` restricts the computation to a subset (other samples stay
    0, without the residual).
    """
    B, T_out = int(q.shape[0]), int(q.shape[1])
    T_in = int(k.shape[1])
    mask = ug_mask(T_out, T_in, c_u, n_u)
    out = np.zeros((B, T_out, q.shape[2], v.shape[3]), dtype=np.float64)
    res = None if residual is None else np.asarray(residual.double() if hasattr(residual, "double")
                                                   else residual, dtype=np.float64)
    for b in (range(B) if samples is None else samples):
        out[b] = masked_softmax_attention(q[b], k[b], v[b], mask, scale)
        if res is not None:
            out[b] = out[b] + res[b]
    return out


def ug_pairs(T_out: int, T_in: int, c_u: int, n_u: int) -> int:
    """Allowed (query, key) pairs of one sample: c_u * n + (T_out - c_u) * T_in."""
    c_u = min(int(c_u), int(T_out))
    n_u = min(int(n_u), int(T_in))
    return c_u * n_u + (int(T_out) - c_u) * int(T_in)
