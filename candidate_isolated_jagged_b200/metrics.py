"""Closed-form work counts used to turn measured times into the reported metrics.

Under the candidate-isolation mask (候选隔离注意力掩码, section 段 ID：掩码的表达方式) every
non-padding query of user b sees the n_b segment-1 keys of its row, and each of the C_b candidates
also sees itself. The allowed (query, key) pairs of user b are therefore
(n_b + C_b) * n_b + C_b, and the effective (unpadded, mask-respecting) attention FLOPs are
4 * d * H * pairs: 2 for QK^T and 2 for PV per pair and per head dimension; softmax is not counted.
"""

from __future__ import annotations

import numpy as np


def allowed_pairs_from_counts(n_seg1, n_cand) -> int:
    n = np.asarray(n_seg1, dtype=np.int64)
    c = np.asarray(n_cand, dtype=np.int64)
    return int(((n + c) * n + c).sum())


def effective_flops(pairs: int, H: int, d: int) -> float:
    return 4.0 * d * H * float(pairs)


def full_attention_bytes(T: int, H: int, d: int, out_bytes: int = 2) -> float:
    """Algorithmic HBM bytes of one full jagged attention launch: Q, K, V read once (bf16) and the
    output written once."""
    return float(T) * H * d * (3 * 2 + out_bytes)


def cand_only_bytes(Nc: int, Th_valid: int, H: int, d: int, out_bytes: int = 2) -> float:
    """Algorithmic HBM bytes of one candidate-only launch: candidate q/k/v read once, frozen history
    K/V read once, the candidate outputs written once."""
    return float(Nc) * H * d * (3 * 2 + out_bytes) + float(Th_valid) * H * d * 2 * 2


def stack_flops(n_seg1, n_cand, rows: int, D: int, H: int, n_layers: int, n_cand_only: int,
                ) -> dict:
    """Useful FLOPs of the layer stack with candidate-only tail layers (候选隔离注意力掩码, section
    只更新候选的末尾层): a full layer projects all `rows` rows four times (2 D^2 FLOPs per row and
    projection) and runs the full attention; a tail layer projects the candidates four times and
    the frozen history twice (its keys and values) and runs the candidate-only attention, where a
    candidate sees the n_b history keys and itself."""
    n = np.asarray(n_seg1, dtype=np.int64)
    c = np.asarray(n_cand, dtype=np.int64)
    d = D // H
    full_gemm = 4 * 2.0 * D * D * rows
    full_attn = effective_flops(allowed_pairs_from_counts(n, c), H, d)
    tail_gemm = 2.0 * D * D * (4 * float(c.sum()) + 2 * float(n.sum()))
    tail_attn = effective_flops(int((c * (n + 1)).sum()), H, d)
    n_full = n_layers - n_cand_only
    return {"gemm": n_full * full_gemm + n_cand_only * tail_gemm,
            "attention": n_full * full_attn + n_cand_only * tail_attn}
