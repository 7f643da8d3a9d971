"""Pins of the closed-form work counts behind the reported rooflines (candidate_isolated_jagged_b200/
metrics.py): the algorithmic bytes of a full and a candidate-only launch counted tensor by tensor,
and the layer stack's FLOPs split into projections and attention, with its candidate-only
attention term equal to the oracle's pair count over the candidate rows."""

import numpy as np

import oracle
import synth
from candidate_isolated_jagged_b200 import metrics


def test_full_attention_bytes_counts_each_tensor_once():
    T, H, d = 136194, 8, 128                       # the 256-user workload
    per_tensor = T * H * d * 2                     # one bf16 [T, H, d] tensor
    assert metrics.full_attention_bytes(T, H, d) == 4 * per_tensor == 1115701248
    assert metrics.full_attention_bytes(T, H, d, out_bytes=4) == 3 * per_tensor + T * H * d * 4


def test_cand_only_bytes_counts_each_tensor_once():
    Nc, Th, H, d = 7, 5, 2, 16
    q_k_v_out = 4 * Nc * H * d * 2                 # cq, ck, cv read, out written (bf16)
    hist = 2 * Th * H * d * 2                      # hk, hv read
    assert metrics.cand_only_bytes(Nc, Th, H, d) == q_k_v_out + hist


def test_stack_flops_split():
    b = synth.custom_batch([3, 0, 9], prefix=[1, 0, 2], n_cand=[4, 2, 0], H=2, d=8, seed=0)
    n = b.prefix + b.hist_real
    c = b.n_cand
    D, rows = b.H * b.d, b.T
    off = oracle.offsets_from_lengths(b.row_lengths)
    seg = oracle.segment_ids(off, b.cand_start, b.valid)
    pairs_full = oracle.allowed_pairs(off, seg)
    pairs_cand = pairs_full - int((n * n).sum())   # candidate rows: n keys + themselves
    full = metrics.stack_flops(n, c, rows, D, b.H, n_layers=3, n_cand_only=0)
    assert full["attention"] == 3 * metrics.effective_flops(pairs_full, b.H, b.d)
    assert full["gemm"] == 3 * 4 * 2.0 * D * D * rows
    tail = metrics.stack_flops(n, c, rows, D, b.H, n_layers=3, n_cand_only=3)
    assert tail["attention"] == 3 * metrics.effective_flops(pairs_cand, b.H, b.d)
    assert tail["gemm"] == 3 * 2.0 * D * D * (4 * c.sum() + 2 * n.sum())
    mixed = metrics.stack_flops(n, c, rows, D, b.H, n_layers=3, n_cand_only=1)
    for k in ("attention", "gemm"):
        assert np.isclose(mixed[k], (2 * full[k] + tail[k]) / 3)
