"""Shared helpers of the parity tests: move seeded inputs to the GPU, run the library through the
C ABI, and compare with the oracle under the stated tolerances."""

from __future__ import annotations

import numpy as np
import torch

import oracle

# Parity bar for bf16-in / fp32-accumulate outputs (fp32 output mode).
MAX_ABS = 1e-2
REL_L2 = 5e-3


def dev():
    return torch.device("cuda:0")


def assert_close(got, ref, what="", max_abs=MAX_ABS, rel_l2=REL_L2):
    got = got.detach().to("cpu", torch.float64).numpy() if isinstance(got, torch.Tensor) else got
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    diff = np.abs(got - ref)
    m = float(diff.max()) if diff.size else 0.0
    denom = float(np.linalg.norm(ref))
    r = float(np.linalg.norm(got - ref)) / denom if denom > 0 else float(np.linalg.norm(got - ref))
    assert m <= max_abs and r <= rel_l2, f"{what}: max_abs={m:.3e} rel_l2={r:.3e}"
    return m, r


def assert_close_bf16(got, ref, what=""):
    """bf16 outputs: |got - ref| <= 1e-2 + half a bf16 ulp of |ref| (the rounding of the store)."""
    got = got.detach().to("cpu", torch.float64).numpy()
    ref = np.asarray(ref, dtype=np.float64)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    bound = MAX_ABS + 0.5 * ulp
    assert np.all(np.abs(got - ref) <= bound), f"{what}: max excess {np.max(np.abs(got - ref) - bound):.3e}"


def offsets_tensor(lengths, idx=torch.int64):
    return torch.tensor(oracle.offsets_from_lengths(lengths), dtype=idx, device=dev())


class FullRun:
    """A batch on the GPU plus the oracle's view of it."""

    def __init__(self, batch, idx=torch.int64):
        self.b = batch
        self.off_np = oracle.offsets_from_lengths(batch.row_lengths)
        self.seg_np = oracle.segment_ids(self.off_np, batch.cand_start, batch.valid)
        self.off = torch.tensor(self.off_np, dtype=idx, device=dev())
        self.cs = torch.tensor(batch.cand_start, dtype=idx, device=dev())
        self.q = batch.q.to(dev())
        self.k = batch.k.to(dev())
        self.v = batch.v.to(dev())
        self.seg = None
        if batch.valid is not None:
            from candidate_isolated_jagged_b200 import jca
            valid = torch.tensor(batch.valid, dtype=torch.uint8, device=dev())
            self.seg = torch.empty(batch.T, dtype=torch.int8, device=dev())
            st = jca.new_status(dev())
            jca.jca_build_segment_ids(self.off, self.cs, valid, False, self.seg, st)
            jca.check_status(st)

    def run(self, out_fp32=True):
        from candidate_isolated_jagged_b200 import jca
        return jca.attention(self.q, self.k, self.v, self.off, self.cs, self.seg, out_fp32=out_fp32)

    def reference(self, users=None):
        return oracle.jagged_cand_attn(self.b.q, self.b.k, self.b.v, self.off_np, self.seg_np,
                                       self.b.scale, users=users)

    def reference_rows(self, rows):
        return oracle.jagged_cand_attn_rows(self.b.q, self.b.k, self.b.v, self.off_np, self.seg_np,
                                            self.b.scale, rows)


class CandOnlyRun:
    def __init__(self, cb, idx=torch.int64, hist_seg=None):
        self.cb = cb
        self.coff_np = oracle.offsets_from_lengths(cb.cand_counts)
        self.hoff_np = oracle.offsets_from_lengths(cb.hist_lengths)
        self.coff = torch.tensor(self.coff_np, dtype=idx, device=dev())
        self.hoff = torch.tensor(self.hoff_np, dtype=idx, device=dev())
        self.hseg_np = hist_seg
        self.hseg = None if hist_seg is None else torch.tensor(hist_seg, dtype=torch.int8,
                                                               device=dev())
        self.cq, self.ck, self.cv = (t.to(dev()) for t in (cb.cq, cb.ck, cb.cv))
        self.hk, self.hv = cb.hk.to(dev()), cb.hv.to(dev())

    def run(self, out_fp32=True):
        from candidate_isolated_jagged_b200 import jca
        return jca.cand_only(self.cq, self.ck, self.cv, self.coff, self.hk, self.hv, self.hoff,
                             self.hseg, out_fp32=out_fp32)

    def reference(self, cand_rows=None):
        cb = self.cb
        return oracle.cand_only_attn(cb.cq, cb.ck, cb.cv, self.coff_np, cb.hk, cb.hv, self.hoff_np,
                                     self.hseg_np, cb.scale, cand_rows=cand_rows)


def sample_rows(offsets, per_user=3, seed=0, extra=()):
    """Rows to check on large workloads: first, last and random rows of every user."""
    rng = np.random.default_rng(seed)
    rows = set(int(x) for x in extra)
    for b in range(len(offsets) - 1):
        s, e = int(offsets[b]), int(offsets[b + 1])
        if e == s:
            continue
        rows.update({s, e - 1})
        rows.update(int(x) for x in rng.integers(s, e, size=per_user))
    return np.asarray(sorted(rows), dtype=np.int64)


def seqpack_layout(batch):
    """The rows of a serving-layout batch rearranged for training with candidate packing: every
    user's prefix + history run first (split at hist_offsets), then every user's candidate run
    (split at cand_offsets, relative to the candidate block). Returns (perm, hist_offsets,
    cand_offsets): packed row i holds serving row perm[i]."""
    off = oracle.offsets_from_lengths(batch.row_lengths)
    cs = np.asarray(batch.cand_start, dtype=np.int64)
    L = np.asarray(batch.row_lengths, dtype=np.int64)
    hist = [np.arange(off[b], off[b] + cs[b]) for b in range(batch.B)]
    cand = [np.arange(off[b] + cs[b], off[b + 1]) for b in range(batch.B)]
    perm = np.concatenate(hist + cand).astype(np.int64) if batch.B else np.zeros(0, np.int64)
    return perm, oracle.offsets_from_lengths(cs), oracle.offsets_from_lengths(L - cs)
