"""Seeded synthetic jagged batches shaped like the pages' workloads.

Layout of one user row (候选隔离注意力掩码, section 为什么需要它): ``[user prefix | history | candidates]``.
Rows are packed back to back, token-major: ``q, k, v`` are ``[T, H, d]`` bf16 tensors on the CPU.

Recipe (the same for every workload):
  * lengths come from ``numpy.random.default_rng(seed)``;
  * tensors are drawn from ``torch.Generator().manual_seed(seed)`` as fp32 N(0, 1), in the order
    stated by each builder, then cast to bf16 with round-to-nearest-even (``Tensor.to``);
  * padding tokens (``valid == 0``) are appended after the last real history token and before the
    first candidate, unless a test asks for another placement through ``custom_batch``.

Nothing here computes offsets, segment IDs, bounds or attention: callers do that on their own side.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional, Sequence

import numpy as np
import torch


@dataclass
class Batch:
    """A jagged batch for the full candidate-isolated attention.

    row_lengths[b]  rows of user b (prefix + history + padding + candidates), int64.
    cand_start[b]   row-relative index of the first candidate (== row_lengths[b] - n_cand[b]).
    valid           uint8 [T] padding mask (1 = real token) or None when no token is padding.
    q, k, v         bf16 [T, H, d] on the CPU.
    """

    name: str
    row_lengths: np.ndarray
    cand_start: np.ndarray
    valid: Optional[np.ndarray]
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    H: int
    d: int
    seed: int
    prefix: np.ndarray = field(default=None)
    hist_real: np.ndarray = field(default=None)
    hist_rows: np.ndarray = field(default=None)
    n_cand: np.ndarray = field(default=None)

    @property
    def B(self) -> int:
        return int(self.row_lengths.shape[0])

    @property
    def T(self) -> int:
        return int(self.q.shape[0])

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.d))


@dataclass
class CandOnlyBatch:
    """Inputs of the candidate-only layer (候选隔离注意力掩码, section 只更新候选的末尾层).

    hist_lengths[b] rows of user b's frozen history K/V (prefix + history [+ padding]).
    hist_valid      uint8 [Th] or None (all rows valid).
    cand_counts[b]  candidates of user b.
    cq, ck, cv      bf16 [Nc, H, d]: the candidates' own query, key and value.
    hk, hv          bf16 [Th, H, d]: frozen history keys and values.
    """

    name: str
    hist_lengths: np.ndarray
    hist_valid: Optional[np.ndarray]
    cand_counts: np.ndarray
    cq: torch.Tensor
    ck: torch.Tensor
    cv: torch.Tensor
    hk: torch.Tensor
    hv: torch.Tensor
    H: int
    d: int
    seed: int

    @property
    def B(self) -> int:
        return int(self.cand_counts.shape[0])

    @property
    def Nc(self) -> int:
        return int(self.cq.shape[0])

    @property
    def Th(self) -> int:
        return int(self.hk.shape[0])

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.d))


def _draw(gen: torch.Generator, rows: int, H: int, d: int) -> torch.Tensor:
    return torch.randn(rows, H, d, generator=gen, dtype=torch.float32).to(torch.bfloat16)


def custom_batch(
    hist_lengths: Sequence[int],
    prefix: int | Sequence[int],
    n_cand: int | Sequence[int],
    H: int,
    d: int,
    seed: int = 0,
    pad_hist_to: Optional[int] = None,
    valid_override: Optional[np.ndarray] = None,
    name: str = "custom",
) -> Batch:
    """Build a batch from per-user sizes.

    ``pad_hist_to``: pad each history (prefix excluded) up to a multiple of this value with
    padding tokens appended after the real history. ``valid_override``: an explicit uint8 [T]
    padding mask that replaces the generated one (used by tests that place holes elsewhere).
    Tensors are drawn q, then k, then v.
    """
    hist_real = np.asarray(hist_lengths, dtype=np.int64)
    B = hist_real.shape[0]
    pre = np.broadcast_to(np.asarray(prefix, dtype=np.int64), (B,)).copy()
    nc = np.broadcast_to(np.asarray(n_cand, dtype=np.int64), (B,)).copy()
    if pad_hist_to:
        m = int(pad_hist_to)
        hist_rows = ((hist_real + m - 1) // m) * m
    else:
        hist_rows = hist_real.copy()
    row_lengths = pre + hist_rows + nc
    cand_start = pre + hist_rows
    T = int(row_lengths.sum())
    valid = None
    if pad_hist_to and np.any(hist_rows != hist_real):
        valid = np.ones(T, dtype=np.uint8)
        base = 0
        for b in range(B):
            lo = base + int(pre[b] + hist_real[b])
            hi = base + int(pre[b] + hist_rows[b])
            valid[lo:hi] = 0
            base += int(row_lengths[b])
    if valid_override is not None:
        valid = np.asarray(valid_override, dtype=np.uint8).copy()
        assert valid.shape == (T,)
    gen = torch.Generator().manual_seed(int(seed))
    q = _draw(gen, T, H, d)
    k = _draw(gen, T, H, d)
    v = _draw(gen, T, H, d)
    return Batch(name, row_lengths, cand_start, valid, q, k, v, int(H), int(d), int(seed),
                 pre, hist_real, hist_rows, nc)


def custom_cand_only(
    hist_lengths: Sequence[int],
    cand_counts: Sequence[int],
    H: int,
    d: int,
    seed: int = 1,
    hist_valid: Optional[np.ndarray] = None,
    name: str = "custom_cand_only",
) -> CandOnlyBatch:
    """Build candidate-only inputs. Tensors are drawn hk, hv, cq, ck, cv in that order."""
    hl = np.asarray(hist_lengths, dtype=np.int64)
    cc = np.asarray(cand_counts, dtype=np.int64)
    assert hl.shape == cc.shape
    Th = int(hl.sum())
    Nc = int(cc.sum())
    gen = torch.Generator().manual_seed(int(seed))
    hk = _draw(gen, Th, H, d)
    hv = _draw(gen, Th, H, d)
    cq = _draw(gen, Nc, H, d)
    ck = _draw(gen, Nc, H, d)
    cv = _draw(gen, Nc, H, d)
    hvld = None if hist_valid is None else np.asarray(hist_valid, dtype=np.uint8).copy()
    return CandOnlyBatch(name, hl, hvld, cc, cq, ck, cv, hk, hv, int(H), int(d), int(seed))


@dataclass
class StackBatch:
    """Inputs of a layer stack over a jagged batch.

    ``batch`` gives the row layout only (its small q, k, v are not used by the stack); ``x`` is the
    bf16 [T, D] input of the first layer (D = H d) and ``weights`` one (Wq, Wk, Wv, Wo) bf16 [D, D]
    tuple per layer, laid out so that a projection is ``x @ W``.
    """

    batch: Batch
    x: torch.Tensor
    weights: list
    n_cand_only: int
    H: int
    d: int

    @property
    def D(self) -> int:
        return int(self.x.shape[1])

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.d))


def custom_stack(hist_lengths: Sequence[int], prefix, n_cand, H: int, d: int, n_layers: int,
                 n_cand_only: int, seed: int = 0, pad_hist_to: Optional[int] = None,
                 valid_override: Optional[np.ndarray] = None, name: str = "custom_stack"
                 ) -> StackBatch:
    """Row layout as ``custom_batch``; then, from a second generator seeded ``seed + 1000``, the
    input x ~ N(0, 1) and, layer by layer, Wq, Wk, Wv ~ N(0, 1/D) and Wo ~ N(0, 1/(D n_layers))
    (fp32, cast to bf16).

    The pages describe no normalisation inside a layer, so nothing resets the residual stream's
    scale: with Wo ~ N(0, 1/D) each layer adds roughly its own variance (attention averages value
    rows whose variance is the stream's), the states grow about 2x in variance per layer, and by
    the eighth layer the scores are so large that softmax is nearly an argmax, where one-ulp
    rounding differences pick other keys. Scaling Wo by 1/sqrt(n_layers) bounds the growth by a
    factor of about e over the whole stack and keeps the scores of order one."""
    b = custom_batch(hist_lengths, prefix, n_cand, H=1, d=16, seed=seed, pad_hist_to=pad_hist_to,
                     valid_override=valid_override, name=name)
    D = H * d
    gen = torch.Generator().manual_seed(int(seed) + 1000)
    x = torch.randn(b.T, D, generator=gen, dtype=torch.float32).to(torch.bfloat16)
    weights = []
    for _ in range(n_layers):
        w = [torch.randn(D, D, generator=gen, dtype=torch.float32) / float(np.sqrt(D))
             for _ in range(4)]
        w[3] = w[3] / float(np.sqrt(n_layers))
        weights.append(tuple(t.to(torch.bfloat16) for t in w))
    return StackBatch(b, x, weights, int(n_cand_only), int(H), int(d))


# ---------------------------------------------------------------------------------------------
# The five named workloads.
# ---------------------------------------------------------------------------------------------

def tiny() -> Batch:
    """3 users, histories [2, 5, 1] (the worked example of 'HSTU scale', section
    手算 padding 的浪费与 offset), 1 prefix token and 3 candidates each; H=2, d=16, seed 0."""
    return custom_batch([2, 5, 1], prefix=1, n_cand=3, H=2, d=16, seed=0, name="tiny")


def three_users() -> Batch:
    """Histories [10, 100, 1000] ('HSTU scale', section 不同长度不是边角问题), 2 prefix tokens,
    32 candidates; history padded to a multiple of 8 with padding tokens; H=4, d=64, seed 0."""
    return custom_batch([10, 100, 1000], prefix=2, n_cand=32, H=4, d=64, seed=0, pad_hist_to=8,
                        name="three_users")


def users256_history_lengths(seed: int = 0) -> np.ndarray:
    """History lengths of the 256-user workload.

    floor(lognormal(ln 280, sigma=1)) clipped to [0, 4096]; users whose index is a multiple of 64
    are forced empty and user 1 is forced to the 4096 cap, so that both edges are exercised.
    """
    rng = np.random.default_rng(seed)
    n = np.floor(rng.lognormal(mean=np.log(280.0), sigma=1.0, size=256))
    n = np.clip(n, 0, 4096).astype(np.int64)
    n[::64] = 0
    n[1] = 4096
    return n


def lognormal_history_lengths(n_users: int, seed: int = 0) -> np.ndarray:
    """History lengths of a batch of n_users users drawn like the 256-user workload:
    floor(lognormal(ln 280, sigma=1)) clipped to [0, 4096], users whose index is a multiple of 64
    empty and user 1 at the 4096 cap."""
    rng = np.random.default_rng(seed)
    n = np.floor(rng.lognormal(mean=np.log(280.0), sigma=1.0, size=int(n_users)))
    n = np.clip(n, 0, 4096).astype(np.int64)
    n[::64] = 0
    if n_users > 1:
        n[1] = 4096
    return n


def users_batch(hist_lengths: Sequence[int], users: Sequence[int], prefix: int, n_cand: int,
                H: int, d: int, seed: int, name: str = "users") -> Batch:
    """The rows of the listed users of a larger batch (histories ``hist_lengths``, no padding), as a
    batch of their own, in the order listed. Each user's Q, K, V are drawn, in that order, from a
    generator of its own, ``torch.Generator().manual_seed(seed * 1000003 + user)``, so that a
    process that owns some of the users draws only theirs and every process draws the same rows
    for the same user."""
    users = [int(u) for u in users]
    n = np.asarray(hist_lengths, dtype=np.int64)[users] if users else np.zeros(0, np.int64)
    B = len(users)
    pre = np.full(B, int(prefix), dtype=np.int64)
    nc = np.full(B, int(n_cand), dtype=np.int64)
    row_lengths = pre + n + nc
    qs, ks, vs = [], [], []
    for u, L in zip(users, row_lengths):
        gen = torch.Generator().manual_seed(int(seed) * 1000003 + u)
        qs.append(_draw(gen, int(L), H, d))
        ks.append(_draw(gen, int(L), H, d))
        vs.append(_draw(gen, int(L), H, d))
    cat = (lambda xs: torch.cat(xs) if xs else torch.zeros(0, H, d, dtype=torch.bfloat16))
    return Batch(name, row_lengths, pre + n, None, cat(qs), cat(ks), cat(vs), int(H), int(d),
                 int(seed), pre, n.copy(), n.copy(), nc)


def users256(H: int = 8, d: int = 128) -> Batch:
    """256 users, lognormal histories (median 280), 4 prefix tokens, 64 candidates each;
    H=8, d=128, seed 0."""
    n = users256_history_lengths(0)
    return custom_batch(n, prefix=4, n_cand=64, H=H, d=d, seed=0, name="users256")


def cand_only256() -> CandOnlyBatch:
    """Candidate-only layer over the 256-user histories (4 prefix + history tokens as frozen K/V),
    512 candidates per user with their own Q/K/V; H=8, d=128, seed 1."""
    n = users256_history_lengths(0)
    return custom_cand_only(n + 4, np.full(256, 512), H=8, d=128, seed=1, name="cand_only256")


def retrieval() -> CandOnlyBatch:
    """Retrieval-shaped candidate-only attention: 16 requests x (240 user-side tokens as K/V,
    40,000 single-token candidates); H=4, d=32 (D = 128), seed 2."""
    return custom_cand_only(np.full(16, 240), np.full(16, 40000), H=4, d=32, seed=2,
                            name="retrieval")


def stack_users256() -> StackBatch:
    """The 256-user rows (as ``users256``) through 8 layers whose last 2 are candidate-only, as in
    the pages' flagship ranking configuration; H=8, d=128 (D = 1024), seed 0."""
    n = users256_history_lengths(0)
    return custom_stack(n, prefix=4, n_cand=64, H=8, d=128, n_layers=8, n_cand_only=2, seed=0,
                        name="stack_users256")


WORKLOADS = {
    "tiny": tiny,
    "three_users": three_users,
    "users256": users256,
    "cand_only256": cand_only256,
    "retrieval": retrieval,
}


def make_workload(name: str):
    return WORKLOADS[name]()


def upstream_grad(shape, seed: int) -> torch.Tensor:
    """A seeded upstream gradient dO for the backward pass: fp32 N(0, 1) from
    ``torch.Generator().manual_seed(seed)``, cast to bf16."""
    gen = torch.Generator().manual_seed(int(seed))
    return torch.randn(*shape, generator=gen, dtype=torch.float32).to(torch.bfloat16)


@dataclass
class UgBatch:
    """Inputs of UG-Sep's masked cross-attention (UG-Sep page, section 分离残差连接): per sample,
    T_out query tokens (the Mixup + PFFN output, the first c_u of them U-tokens) attend to T_in
    key/value tokens (the layer input, the first n_u of them U-tokens).

    q, residual  bf16 [B, T_out, H, d]
    k, v         bf16 [B, T_in, H, d]
    """

    name: str
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    residual: Optional[torch.Tensor]
    c_u: int
    n_u: int
    seed: int

    @property
    def B(self) -> int:
        return int(self.q.shape[0])

    @property
    def T_out(self) -> int:
        return int(self.q.shape[1])

    @property
    def T_in(self) -> int:
        return int(self.k.shape[1])

    @property
    def H(self) -> int:
        return int(self.q.shape[2])

    @property
    def d(self) -> int:
        return int(self.q.shape[3])

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.d))


def custom_ug(B: int, T_out: int, T_in: int, c_u: int, n_u: int, H: int, d: int, seed: int = 0,
              residual: bool = True, name: str = "ug_custom") -> UgBatch:
    """Q, K, V (and the residual) drawn in that order from ``torch.Generator().manual_seed(seed)``,
    fp32 N(0, 1) cast to bf16."""
    gen = torch.Generator().manual_seed(int(seed))
    q = _draw(gen, B * T_out, H, d).reshape(B, T_out, H, d)
    k = _draw(gen, B * T_in, H, d).reshape(B, T_in, H, d)
    v = _draw(gen, B * T_in, H, d).reshape(B, T_in, H, d)
    res = _draw(gen, B * T_out, H, d).reshape(B, T_out, H, d) if residual else None
    return UgBatch(name, q, k, v, res, int(c_u), int(n_u), int(seed))


def ug_sep16k() -> UgBatch:
    """The separated-residual workload: 16,384 samples (candidates of a ranking batch), a pyramid
    layer from 32 input tokens (16 U + 16 G) to 16 output tokens (8 U + 8 G), one head of 128."""
    return custom_ug(16384, 16, 32, 8, 16, 1, 128, seed=11, name="ug_sep16k")
