"""Thin ctypes binding over libjca.so (the C ABI declared in include/jca.h).

Argument marshalling only: tensors are passed as device pointers with their sizes, the stream is
torch's current CUDA stream, and every step of the computation runs in the library's kernels.
PyTorch allocates the outputs, the workspace and the status word. There is no CPU fallback: when
the library is missing, ``lib()`` raises.
"""

from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libjca.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "jca.h")

_lib = None

c_i32, c_i64, c_f32, c_sz, c_vp = (ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t,
                                   ctypes.c_void_p)

_SIGNATURES = {
    "jca_status_string": (ctypes.c_char_p, [c_i32]),
    "jca_offsets_from_lengths": (c_i32, [c_vp, c_vp, c_i64, c_i32, c_vp, c_vp]),
    "jca_build_segment_ids": (c_i32, [c_vp, c_vp, c_vp, c_i32, c_i64, c_i64, c_i32, c_vp, c_vp,
                                      c_vp]),
    "jca_bounds_from_segment_ids": (c_i32, [c_vp, c_vp, c_i64, c_i64, c_i32, c_vp, c_vp, c_vp,
                                            c_vp, c_vp, c_vp]),
    "jca_build_work_queue": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_i32, c_i32,
                                     c_vp, c_i64, c_vp, c_vp, c_vp]),
    "jca_max_work_items": (c_i64, [c_i64, c_i64, c_i32]),
    "jca_workspace_bytes": (c_sz, [c_i64, c_i64, c_i32, c_i32]),
    "jagged_cand_attn_fwd": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_i32, c_vp, c_vp, c_vp, c_i64, c_i64,
                                     c_i32, c_i32, c_f32, c_i32, c_vp, c_sz, c_vp, c_vp]),
    "cand_only_attn_fwd": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_i32,
                                   c_i64, c_i64, c_i64, c_i32, c_i32, c_f32, c_i32, c_vp, c_sz,
                                   c_vp, c_vp]),
    "jagged_cand_attn_plan": (c_i32, [c_vp, c_vp, c_vp, c_i64, c_i64, c_i32, c_i32, c_i32, c_vp,
                                      c_sz, c_vp, c_vp]),
    "jagged_cand_attn_run": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_i32, c_vp, c_i64, c_i64, c_i32,
                                     c_i32, c_f32, c_vp, c_sz, c_vp, c_vp]),
    "cand_only_attn_plan": (c_i32, [c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_i32, c_i32, c_i32,
                                    c_vp, c_sz, c_vp, c_vp]),
    "cand_only_attn_run": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_i32, c_i64, c_i64,
                                   c_i64, c_i32, c_i32, c_f32, c_vp, c_sz, c_vp, c_vp]),
    "jca_rope_positions": (c_i32, [c_vp, c_vp, c_i64, c_i64, c_i64, c_i32, c_vp, c_vp, c_vp]),
    "jca_apply_rope": (c_i32, [c_vp, c_vp, c_vp, c_i64, c_i32, c_i32, c_f32, c_vp]),
    "jagged_cand_attn_fwd_lse": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_i32, c_vp, c_vp, c_vp, c_vp,
                                         c_i64, c_i64, c_i32, c_i32, c_f32, c_i32, c_vp, c_sz,
                                         c_vp, c_vp]),
    "jca_bwd_workspace_bytes": (c_sz, [c_i64, c_i64, c_i32, c_i32]),
    "jagged_causal_attn_fwd": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_i32, c_vp, c_i64, c_i64, c_i32,
                                       c_i32, c_f32, c_i32, c_vp, c_sz, c_vp, c_vp]),
    "ug_masked_cross_attn_fwd": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_vp, c_i32, c_i64, c_i32,
                                         c_i32, c_i32, c_i32, c_i32, c_i32, c_f32, c_vp, c_vp]),
    "jagged_cand_attn_bwd": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp,
                                     c_i32, c_vp, c_vp, c_vp, c_i64, c_i64, c_i32, c_i32, c_f32,
                                     c_i32, c_vp, c_sz, c_vp, c_vp]),
    "jca_rope_attn_workspace_bytes": (c_sz, [c_i64, c_i64, c_i32, c_i32]),
    "jagged_cand_attn_rope_fwd": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_i32, c_vp, c_vp, c_vp, c_i64,
                                          c_i64, c_i32, c_i32, c_f32, c_i64, c_f32, c_i32, c_vp,
                                          c_sz, c_vp, c_vp]),
    "jca_seqpack_workspace_bytes": (c_sz, [c_i64, c_i64, c_i64, c_i32, c_i32]),
    "jca_seqpack_bwd_workspace_bytes": (c_sz, [c_i64, c_i64, c_i64, c_i32, c_i32]),
    "jagged_cand_attn_seqpack_fwd": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_i32, c_vp, c_vp, c_vp, c_vp,
                                             c_i64, c_i64, c_i64, c_i32, c_i32, c_f32, c_i32, c_vp,
                                             c_sz, c_vp, c_vp]),
    "jagged_cand_attn_seqpack_bwd": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_i32, c_vp, c_vp, c_vp, c_vp,
                                             c_vp, c_i32, c_vp, c_vp, c_vp, c_i64, c_i64, c_i64,
                                             c_i32, c_i32, c_f32, c_i32, c_vp, c_sz, c_vp, c_vp]),
    "jca_stack_workspace_bytes": (c_sz, [c_i64, c_i64, c_i64, c_i64, c_i32, c_i32]),
    "jca_stack_fwd": (c_i32, [c_vp, c_vp, c_vp, c_i32, c_i32, c_vp, c_vp, c_vp, c_i64, c_i64, c_i64,
                              c_i64, c_i32, c_i32, c_f32, c_i64, c_f32, c_i32, c_vp, c_sz, c_vp,
                              c_vp]),
    "jca_noalloc_scratch_bytes": (c_sz, []),
    "jca_noalloc_prepare": (c_i32, []),
    "jca_user_tile_cost": (c_i64, [c_i64, c_i64]),
    "jca_selftest_wait_timeout": (c_i32, [c_vp, c_vp]),
    "jca_shard_users": (c_i32, [c_vp, c_vp, c_i64, c_i32, c_vp, c_vp]),
    "jagged_cand_attn_fwd_noalloc": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_i32, c_vp, c_vp, c_vp,
                                             c_i64, c_i64, c_i32, c_i32, c_f32, c_i32, c_vp,
                                             c_vp]),
}


class JcaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = int(code)
        super().__init__(f"{where}: {status_string(code)} (code {code})")


def lib(path: Optional[str] = None):
    """Load libjca.so (once). Raises when it is missing: there is no fallback."""
    global _lib
    if path is not None:
        return _load(path)
    if _lib is None:
        _lib = _load(LIB_PATH)
    return _lib


def _load(path: str):
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           f"`python -m candidate_isolated_jagged_b200.build`")
    L = ctypes.CDLL(path)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


def header_functions(path: str = HEADER_PATH):
    """Names of the functions declared in include/jca.h."""
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\(", text,
                                 flags=re.M)))


def status_string(code: int) -> str:
    return lib().jca_status_string(int(code)).decode()


# ------------------------------------------------------------------------------------------------
# Marshalling helpers
# ------------------------------------------------------------------------------------------------

def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    return ctypes.c_void_p(handle)


def _idx_bits(t: torch.Tensor) -> int:
    if t.dtype == torch.int32:
        return 32
    if t.dtype == torch.int64:
        return 64
    raise TypeError(f"index tensors must be int32 or int64, got {t.dtype}")


def _check(code: int, where: str) -> int:
    if code < 0:
        raise JcaError(code, where)
    return code


def new_status(device) -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


def check_status(status: torch.Tensor, where: str = "device") -> None:
    """Read the device status word (synchronises) and raise on a recorded data error."""
    code = int(status.item())
    if code != 0:
        raise JcaError(code, where)


# ------------------------------------------------------------------------------------------------
# Entry points (same names as the C ABI)
# ------------------------------------------------------------------------------------------------

def jca_offsets_from_lengths(lengths: torch.Tensor, offsets: torch.Tensor, status: torch.Tensor,
                             stream=None) -> int:
    return _check(lib().jca_offsets_from_lengths(_ptr(lengths), _ptr(offsets), lengths.numel(),
                                                 _idx_bits(lengths), _ptr(status), _stream(stream)),
                  "jca_offsets_from_lengths")


def jca_build_segment_ids(offsets, candidate_start, valid_mask, attend_padded_history: bool,
                          seg: torch.Tensor, status: torch.Tensor, stream=None) -> int:
    B = offsets.numel() - 1
    return _check(lib().jca_build_segment_ids(
        _ptr(offsets), _ptr(candidate_start), _ptr(valid_mask), int(bool(attend_padded_history)),
        B, seg.numel(), _idx_bits(offsets), _ptr(seg), _ptr(status), _stream(stream)),
        "jca_build_segment_ids")


def jca_bounds_from_segment_ids(seg, offsets, hist_lo, hist_hi, cand_lo, cand_hi, status,
                                stream=None) -> int:
    B = offsets.numel() - 1
    return _check(lib().jca_bounds_from_segment_ids(
        _ptr(seg), _ptr(offsets), B, seg.numel(), _idx_bits(offsets), _ptr(hist_lo), _ptr(hist_hi),
        _ptr(cand_lo), _ptr(cand_hi), _ptr(status), _stream(stream)), "jca_bounds_from_segment_ids")


def jca_build_work_queue(q_offsets, kv_lo, kv_hi, kv_count, q_rows: int, kv_rows: int, H: int,
                         items: torch.Tensor, n_items: torch.Tensor, status, stream=None) -> int:
    B = q_offsets.numel() - 1
    return _check(lib().jca_build_work_queue(
        _ptr(q_offsets), _ptr(kv_lo), _ptr(kv_hi), _ptr(kv_count), B, int(q_rows), int(kv_rows),
        int(H), _idx_bits(q_offsets), _ptr(items), items.numel() // 4, _ptr(n_items), _ptr(status),
        _stream(stream)), "jca_build_work_queue")


def jca_max_work_items(B: int, rows: int, H: int) -> int:
    return int(lib().jca_max_work_items(int(B), int(rows), int(H)))


def jca_workspace_bytes(B: int, rows: int, H: int, d_head: int) -> int:
    return int(lib().jca_workspace_bytes(int(B), int(rows), int(H), int(d_head)))


def jagged_cand_attn_fwd(q, k, v, out, offsets, candidate_start=None, seg=None, scale: float = 0.0,
                         workspace: Optional[torch.Tensor] = None,
                         status: Optional[torch.Tensor] = None, stream=None) -> int:
    T, H, d = q.shape
    B = offsets.numel() - 1
    if workspace is None:
        workspace = torch.empty(jca_workspace_bytes(B, T, H, d), dtype=torch.uint8, device=q.device)
    if status is None:
        status = new_status(q.device)
    out_fp32 = 1 if out.dtype == torch.float32 else 0
    return _check(lib().jagged_cand_attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), out_fp32, _ptr(offsets), _ptr(candidate_start),
        _ptr(seg), B, T, H, d, float(scale), _idx_bits(offsets), _ptr(workspace),
        workspace.numel(), _ptr(status), _stream(stream)), "jagged_cand_attn_fwd")


def cand_only_attn_fwd(cand_q, own_k, own_v, cand_offsets, hist_k, hist_v, hist_offsets, out,
                       hist_seg=None, scale: float = 0.0, workspace: Optional[torch.Tensor] = None,
                       status: Optional[torch.Tensor] = None, stream=None) -> int:
    Nc, H, d = cand_q.shape
    Th = hist_k.shape[0]
    B = cand_offsets.numel() - 1
    if workspace is None:
        workspace = torch.empty(jca_workspace_bytes(B, Nc, H, d), dtype=torch.uint8,
                                device=cand_q.device)
    if status is None:
        status = new_status(cand_q.device)
    out_fp32 = 1 if out.dtype == torch.float32 else 0
    return _check(lib().cand_only_attn_fwd(
        _ptr(cand_q), _ptr(own_k), _ptr(own_v), _ptr(cand_offsets), _ptr(hist_k), _ptr(hist_v),
        _ptr(hist_offsets), _ptr(hist_seg), _ptr(out), out_fp32, B, Nc, Th, H, d, float(scale),
        _idx_bits(cand_offsets), _ptr(workspace), workspace.numel(), _ptr(status),
        _stream(stream)), "cand_only_attn_fwd")


def jagged_cand_attn_plan(offsets, candidate_start, seg, T: int, H: int, d_head: int,
                          workspace: torch.Tensor, status: torch.Tensor, stream=None) -> int:
    B = offsets.numel() - 1
    return _check(lib().jagged_cand_attn_plan(
        _ptr(offsets), _ptr(candidate_start), _ptr(seg), B, int(T), int(H), int(d_head),
        _idx_bits(offsets), _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream)),
        "jagged_cand_attn_plan")


def jagged_cand_attn_run(q, k, v, out, seg, B: int, workspace: torch.Tensor, status: torch.Tensor,
                         scale: float = 0.0, stream=None) -> int:
    T, H, d = q.shape
    out_fp32 = 1 if out.dtype == torch.float32 else 0
    return _check(lib().jagged_cand_attn_run(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), out_fp32, _ptr(seg), int(B), T, H, d, float(scale),
        _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream)), "jagged_cand_attn_run")


def cand_only_attn_plan(cand_offsets, hist_offsets, hist_seg, Nc: int, Th: int, H: int, d_head: int,
                        workspace: torch.Tensor, status: torch.Tensor, stream=None) -> int:
    B = cand_offsets.numel() - 1
    return _check(lib().cand_only_attn_plan(
        _ptr(cand_offsets), _ptr(hist_offsets), _ptr(hist_seg), B, int(Nc), int(Th), int(H),
        int(d_head), _idx_bits(cand_offsets), _ptr(workspace), workspace.numel(), _ptr(status),
        _stream(stream)), "cand_only_attn_plan")


def cand_only_attn_run(cand_q, own_k, own_v, hist_k, hist_v, hist_seg, out, B: int,
                       workspace: torch.Tensor, status: torch.Tensor, scale: float = 0.0,
                       stream=None) -> int:
    Nc, H, d = cand_q.shape
    Th = hist_k.shape[0]
    out_fp32 = 1 if out.dtype == torch.float32 else 0
    return _check(lib().cand_only_attn_run(
        _ptr(cand_q), _ptr(own_k), _ptr(own_v), _ptr(hist_k), _ptr(hist_v), _ptr(hist_seg),
        _ptr(out), out_fp32, int(B), Nc, Th, H, d, float(scale), _ptr(workspace),
        workspace.numel(), _ptr(status), _stream(stream)), "cand_only_attn_run")


def jca_noalloc_prepare() -> int:
    """Caches the static scratch array's device address for the current device (call it before
    capturing a stream that will hold jagged_cand_attn_fwd_noalloc)."""
    return _check(lib().jca_noalloc_prepare(), "jca_noalloc_prepare")


def jagged_cand_attn_fwd_noalloc(q, k, v, out, offsets, candidate_start=None, seg=None,
                                 scale: float = 0.0, status: Optional[torch.Tensor] = None,
                                 stream=None) -> int:
    """jagged_cand_attn_fwd for callers that cannot allocate device memory at call time: the
    library uses its own fixed 8 MiB static scratch array instead of a caller workspace (see
    include/jca.h for the size limit and the sharing rules). The caller passes the int32 status
    word too (device memory it owns), so that nothing here allocates either; only the C call is
    allocation-free when called some other way."""
    T, H, d = q.shape
    B = offsets.numel() - 1
    if status is None:
        raise ValueError("jagged_cand_attn_fwd_noalloc needs a caller-owned status tensor "
                         "(new_status() once, outside the allocation-free region)")
    out_fp32 = 1 if out.dtype == torch.float32 else 0
    return _check(lib().jagged_cand_attn_fwd_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), out_fp32, _ptr(offsets), _ptr(candidate_start),
        _ptr(seg), B, T, H, d, float(scale), _idx_bits(offsets), _ptr(status), _stream(stream)),
        "jagged_cand_attn_fwd_noalloc")


def jca_selftest_wait_timeout(status, stream=None) -> int:
    """One block that runs the library's bounded pipeline wait on a barrier nothing completes:
    *status becomes JCA_STATUS_TIMEOUT (16) after about 2 s, and the context stays usable."""
    return _check(lib().jca_selftest_wait_timeout(_ptr(status), _stream(stream)),
                  "jca_selftest_wait_timeout")


def shard_users(row_lengths, n_keys, n_shards: int):
    """Host-side LPT split of a batch's users over n_shards GPUs (jca_shard_users).

    row_lengths, n_keys: per-user rows and segment-1 keys (array-likes of int). Returns
    (shard [B] int32, load [n_shards] int64) as numpy arrays."""
    import numpy as np
    rl = np.ascontiguousarray(np.asarray(row_lengths, dtype=np.int64))
    nk = np.ascontiguousarray(np.asarray(n_keys, dtype=np.int64))
    if rl.shape != nk.shape or rl.ndim != 1:
        raise ValueError("row_lengths and n_keys must be 1-D arrays of the same length")
    shard = np.empty(rl.shape[0], dtype=np.int32)
    load = np.empty(int(n_shards), dtype=np.int64)
    _check(lib().jca_shard_users(rl.ctypes.data if rl.size else None,
                                 nk.ctypes.data if nk.size else None, rl.shape[0], int(n_shards),
                                 shard.ctypes.data if shard.size else None, load.ctypes.data),
           "jca_shard_users")
    return shard, load


def user_tile_cost(row_length: int, n_keys: int) -> int:
    """Tile cost of one user (jca_user_tile_cost)."""
    return int(lib().jca_user_tile_cost(int(row_length), int(n_keys)))


def jca_rope_positions(seg, offsets, positions, history_end: int, status, stream=None) -> int:
    """Right-anchored positions (int32 [T]) of the tokens of a segment-ID array."""
    B = offsets.numel() - 1
    T = seg.numel()
    return _check(lib().jca_rope_positions(_ptr(seg), _ptr(offsets), B, T, int(history_end),
                                           _idx_bits(offsets), _ptr(positions), _ptr(status),
                                           _stream(stream)), "jca_rope_positions")


def jca_apply_rope(x, out, positions, base: float = 10000.0, stream=None) -> int:
    """Rotate the rows of a [T, H, d] bf16 tensor by their positions (out may be x)."""
    T, H, d = x.shape
    return _check(lib().jca_apply_rope(_ptr(x), _ptr(out), _ptr(positions), T, H, d, float(base),
                                       _stream(stream)), "jca_apply_rope")


def jagged_cand_attn_fwd_lse(q, k, v, out, lse, offsets, candidate_start=None, seg=None,
                             scale: float = 0.0, workspace: Optional[torch.Tensor] = None,
                             status: Optional[torch.Tensor] = None, stream=None) -> int:
    """jagged_cand_attn_fwd that also writes lse [T, H] fp32 (log of each row's softmax
    denominator; -inf for padding rows)."""
    T, H, d = q.shape
    B = offsets.numel() - 1
    if workspace is None:
        workspace = torch.empty(jca_workspace_bytes(B, T, H, d), dtype=torch.uint8, device=q.device)
    if status is None:
        status = new_status(q.device)
    out_fp32 = 1 if out.dtype == torch.float32 else 0
    return _check(lib().jagged_cand_attn_fwd_lse(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), out_fp32, _ptr(lse), _ptr(offsets),
        _ptr(candidate_start), _ptr(seg), B, T, H, d, float(scale), _idx_bits(offsets),
        _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream)),
        "jagged_cand_attn_fwd_lse")


def jagged_causal_attn_fwd(q, k, v, out, offsets, scale: float = 0.0,
                           workspace: Optional[torch.Tensor] = None,
                           status: Optional[torch.Tensor] = None, stream=None) -> int:
    """Per-user causal attention over packed sequences (row i sees rows j <= i of its user)."""
    T, H, d = q.shape
    B = offsets.numel() - 1
    if workspace is None:
        workspace = torch.empty(jca_workspace_bytes(B, T, H, d), dtype=torch.uint8, device=q.device)
    if status is None:
        status = new_status(q.device)
    out_fp32 = 1 if out.dtype == torch.float32 else 0
    return _check(lib().jagged_causal_attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), out_fp32, _ptr(offsets), B, T, H, d, float(scale),
        _idx_bits(offsets), _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream)),
        "jagged_causal_attn_fwd")


def ug_masked_cross_attn_fwd(q, k, v, out, c_u: int, n_u: int, residual=None,
                             scale: float = 0.0, status: Optional[torch.Tensor] = None,
                             stream=None) -> int:
    """UG-Sep's masked cross-attention: q [B, T_out, H, d], k and v [B, T_in, H, d] (bf16); the
    first c_u outputs read only the first n_u inputs. out [B, T_out, H, d] (bf16 or fp32) gets
    residual + R when a residual is given."""
    B, T_out, H, d = q.shape
    T_in = k.shape[1]
    if status is None:
        status = new_status(q.device)
    out_fp32 = 1 if out.dtype == torch.float32 else 0
    return _check(lib().ug_masked_cross_attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(residual), _ptr(out),
        out_fp32, B, T_out, T_in, int(c_u), int(n_u), H, d, float(scale), _ptr(status),
        _stream(stream)), "ug_masked_cross_attn_fwd")


def jca_bwd_workspace_bytes(B: int, T: int, H: int, d_head: int) -> int:
    return int(lib().jca_bwd_workspace_bytes(int(B), int(T), int(H), int(d_head)))


def jagged_cand_attn_bwd(q, k, v, out, dout, lse, dq, dk, dv, offsets, candidate_start=None,
                         seg=None, scale: float = 0.0, workspace: Optional[torch.Tensor] = None,
                         status: Optional[torch.Tensor] = None, stream=None) -> int:
    """Gradients dq, dk, dv ([T, H, d], bf16 or fp32 as the tensors given) of the jagged
    candidate-isolated attention for the upstream gradient dout."""
    T, H, d = q.shape
    B = offsets.numel() - 1
    if workspace is None:
        workspace = torch.empty(jca_bwd_workspace_bytes(B, T, H, d), dtype=torch.uint8,
                                device=q.device)
    if status is None:
        status = new_status(q.device)
    out_fp32 = 1 if out.dtype == torch.float32 else 0
    grad_fp32 = 1 if dq.dtype == torch.float32 else 0
    assert dk.dtype == dq.dtype and dv.dtype == dq.dtype
    return _check(lib().jagged_cand_attn_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), out_fp32, _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
        _ptr(dv), grad_fp32, _ptr(offsets), _ptr(candidate_start), _ptr(seg), B, T, H, d,
        float(scale), _idx_bits(offsets), _ptr(workspace), workspace.numel(), _ptr(status),
        _stream(stream)), "jagged_cand_attn_bwd")


def jca_rope_attn_workspace_bytes(B: int, T: int, H: int, d_head: int) -> int:
    return int(lib().jca_rope_attn_workspace_bytes(int(B), int(T), int(H), int(d_head)))


def jagged_cand_attn_rope_fwd(q, k, v, out, offsets, candidate_start=None, seg=None,
                              history_end: int = 0, rope_base: float = 10000.0, scale: float = 0.0,
                              workspace: Optional[torch.Tensor] = None,
                              status: Optional[torch.Tensor] = None, stream=None) -> int:
    """Jagged candidate-isolated attention with right-anchored RoPE rotated inside the kernel
    (q and k unrotated, left unchanged)."""
    T, H, d = q.shape
    B = offsets.numel() - 1
    if workspace is None:
        workspace = torch.empty(max(1, jca_rope_attn_workspace_bytes(B, T, H, d)),
                                dtype=torch.uint8, device=q.device)
    if status is None:
        status = new_status(q.device)
    out_fp32 = 1 if out.dtype == torch.float32 else 0
    return _check(lib().jagged_cand_attn_rope_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), out_fp32, _ptr(offsets), _ptr(candidate_start),
        _ptr(seg), B, T, H, d, float(scale), int(history_end), float(rope_base),
        _idx_bits(offsets), _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream)),
        "jagged_cand_attn_rope_fwd")


def jca_seqpack_workspace_bytes(B: int, Th: int, Nc: int, H: int, d_head: int) -> int:
    return int(lib().jca_seqpack_workspace_bytes(int(B), int(Th), int(Nc), int(H), int(d_head)))


def jca_seqpack_bwd_workspace_bytes(B: int, Th: int, Nc: int, H: int, d_head: int) -> int:
    return int(lib().jca_seqpack_bwd_workspace_bytes(int(B), int(Th), int(Nc), int(H),
                                                     int(d_head)))


def jagged_cand_attn_seqpack_fwd(q, k, v, out, hist_offsets, cand_offsets, seg=None, lse=None,
                                 scale: float = 0.0, workspace: Optional[torch.Tensor] = None,
                                 status: Optional[torch.Tensor] = None, stream=None,
                                 Th: Optional[int] = None) -> int:
    """Forward over the candidate-packed matrix [history runs | candidate runs] (rows [0, Th)
    split at hist_offsets, rows [Th, T) split at cand_offsets); lse [T, H] fp32 optional.
    Th (history rows) is read back from hist_offsets when not given."""
    T, H, d = q.shape
    B = hist_offsets.numel() - 1
    Th = _seqpack_th(hist_offsets) if Th is None else int(Th)
    Nc = T - Th
    if workspace is None:
        workspace = torch.empty(max(1, jca_seqpack_workspace_bytes(B, Th, Nc, H, d)),
                                dtype=torch.uint8, device=q.device)
    if status is None:
        status = new_status(q.device)
    out_fp32 = 1 if out.dtype == torch.float32 else 0
    return _check(lib().jagged_cand_attn_seqpack_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), out_fp32, _ptr(lse), _ptr(hist_offsets),
        _ptr(cand_offsets), _ptr(seg), B, Th, Nc, H, d, float(scale), _idx_bits(hist_offsets),
        _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream)),
        "jagged_cand_attn_seqpack_fwd")


def jagged_cand_attn_seqpack_bwd(q, k, v, out, dout, lse, dq, dk, dv, hist_offsets, cand_offsets,
                                 seg=None, scale: float = 0.0,
                                 workspace: Optional[torch.Tensor] = None,
                                 status: Optional[torch.Tensor] = None, stream=None,
                                 Th: Optional[int] = None) -> int:
    """Gradients dq, dk, dv over the candidate-packed matrix (see jagged_cand_attn_seqpack_fwd)."""
    T, H, d = q.shape
    B = hist_offsets.numel() - 1
    Th = _seqpack_th(hist_offsets) if Th is None else int(Th)
    Nc = T - Th
    if workspace is None:
        workspace = torch.empty(max(1, jca_seqpack_bwd_workspace_bytes(B, Th, Nc, H, d)),
                                dtype=torch.uint8, device=q.device)
    if status is None:
        status = new_status(q.device)
    out_fp32 = 1 if out.dtype == torch.float32 else 0
    grad_fp32 = 1 if dq.dtype == torch.float32 else 0
    assert dk.dtype == dq.dtype and dv.dtype == dq.dtype
    return _check(lib().jagged_cand_attn_seqpack_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), out_fp32, _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
        _ptr(dv), grad_fp32, _ptr(hist_offsets), _ptr(cand_offsets), _ptr(seg), B, Th, Nc, H, d,
        float(scale), _idx_bits(hist_offsets), _ptr(workspace), workspace.numel(), _ptr(status),
        _stream(stream)), "jagged_cand_attn_seqpack_bwd")


def _seqpack_th(hist_offsets) -> int:
    """Th = hist_offsets[B], read back to the host (the caller's layout; a device read)."""
    return int(hist_offsets[-1].item())


def jca_stack_workspace_bytes(B: int, T: int, Nc: int, Th: int, H: int, d_head: int) -> int:
    return int(lib().jca_stack_workspace_bytes(int(B), int(T), int(Nc), int(Th), int(H),
                                               int(d_head)))


def jca_stack_fwd(x, x_out, weights, n_cand_only: int, offsets, candidate_start=None, seg=None,
                  Nc: int = 0, Th: int = 0, H: int = 1, scale: float = 0.0,
                  history_end: Optional[int] = None, rope_base: float = 10000.0,
                  workspace: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                  stream=None) -> int:
    """Layer stack with candidate-only tail layers: x [T, D] bf16 -> x_out [T, D] bf16 through
    weights [n_layers, 4, D, D] bf16 (Wq, Wk, Wv, Wo per layer, x @ W). Nc / Th: total candidate and
    history tokens. history_end None turns RoPE off."""
    T, D = x.shape
    n_layers = weights.shape[0] if weights.dim() == 4 else 0
    d = D // int(H)
    B = offsets.numel() - 1
    if workspace is None:
        workspace = torch.empty(jca_stack_workspace_bytes(B, T, Nc, Th, H, d), dtype=torch.uint8,
                                device=x.device)
    if status is None:
        status = new_status(x.device)
    return _check(lib().jca_stack_fwd(
        _ptr(x), _ptr(x_out), _ptr(weights), int(n_layers), int(n_cand_only), _ptr(offsets),
        _ptr(candidate_start), _ptr(seg), B, T, int(Nc), int(Th), int(H), d, float(scale),
        -1 if history_end is None else int(history_end), float(rope_base), _idx_bits(offsets),
        _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream)), "jca_stack_fwd")


def jca_noalloc_scratch_bytes() -> int:
    return int(lib().jca_noalloc_scratch_bytes())


def jca_status_string(code: int) -> str:
    return status_string(code)


# ------------------------------------------------------------------------------------------------
# Convenience: allocate outputs with torch, call, check the status word
# ------------------------------------------------------------------------------------------------

def attention(q, k, v, offsets, candidate_start=None, seg=None, out_fp32: bool = False,
              scale: float = 0.0, check: bool = True) -> torch.Tensor:
    out = torch.empty(q.shape, dtype=torch.float32 if out_fp32 else torch.bfloat16, device=q.device)
    status = new_status(q.device)
    jagged_cand_attn_fwd(q, k, v, out, offsets, candidate_start, seg, scale, status=status)
    if check:
        check_status(status, "jagged_cand_attn_fwd")
    return out


def cand_only(cand_q, own_k, own_v, cand_offsets, hist_k, hist_v, hist_offsets, hist_seg=None,
              out_fp32: bool = False, scale: float = 0.0, check: bool = True) -> torch.Tensor:
    out = torch.empty(cand_q.shape, dtype=torch.float32 if out_fp32 else torch.bfloat16,
                      device=cand_q.device)
    status = new_status(cand_q.device)
    cand_only_attn_fwd(cand_q, own_k, own_v, cand_offsets, hist_k, hist_v, hist_offsets, out,
                       hist_seg, scale, status=status)
    if check:
        check_status(status, "cand_only_attn_fwd")
    return out
