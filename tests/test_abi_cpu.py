"""C-ABI checks that need no GPU: the library loads, exports every function include/jca.h declares,
and host-side argument errors come back as negative codes before anything is launched."""

import ctypes
import os
import subprocess

import pytest

from candidate_isolated_jagged_b200 import jca

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(jca.LIB_PATH):
        from candidate_isolated_jagged_b200 import build
        build.build()
    return jca.lib()


def test_header_declares_the_entry_points():
    names = jca.header_functions()
    for n in ["jca_offsets_from_lengths", "jca_build_segment_ids", "jca_bounds_from_segment_ids",
              "jca_build_work_queue", "jca_max_work_items", "jca_workspace_bytes",
              "jagged_cand_attn_fwd", "cand_only_attn_fwd", "jca_status_string",
              "jagged_cand_attn_plan", "jagged_cand_attn_run", "cand_only_attn_plan",
              "cand_only_attn_run", "jca_stack_workspace_bytes", "jca_stack_fwd",
              "jagged_cand_attn_fwd_lse", "jca_bwd_workspace_bytes", "jagged_cand_attn_bwd",
              "jagged_causal_attn_fwd", "ug_masked_cross_attn_fwd"]:
        assert n in names


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", jca.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for name in jca.header_functions():
        assert name in exported, name
        assert getattr(L, name) is not None


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="missing"):
        jca.lib(str(tmp_path / "libjca.so"))


def test_status_strings(L):
    assert jca.status_string(0) == "ok"
    for code in (-1, -2, -3, -4, -5, -6, -7, -8, -9, 1, 2, 3, 4, 5, 6, 7, 16):
        assert jca.status_string(code) != "unknown code"
    assert jca.status_string(12345) == "unknown code"


def test_workspace_and_queue_bounds(L):
    assert L.jca_workspace_bytes(3, 20, 2, 16) > 0
    assert L.jca_workspace_bytes(3, 20, 2, 48) == 0       # unsupported head dim
    assert L.jca_workspace_bytes(-1, 20, 2, 16) == 0
    assert L.jca_max_work_items(3, 1222, 4) == (5 + 3) * 4
    ws = L.jca_workspace_bytes(256, 131072, 8, 128)
    assert ws % 256 == 0 and ws >= 16 * L.jca_max_work_items(256, 131072, 8)


def _addr(n):
    return ctypes.c_void_p(n)


def test_host_argument_errors(L):
    p = _addr(0x10000)  # never dereferenced: every call below fails its host checks
    st = _addr(0x20000)
    assert L.jca_offsets_from_lengths(p, p, 3, 16, st, None) == -5
    assert L.jca_offsets_from_lengths(p, p, -1, 32, st, None) == -2
    assert L.jca_offsets_from_lengths(None, p, 3, 32, st, None) == -1
    assert L.jca_build_segment_ids(p, p, None, 0, 0, 5, 32, p, st, None) == -2
    assert L.jca_bounds_from_segment_ids(p, p, 2, 10, 32, None, p, p, p, st, None) == -1
    assert L.jca_build_work_queue(p, p, p, None, 2, 10, 10, 0, 32, p, 8, p, st, None) == -2
    assert L.jca_build_work_queue(p, p, p, None, 2, 10, 10, 1, 32, _addr(0x10008), 8, p, st,
                                  None) == -4
    ws = _addr(0x40000)
    # idx_bits, head dim, H, null, alignment, workspace size
    args = [p, p, p, p, 0, p, p, None, 3, 20, 2, 16, 0.0, 32, ws, 1 << 20, st, None]

    def call(**kw):
        a = list(args)
        names = ["q", "k", "v", "out", "out_fp32", "off", "cs", "seg", "B", "T", "H", "d",
                 "scale", "idx_bits", "ws", "ws_bytes", "status", "stream"]
        for key, val in kw.items():
            a[names.index(key)] = val
        return L.jagged_cand_attn_fwd(*a)

    assert call(idx_bits=8) == -5
    assert call(d=48) == -3
    assert call(H=0) == -2
    assert call(B=0) == -2            # rows without users
    assert call(q=None) == -1
    assert call(cs=None) == -1        # neither candidate_start nor seg
    assert call(k=_addr(0x10002)) == -4
    assert call(ws=_addr(0x40010)) == -4
    assert call(ws_bytes=16) == -6
    cargs = [p, p, p, p, p, p, p, None, p, 0, 2, 8, 6, 2, 16, 0.0, 32, ws, 1 << 20, st, None]
    assert L.cand_only_attn_fwd(*cargs[:14], 24, *cargs[15:]) == -3
    cargs_bad = list(cargs)
    cargs_bad[4] = None
    assert L.cand_only_attn_fwd(*cargs_bad) == -1


def test_stack_host_argument_errors(L):
    p = _addr(0x10000)  # never dereferenced: every call below fails its host checks
    st = _addr(0x20000)
    ws = _addr(0x40000)
    assert L.jca_stack_workspace_bytes(3, 20, 9, 8, 2, 16) > 0
    assert L.jca_stack_workspace_bytes(3, 20, 15, 8, 2, 16) == 0     # Nc + Th > T
    assert L.jca_stack_workspace_bytes(3, 20, 9, 8, 2, 24) == 0      # head dim
    names = ["x", "x_out", "w", "n_layers", "n_cand_only", "off", "cs", "seg", "B", "T", "Nc", "Th",
             "H", "d", "scale", "history_end", "base", "idx_bits", "ws", "ws_bytes", "status",
             "stream"]
    args = [p, p, p, 3, 1, p, p, None, 3, 20, 9, 8, 2, 16, 0.0, -1, 10000.0, 32, ws, 1 << 30, st,
            None]

    def call(**kw):
        a = list(args)
        for key, val in kw.items():
            a[names.index(key)] = val
        return L.jca_stack_fwd(*a)

    assert call(idx_bits=16) == -5
    assert call(d=24) == -3
    assert call(n_cand_only=4) == -2         # more tail layers than layers
    assert call(n_layers=-1) == -2
    assert call(Nc=15) == -2                 # Nc + Th > T
    assert call(history_end=5, base=1.0) == -2
    assert call(x=None) == -1
    assert call(w=None) == -1
    assert call(cs=None) == -1               # neither candidate_start nor seg
    assert call(x_out=_addr(0x10004)) == -4
    assert call(ws=_addr(0x40010)) == -4
    assert call(ws_bytes=4096) == -6


def test_training_host_argument_errors(L):
    p = _addr(0x10000)  # never dereferenced: every call below fails its host checks
    st = _addr(0x20000)
    ws = _addr(0x40000)
    assert L.jca_bwd_workspace_bytes(3, 20, 2, 16) >= L.jca_workspace_bytes(3, 20, 2, 16)
    assert L.jca_bwd_workspace_bytes(3, 20, 2, 24) == 0
    fargs = [p, p, p, p, 0, p, p, p, None, 3, 20, 2, 16, 0.0, 32, ws, 1 << 20, st, None]
    assert L.jagged_cand_attn_fwd_lse(*fargs[:5], None, *fargs[6:]) == -1      # lse missing
    assert L.jagged_cand_attn_fwd_lse(*fargs[:5], _addr(0x10002), *fargs[6:]) == -4
    names = ["q", "k", "v", "out", "out_fp32", "dout", "lse", "dq", "dk", "dv", "grad_fp32",
             "off", "cs", "seg", "B", "T", "H", "d", "scale", "idx_bits", "ws", "ws_bytes",
             "status", "stream"]
    args = [p, p, p, p, 0, p, p, p, p, p, 1, p, p, None, 3, 20, 2, 16, 0.0, 32, ws, 1 << 20, st,
            None]

    def call(**kw):
        a = list(args)
        for key, val in kw.items():
            a[names.index(key)] = val
        return L.jagged_cand_attn_bwd(*a)

    assert call(idx_bits=8) == -5
    assert call(d=48) == -3
    assert call(H=0) == -2
    assert call(dout=None) == -1
    assert call(lse=None) == -1
    assert call(cs=None) == -1
    assert call(dk=_addr(0x10008)) == -4
    assert call(ws=_addr(0x40010)) == -4
    assert call(ws_bytes=64) == -6


def test_causal_host_argument_errors(L):
    p = _addr(0x10000)  # never dereferenced: every call below fails its host checks
    st = _addr(0x20000)
    ws = _addr(0x40000)
    args = [p, p, p, p, 0, p, 3, 20, 2, 16, 0.0, 32, ws, 1 << 20, st, None]
    assert L.jagged_causal_attn_fwd(*args[:11], 8, *args[12:]) == -5         # idx_bits
    assert L.jagged_causal_attn_fwd(*args[:9], 48, *args[10:]) == -3          # head dim
    assert L.jagged_causal_attn_fwd(None, *args[1:]) == -1
    assert L.jagged_causal_attn_fwd(*args[:5], None, *args[6:]) == -1         # offsets
    assert L.jagged_causal_attn_fwd(*args[:3], _addr(0x10002), *args[4:]) == -4
    assert L.jagged_causal_attn_fwd(*args[:13], 16, *args[14:]) == -6         # workspace


def test_ug_host_argument_errors(L):
    p = _addr(0x10000)  # never dereferenced: every call below returns before any device work
    st = _addr(0x20000)

    def call(q=p, k=p, v=p, res=None, out=p, B=4, T_out=16, T_in=32, c_u=8, n_u=16, H=1, d=128,
             status=st):
        return L.ug_masked_cross_attn_fwd(q, k, v, res, out, 0, B, T_out, T_in, c_u, n_u, H, d,
                                          0.0, status, None)

    assert call(d=48) == -3
    assert call(T_in=129) == -2
    assert call(T_out=129) == -2
    assert call(c_u=17) == -2
    assert call(n_u=33) == -2
    assert call(c_u=-1) == -2
    assert call(H=0) == -2
    assert call(B=-1) == -2
    assert call(B=1 << 40) == -2          # row coordinates beyond 32 bits
    assert call(q=None) == -1
    assert call(status=None) == -1
    assert call(k=None) == -1
    assert call(out=None) == -1
    assert call(q=None, k=None, v=None, T_in=0, n_u=0) == -1   # k, v may be null, q may not
    assert call(v=_addr(0x10004)) == -4
    assert call(res=_addr(0x10008)) == -4
    assert call(B=0) == 0                 # nothing to do, nothing launched
    assert call(T_out=0, c_u=0) == 0
