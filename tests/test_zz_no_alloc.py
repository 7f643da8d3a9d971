"""The workspace-free entry point, jagged_cand_attn_fwd_noalloc.

It serves callers that cannot allocate device memory when they call (fixed-memory serving loops,
plugins handed only their tensors, code that must avoid cudaMalloc's implicit synchronisation):
the library keeps the scratch in its own static device array. These tests call it through the C
ABI, twice in a row on the same array, and compare each result with jagged_cand_attn_fwd given a
caller workspace, under the tolerance of the other parity tests, and with the CPU oracle directly.
This file is collected last so that a run stopping at its first failure has already run every
other test.
"""

import numpy as np
import pytest
import torch

import synth
from candidate_isolated_jagged_b200 import jca
from helpers import FullRun, assert_close, dev

pytestmark = pytest.mark.gpu


def _with_workspace(r, out_fp32):
    out = torch.empty(r.q.shape, dtype=torch.float32 if out_fp32 else torch.bfloat16, device=dev())
    st = jca.new_status(dev())
    jca.jagged_cand_attn_fwd(r.q, r.k, r.v, out, r.off, r.cs, r.seg, status=st)
    jca.check_status(st)
    return out


def _no_alloc(r, out_fp32):
    out = torch.full(r.q.shape, float("nan"),
                     dtype=torch.float32 if out_fp32 else torch.bfloat16, device=dev())
    st = jca.new_status(dev())
    jca.jagged_cand_attn_fwd_noalloc(r.q, r.k, r.v, out, r.off, r.cs, r.seg, status=st)
    jca.check_status(st)
    return out


@pytest.mark.parametrize("name", ["three_users", "mixed"])
@pytest.mark.parametrize("out_fp32", [True, False])
def test_no_alloc_matches_workspace_call_twice(name, out_fp32):
    if name == "three_users":
        b = synth.three_users()
    else:
        b = synth.custom_batch([0, 1, 127, 300, 1000, 37], prefix=[0, 2, 1, 4, 4, 3],
                               n_cand=[3, 0, 64, 64, 129, 5], H=8, d=128, seed=21)
    r = FullRun(b)
    ref = _with_workspace(r, out_fp32).to(torch.float64).cpu().numpy()
    first = _no_alloc(r, out_fp32)
    second = _no_alloc(r, out_fp32)       # same static array, left over from the first call
    for got in (first, second):
        assert_close(got, ref, f"no-alloc {name}")
    assert torch.equal(first, second)
    if out_fp32:
        assert_close(first, r.reference(), f"no-alloc {name} vs oracle")


def test_no_alloc_prepare_then_call():
    # jca_noalloc_prepare caches the array's address for the current device (what a caller does
    # before capturing a stream); calls after it give the same result as before, bit for bit.
    r = FullRun(synth.three_users())
    before = _no_alloc(r, True)
    assert jca.jca_noalloc_prepare() == 0
    after = _no_alloc(r, True)
    assert torch.equal(before, after)


def test_no_alloc_after_a_different_problem():
    # the array keeps the previous call's contents; a smaller problem afterwards is unaffected
    big = FullRun(synth.custom_batch([900, 50], prefix=2, n_cand=[40, 8], H=4, d=64, seed=3))
    _no_alloc(big, True)
    small = FullRun(synth.tiny())
    assert_close(_no_alloc(small, True), _with_workspace(small, True).double().cpu().numpy(),
                 "no-alloc tiny after a larger problem")


def test_no_alloc_rejects_problems_beyond_the_array():
    limit = jca.jca_noalloc_scratch_bytes()
    assert limit == 8 << 20
    rows = 1 << 30                        # segment IDs alone would need 1 GiB of scratch
    assert jca.jca_workspace_bytes(1, rows, 1, 16) > limit
    L = jca.lib()
    import ctypes
    st = jca.new_status(dev())
    # No tensor is passed: the size check comes first, so the call must return before it would
    # look at any pointer (and, were that check ever lost, stop at the null-pointer check).
    code = L.jagged_cand_attn_fwd_noalloc(None, None, None, None, 1, None, None, None, 1, rows, 1,
                                          16, 0.0, 64, ctypes.c_void_p(st.data_ptr()), None)
    assert code == -9
    assert "static array" in jca.status_string(code)
    assert int(st.item()) == 0
