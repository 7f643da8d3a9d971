"""GPU parity of the per-user causal variant (jagged_causal_attn_fwd) against the oracle
(oracle/variants.py): row i of user b sees rows j <= i of user b. Tile edges around 128 and 256
rows, head sizes 16-128, int32 and int64 offsets, bf16 and fp32 outputs, the 256-user row lengths
at H = 8, d = 128 on sampled rows, and a bad-offsets status."""

import numpy as np
import pytest
import torch

import oracle
import oracle.variants as ov
import synth
from candidate_isolated_jagged_b200 import jca
from helpers import assert_close, assert_close_bf16, dev, sample_rows

pytestmark = pytest.mark.gpu

EDGE_LENGTHS = [1, 5, 0, 17, 64, 127, 128, 129, 255, 256, 257, 300, 513, 1000]


def _run(b, idx=torch.int64, out_fp32=True):
    off = torch.tensor(oracle.offsets_from_lengths(b.row_lengths), dtype=idx, device=dev())
    out = torch.full(b.q.shape, float("nan"),
                     dtype=torch.float32 if out_fp32 else torch.bfloat16, device=dev())
    st = jca.new_status(dev())
    jca.jagged_causal_attn_fwd(b.q.to(dev()), b.k.to(dev()), b.v.to(dev()), out, off, status=st)
    torch.cuda.synchronize()
    jca.check_status(st, "jagged_causal_attn_fwd")
    return out


@pytest.mark.parametrize("idx", [torch.int32, torch.int64])
@pytest.mark.parametrize("d", [16, 32, 64, 128])
def test_causal_tile_edges(d, idx):
    b = synth.custom_batch(EDGE_LENGTHS, prefix=0, n_cand=0, H=2, d=d, seed=d)
    got = _run(b, idx)
    ref = ov.jagged_causal_attn(b.q, b.k, b.v, oracle.offsets_from_lengths(b.row_lengths), b.scale)
    assert_close(got, ref, f"causal d={d}")


def test_causal_bf16_output():
    b = synth.custom_batch([3, 200, 700], prefix=0, n_cand=0, H=4, d=64, seed=7)
    got = _run(b, out_fp32=False)
    ref = ov.jagged_causal_attn(b.q, b.k, b.v, oracle.offsets_from_lengths(b.row_lengths), b.scale)
    assert_close_bf16(got, ref, "causal bf16")


def test_causal_users256_sampled_rows():
    """The 256-user row lengths (4 prefix + history + 64 candidates per user) as causal sequences,
    H = 8, d = 128, in the configuration the benchmark times; sampled rows are computed one by one
    by the oracle's masked softmax over the row's prefix of its user."""
    n = synth.users256_history_lengths(0)
    b = synth.custom_batch(n + 68, prefix=0, n_cand=0, H=8, d=128, seed=0)
    got = _run(b, out_fp32=True)
    off = oracle.offsets_from_lengths(b.row_lengths)
    rows = sample_rows(off, per_user=2, seed=3)
    users = np.searchsorted(off, rows, side="right") - 1
    ref = np.zeros((rows.size, b.H, b.d))
    for i, (row, u) in enumerate(zip(rows, users)):
        s = int(off[u])
        ref[i] = oracle.masked_softmax_attention(b.q[row:row + 1], b.k[s:row + 1], b.v[s:row + 1],
                                                 np.ones((1, row + 1 - s), bool), b.scale)[0]
    assert_close(got[torch.from_numpy(rows).to(dev())], ref, "causal users256 sampled")
    assert bool(torch.isfinite(got).all())


def test_causal_bad_offsets_status():
    b = synth.custom_batch([4, 9], prefix=0, n_cand=0, H=1, d=16, seed=1)
    off = torch.tensor([0, 10, 9], dtype=torch.int64, device=dev())   # decreasing, short of T
    out = torch.full(b.q.shape, 7.0, dtype=torch.float32, device=dev())
    st = jca.new_status(dev())
    jca.jagged_causal_attn_fwd(b.q.to(dev()), b.k.to(dev()), b.v.to(dev()), out, off, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 2          # JCA_STATUS_BAD_OFFSETS
    assert bool((out == 7.0).all())     # nothing written
