"""GPU parity of the layer stack (jca_stack_fwd) against the oracle's stack (oracle/stack.py):
full layers over whole rows, the split into frozen history and candidates, and candidate-only tail
layers (候选隔离注意力掩码, section 只更新候选的末尾层), with and without right-anchored RoPE.

Tolerance. Both sides round to bf16 at the same points (each projection, RoPE output, attention
output and residual sum); the GPU accumulates in fp32 (cuBLASLt, the attention kernels), the oracle
in fp64. Two checks:

* Layer by layer, element by element. The oracle's layer l is applied to the GPU's own states after
  layer l - 1 (the GPU stack cut after l - 1 layers), and the GPU's states after layer l must agree
  within 1e-2 + ulp_bf16(|ref|) per element: the benchmark spec's 1e-2 for the fp32-accumulated
  arithmetic, plus one bf16 ulp of the element for the rounding of the stored state (both sides
  round values less than 1e-2 apart, each by up to half an ulp, so they can land on neighbouring
  bf16 numbers). A torch fp32 emulation of the GPU's rounding points needs at most
  1e-2 + 0.36 ulp on the three-user and the 256-user stacks.
* End to end: relative L2 <= 5e-3 over the whole output (the spec bar). A one-ulp rounding
  difference in one layer moves every later layer's scores, so two stacks that round at the same
  points agree in relative L2 (1e-3 to 2e-3 in the emulation) but not element by element after
  eight layers; the per-layer check is what holds each layer's kernels to the element-wise bar.
"""

import numpy as np
import pytest
import torch

import oracle
import oracle.stack as ostack
import synth
from candidate_isolated_jagged_b200 import jca
from helpers import dev

pytestmark = pytest.mark.gpu

REL_L2 = 5e-3


def _ulp(a):
    """bf16 ulp of each |a| (2^-7 of its binade)."""
    return np.exp2(np.floor(np.log2(np.maximum(np.abs(np.asarray(a, dtype=np.float64)),
                                                2.0 ** -30))) - 7)


def assert_stack_close(got, ref, what=""):
    """End to end: relative L2 over the whole output."""
    got = got.detach().to("cpu", torch.float64).numpy() if isinstance(got, torch.Tensor) else got
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    r = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    assert r <= REL_L2, f"{what}: rel_l2={r:.3e}"
    return r


def assert_layer_close(got, ref, what=""):
    """One layer on the GPU's own input states: 1e-2 + one bf16 ulp of each element."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape
    excess = np.abs(got - ref) - (1e-2 + _ulp(ref))
    r = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert float(excess.max()) <= 0 and r <= REL_L2, \
        f"{what}: max excess over 1e-2 + ulp {excess.max():.3e}, rel_l2={r:.3e}"


def _layout(sb):
    b = sb.batch
    off = oracle.offsets_from_lengths(b.row_lengths)
    seg = oracle.segment_ids(off, b.cand_start, b.valid)
    return off, seg


def _weights(sb):
    return torch.stack([torch.stack(list(w)) for w in sb.weights]).to(dev()) if sb.weights else \
        torch.empty(0, 4, sb.D, sb.D, dtype=torch.bfloat16, device=dev())


def run_gpu(sb, off, seg, history_end=None, idx=torch.int64, pass_seg=True, in_place=False,
            Nc=None, Th=None, check=True):
    b = sb.batch
    x = sb.x.to(dev())
    out = x if in_place else torch.full_like(x, float("nan"))
    offs = torch.tensor(off, dtype=idx, device=dev())
    cs = torch.tensor(b.cand_start, dtype=idx, device=dev())
    seg_t = torch.tensor(seg, device=dev()) if pass_seg else None
    Nc = int(np.sum(seg == -1)) if Nc is None else Nc
    Th = int(np.sum(seg == 1)) if Th is None else Th
    st = jca.new_status(dev())
    jca.jca_stack_fwd(x, out, _weights(sb), sb.n_cand_only, offs, None if pass_seg else cs, seg_t,
                      Nc=Nc, Th=Th, H=sb.H, scale=sb.scale, history_end=history_end, status=st)
    torch.cuda.synchronize()
    if check:
        jca.check_status(st, "jca_stack_fwd")
    return out, int(st.item())


def ref_stack(sb, off, seg, history_end=None):
    return ostack.stack_forward(sb.x, sb.weights, off, seg, sb.H, sb.n_cand_only, sb.scale,
                                history_end=history_end)


def check_layerwise(sb, off, seg, history_end=None, users=None, idx=torch.int64, what=""):
    """Teacher-forced check of every layer. The GPU stack cut after l layers (the same first l
    layers, the same split point) gives the GPU's states S_l; the oracle's layer l + 1 applied to
    S_l must match S_{l+1} element by element. Only the rows of `users` (default: all) are
    compared; users never interact, so the oracle runs on a batch of just those users."""
    import oracle.rope as orope
    b = sb.batch
    L, split = len(sb.weights), len(sb.weights) - sb.n_cand_only
    users = list(range(b.B)) if users is None else list(users)
    rows = np.concatenate([np.arange(off[u], off[u + 1]) for u in users]).astype(np.int64)
    soff = oracle.offsets_from_lengths(np.asarray(b.row_lengths)[users])
    sseg = np.asarray(seg)[rows]
    rows_t = torch.from_numpy(rows).to(dev())
    states = []
    for l in range(L + 1):
        cut = synth.StackBatch(b, sb.x, sb.weights[:l], max(0, l - split), sb.H, sb.d)
        got, _ = run_gpu(cut, off, seg, history_end, idx=idx)
        states.append(got[rows_t].to("cpu", torch.float64).numpy())
    w64 = [tuple(m.double().numpy() for m in w) for w in sb.weights]
    pos = None if history_end is None else orope.right_anchored_positions(soff, sseg, history_end)
    hist, cand, hoff, coff = ostack.split_history_and_candidates(soff, sseg)
    keep = sseg != -1
    for l in range(L):
        x_in, x_out = states[l], states[l + 1]
        if l < split:
            ref = ostack.full_layer(x_in, w64[l], soff, sseg, sb.H, sb.scale, pos)
            assert_layer_close(x_out, ref, f"{what} layer {l} (full)")
        else:
            ref = ostack.candidate_only_layer(x_in[cand], x_in[hist], w64[l], coff, hoff, sb.H,
                                              sb.scale, None if pos is None else pos[cand],
                                              None if pos is None else pos[hist])
            assert_layer_close(x_out[cand], ref, f"{what} layer {l} (candidate-only)")
            assert np.array_equal(x_out[keep], x_in[keep]), f"{what} layer {l}: frozen rows moved"
    return states[L]


def _small(seed=0, **kw):
    args = dict(hist_lengths=[0, 1, 7, 13], prefix=[1, 0, 2, 3], n_cand=[2, 3, 0, 5], H=2, d=16,
                n_layers=3, n_cand_only=2, seed=seed, pad_hist_to=4)
    args.update(kw)
    return synth.custom_stack(**args)


@pytest.mark.parametrize("idx", [torch.int32, torch.int64])
@pytest.mark.parametrize("history_end", [None, 50])
@pytest.mark.parametrize("pass_seg", [True, False])
def test_small_stack(idx, history_end, pass_seg):
    sb = _small(0) if pass_seg else _small(0, pad_hist_to=None)
    off, seg = _layout(sb)
    got, _ = run_gpu(sb, off, seg, history_end, idx=idx, pass_seg=pass_seg)
    assert_stack_close(got, ref_stack(sb, off, seg, history_end), "small")
    if pass_seg:
        last = check_layerwise(sb, off, seg, history_end, idx=idx, what="small")
        assert np.array_equal(last, got.to("cpu", torch.float64).numpy())


@pytest.mark.parametrize("n_layers,n_cand_only", [(2, 0), (2, 2), (3, 1), (1, 1), (0, 0)])
def test_split_points(n_layers, n_cand_only):
    sb = _small(4, n_layers=n_layers, n_cand_only=n_cand_only, H=4, d=32)
    off, seg = _layout(sb)
    got, _ = run_gpu(sb, off, seg, 17)
    assert_stack_close(got, ref_stack(sb, off, seg, 17), f"{n_layers}/{n_cand_only}")
    check_layerwise(sb, off, seg, 17, what=f"{n_layers}/{n_cand_only}")


def test_in_place():
    sb = _small(5, H=2, d=64)
    off, seg = _layout(sb)
    got, _ = run_gpu(sb, off, seg, 9, in_place=True)
    assert_stack_close(got, ref_stack(sb, off, seg, 9), "in place")


@pytest.mark.parametrize("history_end", [None, 2000])
def test_three_users_stack(history_end):
    # Histories [10, 100, 1000] padded to a multiple of 8, 2 prefix, 32 candidates; H=4, d=64.
    sb = synth.custom_stack([10, 100, 1000], 2, 32, H=4, d=64, n_layers=4, n_cand_only=2, seed=0,
                            pad_hist_to=8)
    off, seg = _layout(sb)
    got, _ = run_gpu(sb, off, seg, history_end)
    assert_stack_close(got, ref_stack(sb, off, seg, history_end), "three users")
    check_layerwise(sb, off, seg, history_end, what="three users")


def test_padding_and_history_rows_frozen_at_split():
    # Rows that are not candidates keep the state they had after the last full layer: the same
    # stack with all tail layers removed gives them exactly.
    sb = synth.custom_stack([5, 40, 0, 130], [2, 1, 3, 0], [7, 1, 9, 33], H=2, d=32, n_layers=3,
                            n_cand_only=2, seed=3, pad_hist_to=16)
    off, seg = _layout(sb)
    got, _ = run_gpu(sb, off, seg, 300)
    head = synth.StackBatch(sb.batch, sb.x, sb.weights[:1], 0, sb.H, sb.d)
    got_head, _ = run_gpu(head, off, seg, 300)
    keep = torch.tensor(seg != -1, device=dev())
    assert torch.equal(got[keep], got_head[keep])
    assert not torch.equal(got[~keep], got_head[~keep])


def test_bad_split_totals():
    sb = _small(1)
    off, seg = _layout(sb)
    Nc = int(np.sum(seg == -1))
    _, code = run_gpu(sb, off, seg, None, Nc=Nc - 1, check=False)
    assert code == 7   # JCA_STATUS_BAD_SPLIT
    _, code = run_gpu(sb, off, seg, None, Th=int(np.sum(seg == 1)) + 1, check=False)
    assert code == 7


def test_users256_stack_sampled_users():
    """The full 256-user stack (8 layers, the last 2 candidate-only, H=8, d=128, D=1024) in the
    launch configuration the benchmark times, checked on sampled users: rows of different users
    never interact, so the oracle's stack over a batch of just those users gives their outputs."""
    sb = synth.stack_users256()
    off, seg = _layout(sb)
    got, _ = run_gpu(sb, off, seg, 8192)
    b = sb.batch
    n = b.hist_real
    users = [0, int(np.argsort(n)[128]), int(np.argsort(n)[200])]   # empty, median, longer
    rows = np.concatenate([np.arange(off[u], off[u + 1]) for u in users])
    sub = synth.StackBatch(
        synth.Batch("sub", b.row_lengths[users], b.cand_start[users], None, b.q[:0], b.k[:0],
                    b.v[:0], 1, 16, 0),
        sb.x[torch.from_numpy(rows)], sb.weights, sb.n_cand_only, sb.H, sb.d)
    soff = oracle.offsets_from_lengths(b.row_lengths[users])
    sseg = seg[rows]
    ref = ostack.stack_forward(sub.x, sub.weights, soff, sseg, sb.H, sb.n_cand_only, sb.scale,
                               history_end=8192)
    assert_stack_close(got[torch.from_numpy(rows).to(dev())], ref, "users256 sampled")
    assert bool(torch.isfinite(got.float()).all())
    last = check_layerwise(sb, off, seg, 8192, users=users, what="users256 sampled")
    assert np.array_equal(last, got[torch.from_numpy(rows).to(dev())].to("cpu", torch.float64).numpy())
