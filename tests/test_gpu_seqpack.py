"""GPU parity of training with candidate packing (jagged_cand_attn_seqpack_fwd / _bwd) against
the oracle (oracle/seqpack.py): users' history runs first, then every user's candidates stored
apart in one block (候选隔离注意力掩码, section 训练时的序列打包). Each serving-layout batch is
rearranged into that layout row for row; the forward, its log-sum-exp and the gradients are
compared with the oracle on the packed rows, under the tolerances of the serving-layout tests
(forward: max-abs 1e-2 and rel-L2 5e-3; gradients: rel-L2 5e-3 and max-abs 1e-2 * max(1, max|ref|),
see test_gpu_backward.py for the reasoning; log-sum-exp: 1e-3).
"""

import numpy as np
import pytest
import torch

import oracle
import oracle.seqpack as osp
import synth
from candidate_isolated_jagged_b200 import jca
from helpers import FullRun, assert_close, dev, seqpack_layout

pytestmark = pytest.mark.gpu

GRAD_MAX_ABS = 1e-2
GRAD_REL_L2 = 5e-3


class Packed:
    """A serving-layout batch rearranged into the candidate-packed layout, on the GPU."""

    def __init__(self, b, idx=torch.int64, pass_seg=None):
        self.b = b
        off = oracle.offsets_from_lengths(b.row_lengths)
        seg = oracle.segment_ids(off, b.cand_start, b.valid)
        self.perm, self.hoff_np, self.coff_np = seqpack_layout(b)
        self.seg_np = seg[self.perm]
        self.Th = int(self.hoff_np[-1])
        p = torch.from_numpy(self.perm)
        self.q, self.k, self.v = (t[p].to(dev()) for t in (b.q, b.k, b.v))
        self.hoff = torch.tensor(self.hoff_np, dtype=idx, device=dev())
        self.coff = torch.tensor(self.coff_np, dtype=idx, device=dev())
        if pass_seg is None:
            pass_seg = b.valid is not None
        self.seg = torch.tensor(self.seg_np, device=dev()) if pass_seg else None

    def fwd(self, out_fp32=True, with_lse=True, status=None):
        T, H, d = self.q.shape
        out = torch.full((T, H, d), float("nan"),
                         dtype=torch.float32 if out_fp32 else torch.bfloat16, device=dev())
        lse = torch.full((T, H), float("nan"), device=dev()) if with_lse else None
        st = jca.new_status(dev()) if status is None else status
        jca.jagged_cand_attn_seqpack_fwd(self.q, self.k, self.v, out, self.hoff, self.coff,
                                         self.seg, lse, status=st, Th=self.Th)
        torch.cuda.synchronize()
        return out, lse, st

    def bwd(self, out, lse, dout, grad_fp32=True):
        T, H, d = self.q.shape
        gdt = torch.float32 if grad_fp32 else torch.bfloat16
        dq, dk, dv = (torch.full((T, H, d), float("nan"), dtype=gdt, device=dev())
                      for _ in range(3))
        st = jca.new_status(dev())
        jca.jagged_cand_attn_seqpack_bwd(self.q, self.k, self.v, out, dout.to(dev()), lse, dq,
                                         dk, dv, self.hoff, self.coff, self.seg, status=st,
                                         Th=self.Th)
        torch.cuda.synchronize()
        jca.check_status(st, "seqpack bwd")
        return dq, dk, dv


def _batches():
    return {
        "tiny": synth.tiny(),
        "holes_d32": synth.custom_batch([0, 7, 300, 129, 1], prefix=[2, 0, 4, 1, 0],
                                        n_cand=[5, 1, 140, 0, 3], H=3, d=32, seed=4, pad_hist_to=16),
        "three_users": synth.three_users(),
        "d128_edges": synth.custom_batch([127, 128, 129, 255, 0], prefix=1, n_cand=[1, 130, 2, 0, 9],
                                         H=2, d=128, seed=6),
    }


NAMES = ["tiny", "holes_d32", "three_users", "d128_edges"]


@pytest.mark.parametrize("idx", [torch.int32, torch.int64])
@pytest.mark.parametrize("name", NAMES)
def test_forward_and_lse(name, idx):
    P = Packed(_batches()[name], idx=idx)
    out, lse, st = P.fwd()
    jca.check_status(st, "seqpack fwd")
    b = P.b
    ref = osp.seqpack_attn(P.q.cpu(), P.k.cpu(), P.v.cpu(), P.hoff_np, P.coff_np, P.seg_np,
                           b.scale)
    assert_close(out, ref, f"{name} seqpack out")
    ref_lse = osp.seqpack_log_sum_exp(P.q.cpu(), P.k.cpu(), P.hoff_np, P.coff_np, P.seg_np,
                                      b.scale)
    got = lse.double().cpu().numpy()
    fin = np.isfinite(ref_lse)
    assert np.array_equal(fin, np.isfinite(got))
    assert np.all(got[~fin] == -np.inf)
    assert np.max(np.abs(got[fin] - ref_lse[fin]), initial=0.0) <= 1e-3
    # without lse: the same output bit for bit
    out2, _, st2 = P.fwd(with_lse=False)
    jca.check_status(st2)
    assert torch.equal(out, out2)


@pytest.mark.parametrize("name", NAMES)
def test_same_rows_as_the_serving_layout(name):
    # Packing moves rows, not what they compute: every packed row equals its serving-layout row
    # (the serving-layout forward on the same batch), within the forward tolerance.
    P = Packed(_batches()[name])
    out, _, st = P.fwd()
    jca.check_status(st)
    serving = FullRun(P.b).run(out_fp32=True)
    assert_close(out, serving[torch.from_numpy(P.perm).to(dev())].double().cpu().numpy(),
                 f"{name} packed vs serving rows")


@pytest.mark.parametrize("idx", [torch.int32, torch.int64])
@pytest.mark.parametrize("name", NAMES)
def test_backward(name, idx):
    P = Packed(_batches()[name], idx=idx)
    out, lse, st = P.fwd()
    jca.check_status(st)
    dout = synth.upstream_grad(P.q.shape, 21)
    dq, dk, dv = P.bwd(out, lse, dout)
    ref = osp.seqpack_attn_bwd(P.q.cpu(), P.k.cpu(), P.v.cpu(), dout.double().numpy(), P.hoff_np,
                               P.coff_np, P.seg_np, P.b.scale)
    for nm, g, f in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        bound = GRAD_MAX_ABS * max(1.0, float(np.max(np.abs(f))) if f.size else 1.0)
        assert_close(g, f, f"{name} seqpack {nm}", max_abs=bound, rel_l2=GRAD_REL_L2)
    pad = torch.from_numpy(P.seg_np == 0).to(dev())
    for g in (dq, dk, dv):
        assert bool((g[pad] == 0).all())


def test_backward_bf16_outputs_and_candidate_isolation():
    # dO on one candidate only: every other candidate and every row of other users get exactly 0;
    # the bf16 outputs hold the fp32 bar plus half a bf16 ulp.
    P = Packed(_batches()["holes_d32"])
    out, lse, st = P.fwd(out_fp32=False)
    jca.check_status(st)
    cands = np.nonzero(P.seg_np == -1)[0]
    i = int(cands[len(cands) // 3])
    dout = torch.zeros(P.q.shape, dtype=torch.bfloat16)
    dout[i] = synth.upstream_grad(P.q.shape, 22)[i]
    dq, dk, dv = P.bwd(out, lse, dout, grad_fp32=False)
    user = int(np.searchsorted(P.coff_np, i - P.Th, side="right") - 1)
    hist_rows = np.arange(P.hoff_np[user], P.hoff_np[user + 1])
    others = np.setdiff1d(np.arange(P.q.shape[0]), np.concatenate([hist_rows, [i]]))
    o = torch.from_numpy(others).to(dev())
    for g in (dq, dk, dv):
        assert bool((g[o] == 0).all())
    ref = osp.seqpack_attn_bwd(P.q.cpu(), P.k.cpu(), P.v.cpu(), dout.double().numpy(), P.hoff_np,
                               P.coff_np, P.seg_np, P.b.scale)
    for nm, g, f in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(f), 1e-30))) - 7)
        scale = max(1.0, float(np.max(np.abs(f))))
        excess = np.abs(g.double().cpu().numpy() - f) - (GRAD_MAX_ABS * scale + 0.5 * ulp)
        assert np.all(excess <= 0), f"{nm}: max excess {excess.max():.3e}"


def test_bad_offsets_and_segment_values():
    P = Packed(_batches()["tiny"])
    bad = P.coff.clone()
    bad[1] = bad[2] + 1                        # decreasing candidate offsets
    P2 = Packed(_batches()["tiny"])
    P2.coff = bad
    out, _, st = P2.fwd()
    assert int(st.item()) == 2                  # JCA_STATUS_BAD_OFFSETS
    assert bool(torch.isnan(out).all())         # nothing written
    P3 = Packed(_batches()["tiny"], pass_seg=True)
    P3.seg = P3.seg.clone()
    P3.seg[-1] = 1                              # a history ID in the candidate block
    out, _, st = P3.fwd()
    assert int(st.item()) == 5                  # JCA_STATUS_BAD_SEG_VALUE
    assert bool(torch.isnan(out).all())


def test_users256_packed_sampled_users():
    """The 256-user workload rearranged into the candidate-packed layout, forward with LSE and
    backward in full; the oracle checks three users (an empty history, the median, the
    4096-token history), whose rows no other user touches."""
    b = synth.users256()
    P = Packed(b)
    out, lse, st = P.fwd(out_fp32=False)
    jca.check_status(st)
    dout = synth.upstream_grad(P.q.shape, 23)
    dq, dk, dv = P.bwd(out, lse, dout)
    users = [0, int(np.argsort(b.hist_real)[128]), 1]
    rows = np.concatenate([osp.user_rows(P.hoff_np, P.coff_np, u) for u in users])
    sub_h = oracle.offsets_from_lengths([P.hoff_np[u + 1] - P.hoff_np[u] for u in users])
    sub_c = oracle.offsets_from_lengths([P.coff_np[u + 1] - P.coff_np[u] for u in users])
    hrows = np.concatenate([np.arange(P.hoff_np[u], P.hoff_np[u + 1]) for u in users])
    crows = np.concatenate([P.Th + np.arange(P.coff_np[u], P.coff_np[u + 1]) for u in users])
    sub = np.concatenate([hrows, crows])
    q, k, v = (t[torch.from_numpy(sub).to(dev())].cpu() for t in (P.q, P.k, P.v))
    sseg = P.seg_np[sub]
    ref = osp.seqpack_attn(q, k, v, sub_h, sub_c, sseg, b.scale)
    from helpers import assert_close_bf16
    assert_close_bf16(out[torch.from_numpy(sub).to(dev())], ref, "users256 packed out")
    g_ref = osp.seqpack_attn_bwd(q, k, v, dout[torch.from_numpy(sub)].double().numpy(), sub_h,
                                 sub_c, sseg, b.scale)
    for nm, g, f in zip(("dq", "dk", "dv"), (dq, dk, dv), g_ref):
        gs = g[torch.from_numpy(sub).to(dev())]
        bound = GRAD_MAX_ABS * max(1.0, float(np.max(np.abs(f))))
        assert_close(gs, f, f"users256 packed {nm}", max_abs=bound, rel_l2=GRAD_REL_L2)
    assert set(rows.tolist()) == set(sub.tolist())
    for g in (dq, dk, dv):
        assert bool(torch.isfinite(g).all())
