"""Pins of the layer-stack oracle (oracle/stack.py): the split by hand, the candidate-only tail
against the pages' fallback, the freezing premise (history independent of candidates), candidate
isolation through the whole stack, and special cases that reduce to a library routine or a closed
form, so that a wrong index, a dropped term or a leaked padding row in it fails here."""

import numpy as np
import pytest
import torch

import oracle
import oracle.stack as ostack
import synth


def _layout(sb):
    b = sb.batch
    off = oracle.offsets_from_lengths(b.row_lengths)
    seg = oracle.segment_ids(off, b.cand_start, b.valid)
    return off, seg


def _small(seed=0, n_layers=3, n_cand_only=2, **kw):
    args = dict(hist_lengths=[0, 1, 7, 13], prefix=[1, 0, 2, 3], n_cand=[2, 3, 0, 5], H=2, d=8,
                n_layers=n_layers, n_cand_only=n_cand_only, seed=seed, pad_hist_to=4)
    args.update(kw)
    return synth.custom_stack(**args)


def _run(sb, off, seg, **kw):
    return ostack.stack_forward(sb.x, sb.weights, off, seg, sb.H, sb.n_cand_only, sb.scale, **kw)


def test_split_hand_case():
    # rows: user 0 = [1 1 0 -1 -1], user 1 = [], user 2 = [0 1 -1], user 3 = [-1]
    off = oracle.offsets_from_lengths([5, 0, 3, 1])
    seg = np.array([1, 1, 0, -1, -1, 0, 1, -1, -1], dtype=np.int8)
    hist, cand, hoff, coff = ostack.split_history_and_candidates(off, seg)
    assert hist.tolist() == [0, 1, 6]
    assert cand.tolist() == [3, 4, 7, 8]
    assert hoff.tolist() == [0, 2, 2, 3, 3]
    assert coff.tolist() == [0, 2, 2, 3, 4]


@pytest.mark.parametrize("history_end", [None, 50])
@pytest.mark.parametrize("seed", [0, 1])
def test_candidate_only_tail_equals_fallback(seed, history_end):
    sb = _small(seed)
    off, seg = _layout(sb)
    a = _run(sb, off, seg, history_end=history_end, bf16=False)
    f = _run(sb, off, seg, history_end=history_end, bf16=False, fallback=True)
    assert np.max(np.abs(a - f)) < 1e-10


def test_candidate_only_tail_equals_fallback_bf16():
    # With bf16 rounding, the two orders of summation may round a value to neighbouring bf16 numbers
    # at a few places; the states agree to within a few bf16 ulps everywhere.
    sb = _small(2, n_layers=4, n_cand_only=2)
    off, seg = _layout(sb)
    a = _run(sb, off, seg, history_end=30)
    f = _run(sb, off, seg, history_end=30, fallback=True)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(f), 2.0 ** -30))) - 7)
    assert np.all(np.abs(a - f) <= 4 * ulp)
    assert np.mean(a == f) > 0.99


def test_freezing_changes_candidates():
    # The tail is not a plain stack: letting the history update in the last layers (all layers
    # full) changes the candidates' outputs, so the equivalence above is not vacuous.
    sb = _small(3)
    off, seg = _layout(sb)
    frozen = _run(sb, off, seg, bf16=False)
    sb_full = synth.StackBatch(sb.batch, sb.x, sb.weights, 0, sb.H, sb.d)
    unfrozen = _run(sb_full, off, seg, bf16=False)
    cand = seg == -1
    assert np.max(np.abs(frozen[cand] - unfrozen[cand])) > 1e-3
    assert np.max(np.abs(frozen[~cand] - unfrozen[~cand])) > 1e-3    # history moved on


def test_history_independent_of_candidates():
    # The premise of freezing: with every layer full, the history states never depend on the
    # candidates. Change every candidate's input state and the number of candidates of user 3.
    sb = _small(4, n_cand_only=0)
    off, seg = _layout(sb)
    base = _run(sb, off, seg, bf16=False)
    x2 = sb.x.clone()
    x2[torch.tensor(seg == -1)] = torch.randn(int((seg == -1).sum()), sb.D).to(torch.bfloat16)
    other = _run(synth.StackBatch(sb.batch, x2, sb.weights, 0, sb.H, sb.d), off, seg, bf16=False)
    h = seg == 1
    assert np.max(np.abs(base[h] - other[h])) < 1e-12
    # fewer candidates for the last user: drop its last two rows
    T = sb.x.shape[0]
    keep = np.ones(T, dtype=bool)
    keep[T - 2:] = False
    b = sb.batch
    rl = b.row_lengths.copy()
    rl[-1] -= 2
    off3 = oracle.offsets_from_lengths(rl)
    seg3 = oracle.segment_ids(off3, b.cand_start, None if b.valid is None else b.valid[keep])
    out3 = ostack.stack_forward(sb.x[torch.tensor(keep)], sb.weights, off3, seg3, sb.H, 0, sb.scale,
                                bf16=False)
    assert np.max(np.abs(out3[seg3 == 1] - base[h])) < 1e-12


@pytest.mark.parametrize("history_end", [None, 17])
def test_candidate_isolation_through_the_stack(history_end):
    # Removing a candidate, or reversing the order of a user's candidates, leaves every other
    # candidate's final state unchanged (the pages' order invariance, with RoPE on).
    sb = _small(5, n_layers=3, n_cand_only=1)
    off, seg = _layout(sb)
    base = _run(sb, off, seg, history_end=history_end, bf16=False)
    b = sb.batch
    s, e = int(off[3]), int(off[4])
    cands = np.nonzero(seg[s:e] == -1)[0] + s
    perm = np.arange(sb.x.shape[0])
    perm[cands] = cands[::-1]
    sbp = synth.StackBatch(b, sb.x[torch.tensor(perm)], sb.weights, 1, sb.H, sb.d)
    outp = _run(sbp, off, seg, history_end=history_end, bf16=False)
    assert np.max(np.abs(outp[perm] - base)) < 1e-12
    # remove the first candidate of user 3
    keep = np.ones(sb.x.shape[0], dtype=bool)
    keep[cands[0]] = False
    rl = b.row_lengths.copy()
    rl[3] -= 1
    off2 = oracle.offsets_from_lengths(rl)
    seg2 = oracle.segment_ids(off2, b.cand_start, None if b.valid is None else b.valid[keep])
    out2 = ostack.stack_forward(sb.x[torch.tensor(keep)], sb.weights, off2, seg2, sb.H, 1, sb.scale,
                                history_end=history_end, bf16=False)
    assert np.max(np.abs(out2 - base[keep])) < 1e-12


def test_full_layers_without_candidates_match_sdpa():
    # Rows with no candidates and no padding: every layer is plain non-causal attention per user,
    # which torch's scaled_dot_product_attention computes independently of the mask builder.
    sb = synth.custom_stack([5, 9, 1], prefix=0, n_cand=0, H=2, d=4, n_layers=3, n_cand_only=0,
                            seed=6)
    off, seg = _layout(sb)
    got = _run(sb, off, seg, bf16=False)
    x = sb.x.to(torch.float64)
    for wq, wk, wv, wo in sb.weights:
        wq, wk, wv, wo = (w.to(torch.float64) for w in (wq, wk, wv, wo))
        new = x.clone()
        for bi in range(len(off) - 1):
            s, e = int(off[bi]), int(off[bi + 1])
            xs = x[s:e]
            q, k, v = ((xs @ w).reshape(e - s, sb.H, sb.d).transpose(0, 1) for w in (wq, wk, wv))
            a = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=sb.scale)
            new[s:e] = xs + a.transpose(0, 1).reshape(e - s, -1) @ wo
        x = new
    assert np.max(np.abs(got - x.numpy())) < 1e-10


def test_candidate_only_layer_per_candidate_sdpa():
    # Each candidate on its own: one query over [frozen history keys ; its own key], computed with
    # torch's scaled_dot_product_attention, one candidate at a time.
    rng = np.random.default_rng(7)
    H, d = 2, 4
    D = H * d
    hist_len, cand_cnt = [3, 0, 6], [2, 4, 1]
    hoff = oracle.offsets_from_lengths(hist_len)
    coff = oracle.offsets_from_lengths(cand_cnt)
    xh = rng.standard_normal((int(hoff[-1]), D))
    xc = rng.standard_normal((int(coff[-1]), D))
    w = tuple(rng.standard_normal((D, D)) / np.sqrt(D) for _ in range(4))
    got = ostack.candidate_only_layer(xc, xh, w, coff, hoff, H, 0.5, bf16=False)
    t = lambda a: torch.tensor(a, dtype=torch.float64)
    wq, wk, wv, wo = (t(m) for m in w)
    for b in range(3):
        hk = t(xh[hoff[b]:hoff[b + 1]]) @ wk
        hv = t(xh[hoff[b]:hoff[b + 1]]) @ wv
        for i in range(int(coff[b]), int(coff[b + 1])):
            xi = t(xc[i:i + 1])
            keys = torch.cat([hk, xi @ wk]).reshape(-1, H, d).transpose(0, 1)
            vals = torch.cat([hv, xi @ wv]).reshape(-1, H, d).transpose(0, 1)
            q = (xi @ wq).reshape(1, H, d).transpose(0, 1)
            a = torch.nn.functional.scaled_dot_product_attention(q, keys, vals, scale=0.5)
            ref = xi + a.transpose(0, 1).reshape(1, D) @ wo
            assert np.max(np.abs(got[i] - ref.numpy()[0])) < 1e-12


def test_closed_form_one_history_one_candidate():
    # H = 1, one user [h, c], one candidate-only layer with identity projections: the candidate's
    # new state is c + (e^{s1} h + e^{s2} c) / (e^{s1} + e^{s2}), s1 = scale c.h, s2 = scale c.c.
    D = 4
    eye = np.eye(D)
    h = np.array([0.5, -1.0, 2.0, 0.25])
    c = np.array([1.5, 0.5, -0.5, 1.0])
    x = np.stack([h, c])
    out = ostack.stack_forward(x, [(eye, eye, eye, eye)], [0, 2], np.array([1, -1], np.int8), 1, 1,
                               0.5, bf16=False)
    s1, s2 = 0.5 * c @ h, 0.5 * c @ c
    want = c + (np.exp(s1) * h + np.exp(s2) * c) / (np.exp(s1) + np.exp(s2))
    assert np.allclose(out[1], want, atol=1e-14) and np.array_equal(out[0], h)


def test_zero_output_projection_is_identity():
    sb = _small(8)
    off, seg = _layout(sb)
    w0 = [(wq, wk, wv, torch.zeros_like(wo)) for wq, wk, wv, wo in sb.weights]
    out = ostack.stack_forward(sb.x, w0, off, seg, sb.H, sb.n_cand_only, sb.scale)
    assert np.array_equal(out, sb.x.to(torch.float64).numpy())


def test_planted_padding_leak_is_caught(monkeypatch):
    # Plant a mistake in the oracle's split: padding rows join the frozen history. The fallback
    # (which never sees padding as a key) then disagrees.
    sb = _small(9)
    off, seg = _layout(sb)
    assert np.any(seg == 0)
    real = ostack.split_history_and_candidates

    def leaky(offsets, s):
        s2 = np.where(np.asarray(s) == 0, 1, s)
        return real(offsets, s2)

    monkeypatch.setattr(ostack, "split_history_and_candidates", leaky)
    a = _run(sb, off, seg, bf16=False)
    f = _run(sb, off, seg, bf16=False, fallback=True)
    assert np.max(np.abs(a - f)) > 1e-3


def test_planted_unfrozen_history_is_caught(monkeypatch):
    # Plant a mistake: the candidate-only layers take their history K/V from states that are not
    # the frozen ones (scaled by 1.01). The fallback disagrees.
    sb = _small(10, n_layers=3, n_cand_only=2)
    off, seg = _layout(sb)
    real = ostack.candidate_only_layer

    def drifting(xc, xh, w, *args, **kw):
        return real(xc, xh * 1.01, w, *args, **kw)

    monkeypatch.setattr(ostack, "candidate_only_layer", drifting)
    a = _run(sb, off, seg, bf16=False)
    f = _run(sb, off, seg, bf16=False, fallback=True)
    assert np.max(np.abs(a - f)) > 1e-4
