"""Pins of the CPU oracle against what the pages and the mathematics fix (CPU only).

Each pin checks the oracle against something other than itself: values the pages print (fixtures
under tests/golden/, each with its citation), closed forms, invariants the pages state, special cases
that reduce to a library routine, and an independent pure-Python brute force on tiny inputs.
The mutation tests at the end plant plausible mistakes in copies of the oracle's rule and check
that at least one pin catches each of them.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from oracle import jagged_oracle as jo
import synth
from candidate_isolated_jagged_b200 import metrics

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def batch_seg(batch):
    off = oracle.offsets_from_lengths(batch.row_lengths)
    seg = oracle.segment_ids(off, batch.cand_start, batch.valid)
    return off, seg


def to_lists(t):
    return t.to(torch.float64).tolist()


# ------------------------------------------------------------------------------------------------
# Storage pins ('HSTU scale' tutorial)
# ------------------------------------------------------------------------------------------------

def test_offsets_worked_example():
    g = load("offsets_worked_example.json")
    off = oracle.offsets_from_lengths(g["lengths"])
    assert off.tolist() == g["offsets"]
    values = [x for s in g["sequences"] for x in s]
    assert oracle.split_by_offsets(values, off) == g["sequences"]
    lo, hi = g["third_slice"]
    assert (int(off[2]), int(off[3])) == (lo, hi)
    assert values[lo:hi] == g["sequences"][2]
    assert len(g["lengths"]) * max(g["lengths"]) == g["dense_positions"]
    assert int(off[-1]) == g["real_positions"]


def test_offsets_empty_sequences_and_errors():
    assert oracle.offsets_from_lengths([]).tolist() == [0]
    assert oracle.offsets_from_lengths([0, 3, 0, 0, 2]).tolist() == [0, 0, 3, 3, 3, 5]
    with pytest.raises(ValueError):
        oracle.offsets_from_lengths([1, -1])


def test_packing_counts():
    g = load("packing_counts.json")
    padded, ragged, ratio = oracle.packing_counts(g["lengths"])
    assert padded == g["padded_positions"]
    assert ragged == g["ragged_positions"]
    # closed form of the page's pair-work ratio: B * max^2 / sum n^2
    assert ratio == pytest.approx(3 * 1000 ** 2 / g["per_sequence_pair_work"], rel=1e-15)
    assert round(ratio, 3) == 2.970


# ------------------------------------------------------------------------------------------------
# Segment IDs, bounds, mask (候选隔离注意力掩码)
# ------------------------------------------------------------------------------------------------

def test_segment_ids_hand_cases():
    g = load("segment_ids_hand.json")
    for c in g["cases"]:
        got = oracle.attention_segment_ids(c["row_len"], c["candidate_start"],
                                           np.asarray(c["padding_mask"], dtype=bool),
                                           c["attend_padded_history"])
        assert got.tolist() == c["segment_ids"], c


def test_bounds_hand_case():
    g = load("segment_ids_hand.json")["bounds_case"]
    hl, hh, cl, ch, ok = oracle.bounds_from_segment_ids(np.asarray(g["segment_ids"], np.int8),
                                                        g["offsets"])
    assert hl.tolist() == g["hist_lo"]
    assert hh.tolist() == g["hist_hi"]
    assert cl.tolist() == g["cand_lo"]
    assert ch.tolist() == g["cand_hi"]
    assert ok.all()
    # no candidates -> cand_lo = cand_hi = row end; a history token after a candidate is flagged
    hl, hh, cl, ch, ok = oracle.bounds_from_segment_ids(np.asarray([1, 1, 0, 1, -1, 1], np.int8),
                                                        [0, 3, 6])
    assert (cl[0], ch[0]) == (3, 3)
    assert ok.tolist() == [True, False]


def test_mask_matches_printed_table():
    g = load("mask_table.json")
    mask = oracle.history_candidate_mask(np.asarray(g["segment_ids"], np.int8))
    for name, row in g["printed_rows"].items():
        i = g["layout"].index(name)
        assert mask[i].astype(int).tolist() == row, name
    # reading for the row the extracted table lacks: H2 behaves as H0 and H1
    assert mask[g["layout"].index("H2")].tolist() == mask[g["layout"].index("H0")].tolist()


def test_mask_padding_and_no_cross_user():
    seg = np.asarray([1, 0, 1, -1, 0, -1], np.int8)
    m = oracle.history_candidate_mask(seg)
    assert not m[1].any() and not m[4].any()          # padding queries see nothing
    assert not m[:, 1].any() and not m[:, 4].any()    # nobody sees padding keys
    assert m[3].tolist() == [1, 0, 1, 1, 0, 0]
    # across users: an output row depends only on its own user's K/V
    b = synth.tiny()
    off, seg = batch_seg(b)
    ref = oracle.jagged_cand_attn(b.q, b.k, b.v, off, seg, b.scale)
    k2 = b.k.clone()
    k2[int(off[1]):int(off[2])] = torch.randn(int(off[2] - off[1]), b.H, b.d).to(torch.bfloat16)
    got = oracle.jagged_cand_attn(b.q, k2, b.v, off, seg, b.scale)
    assert np.array_equal(ref[:int(off[1])], got[:int(off[1])])
    assert np.array_equal(ref[int(off[2]):], got[int(off[2]):])


# ------------------------------------------------------------------------------------------------
# Attention pins
# ------------------------------------------------------------------------------------------------

def brute_vs_oracle(batch, mask_fn=jo.history_candidate_mask):
    off, seg = batch_seg(batch)
    ref = oracle.jagged_cand_attn(batch.q, batch.k, batch.v, off, seg, batch.scale, mask_fn=mask_fn)
    bf = brute.jagged_attention(to_lists(batch.q), to_lists(batch.k), to_lists(batch.v),
                                [int(x) for x in batch.row_lengths], seg.tolist(), batch.scale)
    bf = np.asarray(bf, dtype=np.float64)
    return np.max(np.abs(ref - bf))


def test_brute_force_tiny():
    assert brute_vs_oracle(synth.tiny()) < 1e-12


def test_brute_force_holes_everywhere():
    # padding at the front of the history, in its middle, and among the candidates
    hist = [3, 4, 0, 2]
    b0 = synth.custom_batch(hist, prefix=1, n_cand=[2, 3, 2, 0], H=2, d=16, seed=5)
    valid = np.ones(b0.T, np.uint8)
    valid[[1, 6, 9, 13, 15]] = 0
    b = synth.custom_batch(hist, prefix=1, n_cand=[2, 3, 2, 0], H=2, d=16, seed=5,
                           valid_override=valid)
    assert brute_vs_oracle(b) < 1e-12


def test_no_candidates_equals_sdpa():
    # two-tower user tower: prefix + history only, all segment 1, bidirectional
    # (候选隔离注意力掩码, section 在哪里生效) == plain non-causal softmax attention
    b = synth.custom_batch([5, 17, 1], prefix=2, n_cand=0, H=3, d=32, seed=3)
    off, seg = batch_seg(b)
    assert (seg == 1).all()
    ref = oracle.jagged_cand_attn(b.q, b.k, b.v, off, seg, b.scale)
    for u in range(b.B):
        s, e = int(off[u]), int(off[u + 1])
        q = b.q[s:e].to(torch.float64).transpose(0, 1)
        k = b.k[s:e].to(torch.float64).transpose(0, 1)
        v = b.v[s:e].to(torch.float64).transpose(0, 1)
        sd = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=b.scale)
        assert np.max(np.abs(sd.transpose(0, 1).numpy() - ref[s:e])) < 1e-12


def test_single_key_closed_forms():
    # a candidate with neither prefix nor history sees only itself -> output = its own v
    b = synth.custom_batch([0, 1], prefix=0, n_cand=[3, 0], H=2, d=16, seed=4)
    off, seg = batch_seg(b)
    out = oracle.jagged_cand_attn(b.q, b.k, b.v, off, seg, b.scale)
    v = b.v.to(torch.float64).numpy()
    assert np.array_equal(out[0:3], v[0:3])
    # a user whose row is a single history token -> output = that token's v
    assert np.array_equal(out[3], v[3])


def test_padding_rows_output_zero():
    b = synth.three_users()
    off, seg = batch_seg(b)
    out = oracle.jagged_cand_attn(b.q, b.k, b.v, off, seg, b.scale, users=[0, 1])
    pad = np.nonzero(seg[:int(off[2])] == 0)[0]
    assert pad.size == 10
    assert np.all(out[pad] == 0.0)


def test_rows_sampler_matches_full():
    b = synth.three_users()
    off, seg = batch_seg(b)
    full = oracle.jagged_cand_attn(b.q, b.k, b.v, off, seg, b.scale, users=[0, 1])
    rows = np.array([0, 5, 12, 17, 20, 49, 50, 60, 155, 187])
    got = oracle.jagged_cand_attn_rows(b.q, b.k, b.v, off, seg, b.scale, rows)
    assert np.max(np.abs(got - full[rows])) < 1e-12


# --- invariants stated by the pages (候选隔离注意力掩码, sections 核心结论 and 为什么需要它) ---

def _one_user(hist=6, prefix=1, n_cand=5, seed=11, H=2, d=16):
    return synth.custom_batch([hist], prefix=prefix, n_cand=n_cand, H=H, d=d, seed=seed)


def close(a, b):
    """Equal up to fp64 rounding order (BLAS sums a different number of exact zeros)."""
    return a.shape == b.shape and np.max(np.abs(a - b)) < 1e-13


def _run(q, k, v, row_len, cand_start, scale):
    off = oracle.offsets_from_lengths([row_len])
    seg = oracle.segment_ids(off, [cand_start])
    return oracle.jagged_cand_attn(q, k, v, off, seg, scale)


def test_candidate_isolation_permute_add_remove():
    b = _one_user()
    L, cs = int(b.row_lengths[0]), int(b.cand_start[0])
    ref = _run(b.q, b.k, b.v, L, cs, b.scale)
    # permute candidates
    perm = torch.tensor(list(range(cs)) + list(cs + np.random.default_rng(0).permutation(L - cs)))
    out = _run(b.q[perm], b.k[perm], b.v[perm], L, cs, b.scale)
    assert close(out, ref[perm.numpy()])
    # remove candidate 2 (others unchanged)
    keep = torch.tensor([i for i in range(L) if i != cs + 2])
    out = _run(b.q[keep], b.k[keep], b.v[keep], L - 1, cs, b.scale)
    assert close(out, ref[keep.numpy()])
    # add two more candidates
    extra = synth.custom_batch([0], prefix=0, n_cand=2, H=b.H, d=b.d, seed=99)
    q2, k2, v2 = (torch.cat([t, e]) for t, e in ((b.q, extra.q), (b.k, extra.k), (b.v, extra.v)))
    out = _run(q2, k2, v2, L + 2, cs, b.scale)
    assert close(out[:L], ref)


def test_history_independent_of_candidates():
    b = _one_user()
    L, cs = int(b.row_lengths[0]), int(b.cand_start[0])
    ref = _run(b.q, b.k, b.v, L, cs, b.scale)
    q2, k2, v2 = b.q.clone(), b.k.clone(), b.v.clone()
    g = torch.Generator().manual_seed(7)
    for t in (q2, k2, v2):
        t[cs:] = torch.randn(L - cs, b.H, b.d, generator=g).to(torch.bfloat16)
    out = _run(q2, k2, v2, L, cs, b.scale)
    assert close(out[:cs], ref[:cs])
    out = _run(b.q[:cs], b.k[:cs], b.v[:cs], cs, cs, b.scale)   # all candidates removed
    assert close(out, ref[:cs])


def test_cand_only_equals_full_candidate_rows():
    # candidate-only layer == candidate rows of the full layer given the same K/V
    # (候选隔离注意力掩码, section 只更新候选的末尾层)
    b = synth.custom_batch([4, 0, 9], prefix=[1, 0, 2], n_cand=[3, 2, 4], H=2, d=16, seed=8)
    off, seg = batch_seg(b)
    full = oracle.jagged_cand_attn(b.q, b.k, b.v, off, seg, b.scale)
    hist_idx, cand_idx, hl, cc = [], [], [], []
    for u in range(b.B):
        s, e, cs = int(off[u]), int(off[u + 1]), int(off[u] + b.cand_start[u])
        hist_idx += list(range(s, cs))
        cand_idx += list(range(cs, e))
        hl.append(cs - s)
        cc.append(e - cs)
    hi, ci = torch.tensor(hist_idx, dtype=torch.long), torch.tensor(cand_idx, dtype=torch.long)
    got = oracle.cand_only_attn(b.q[ci], b.k[ci], b.v[ci], oracle.offsets_from_lengths(cc),
                                b.k[hi], b.v[hi], oracle.offsets_from_lengths(hl), None, b.scale)
    assert np.max(np.abs(got - full[ci.numpy()])) < 1e-12
    rows = np.array([0, 4, 8])
    got_rows = oracle.cand_only_attn(b.q[ci], b.k[ci], b.v[ci], oracle.offsets_from_lengths(cc),
                                     b.k[hi], b.v[hi], oracle.offsets_from_lengths(hl), None,
                                     b.scale, cand_rows=rows)
    assert np.max(np.abs(got_rows - got[rows])) < 1e-12


def test_cand_only_history_padding_is_ignored():
    cb = synth.custom_cand_only([5, 3], [2, 3], H=2, d=16, seed=3)
    hseg = np.ones(cb.Th, np.int8)
    hseg[[1, 6]] = 0
    coff, hoff = oracle.offsets_from_lengths(cb.cand_counts), oracle.offsets_from_lengths(cb.hist_lengths)
    got = oracle.cand_only_attn(cb.cq, cb.ck, cb.cv, coff, cb.hk, cb.hv, hoff, hseg, cb.scale)
    keep = torch.tensor([i for i in range(cb.Th) if hseg[i] == 1])
    ref = oracle.cand_only_attn(cb.cq, cb.ck, cb.cv, coff, cb.hk[keep], cb.hv[keep],
                                oracle.offsets_from_lengths([4, 2]), None, cb.scale)
    assert np.max(np.abs(got - ref)) < 1e-12


# ------------------------------------------------------------------------------------------------
# Work counting pins
# ------------------------------------------------------------------------------------------------

def test_allowed_pairs_closed_form():
    for b in (synth.tiny(), synth.three_users()):
        off, seg = batch_seg(b)
        n1 = [int((seg[int(off[u]):int(off[u + 1])] == 1).sum()) for u in range(b.B)]
        nc = [int((seg[int(off[u]):int(off[u + 1])] == -1).sum()) for u in range(b.B)]
        assert oracle.allowed_pairs(off, seg) == metrics.allowed_pairs_from_counts(n1, nc)
    b = synth.tiny()
    off, seg = batch_seg(b)
    assert oracle.allowed_pairs(off, seg) == 91
    assert metrics.effective_flops(91, b.H, b.d) == 11648.0


def test_flops_cross_check_against_retrieval_formula():
    g = load("flops_per_candidate.json")
    D, Lu = g["D"], g["L_u"]
    # the page's per-candidate formula reproduces its reported totals
    f = lambda D_, Lt, Nl: 4 * D_ * Lt * (4 * D_ + Lu) * Nl
    assert f(128, 1, 5) / 1e6 == pytest.approx(g["reported_mflops"]["128D-5L-1tok"],
                                                rel=g["reported_rel_tolerance"])
    assert f(64, 8, 3) / 1e6 == pytest.approx(g["reported_mflops"]["64D-3L-8tok"],
                                              rel=g["reported_rel_tolerance"])
    # our counter for the retrieval workload (H=4, d=32: H*d = D) minus the self term equals the
    # page's attention term 4*D*L_u per candidate per layer
    H, d = 4, 32
    per_cand = metrics.effective_flops(metrics.allowed_pairs_from_counts([Lu], [1]) - Lu * Lu, H, d)
    assert per_cand == 4 * H * d * (Lu + 1) == 123392
    assert per_cand - 4 * H * d == g["attention_term_per_candidate_per_layer"] == 4 * D * Lu
    # and the oracle's explicit-mask count agrees on a small retrieval-shaped user
    cb = synth.custom_cand_only([7], [5], H=1, d=16)
    seg = np.asarray([1] * 7 + [-1] * 5, np.int8)
    assert oracle.allowed_pairs([0, 12], seg) - 7 * 7 == 5 * (7 + 1)


def test_work_items_cover_every_tile():
    b = synth.three_users()
    off, seg = batch_seg(b)
    items = oracle.work_items(off, seg, b.H)
    assert len(items) == b.H * sum(-(-int(L) // 256) for L in b.row_lengths)
    costs = {(it[0]): it[3] for it in items}
    assert costs == {0: 1, 1: 1, 2: 8}


# ------------------------------------------------------------------------------------------------
# Mutation tests: plausible mistakes planted in copies of the oracle's rule must fail a pin
# ------------------------------------------------------------------------------------------------

def _mask_ok_against_table(mask_fn):
    g = load("mask_table.json")
    mask = mask_fn(np.asarray(g["segment_ids"], np.int8))
    return all(mask[g["layout"].index(n)].astype(int).tolist() == r
               for n, r in g["printed_rows"].items())


def _mut_causal(seg):
    m = jo.history_candidate_mask(seg)
    return m & np.tril(np.ones_like(m))


def _mut_cand_sees_cands(seg):
    s = np.asarray(seg)
    return jo.history_candidate_mask(seg) | ((s == -1)[:, None] & (s == -1)[None, :])


def _mut_no_self(seg):
    s = np.asarray(seg)
    return (s == 1)[None, :] & ((s == 1) | (s == -1))[:, None]


def _mut_history_sees_cands(seg):
    s = np.asarray(seg)
    return jo.history_candidate_mask(seg) | ((s == 1)[:, None] & (s == -1)[None, :])


def _mut_transposed(seg):
    return jo.history_candidate_mask(seg).T


def _mut_padding_keys_visible(seg):
    s = np.asarray(seg)
    return jo.history_candidate_mask(seg) | ((s != 0)[:, None] & (s == 0)[None, :])


@pytest.mark.parametrize("mut", [_mut_causal, _mut_cand_sees_cands, _mut_no_self,
                                 _mut_history_sees_cands, _mut_transposed,
                                 _mut_padding_keys_visible])
def test_planted_mask_mistakes_are_caught(mut):
    caught = not _mask_ok_against_table(mut)
    b = synth.custom_batch([3, 4], prefix=1, n_cand=[2, 3], H=2, d=16, seed=5, pad_hist_to=4)
    caught = caught or brute_vs_oracle(b, mask_fn=mut) > 1e-6
    assert caught


def test_planted_softmax_mistakes_are_caught(monkeypatch):
    orig = jo.masked_softmax_attention

    def no_scale(q, k, v, mask, scale):
        return orig(q, k, v, mask, 1.0)

    def swapped_qk(q, k, v, mask, scale):
        return orig(k, q, v, mask, scale)

    def no_norm(q, k, v, mask, scale):
        out = orig(q, k, v, mask, scale)
        return out * 1.5

    for bad in (no_scale, swapped_qk, no_norm):
        monkeypatch.setattr(jo, "masked_softmax_attention", bad)
        assert brute_vs_oracle(synth.tiny()) > 1e-6
    monkeypatch.setattr(jo, "masked_softmax_attention", orig)
    assert brute_vs_oracle(synth.tiny()) < 1e-12


def test_planted_segment_mistake_is_caught():
    g = load("segment_ids_hand.json")
    c = g["cases"][0]

    def off_by_one(row_len, cs, pm, flag):
        return oracle.attention_segment_ids(row_len, cs + 1, pm, flag)

    got = off_by_one(c["row_len"], c["candidate_start"], np.asarray(c["padding_mask"], bool), False)
    assert got.tolist() != c["segment_ids"]
