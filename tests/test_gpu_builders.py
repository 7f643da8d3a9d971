"""GPU parity of the builder kernels (offsets, segment IDs, bounds, work queue) against the oracle:
bit-exact for every index and ID, in int32 and int64, plus the device-side data errors."""

import numpy as np
import pytest
import torch

import oracle
import synth
from candidate_isolated_jagged_b200 import jca
from helpers import dev

pytestmark = pytest.mark.gpu

IDX = [torch.int32, torch.int64]


def _lengths_cases():
    rng = np.random.default_rng(3)
    big = rng.integers(0, 40, size=5000)
    big[rng.integers(0, 5000, size=500)] = 0
    n256 = synth.users256_history_lengths(0) + 4 + 64
    return {"worked": [2, 5, 1], "three": [10, 100, 1000], "empty_batch": [], "one_zero": [0],
            "zeros": [0, 0, 3, 0], "random5000": big.tolist(), "users256": n256.tolist()}


@pytest.mark.parametrize("idx", IDX)
@pytest.mark.parametrize("case", list(_lengths_cases()))
def test_offsets_bit_exact(idx, case):
    lengths = _lengths_cases()[case]
    ln = torch.tensor(lengths, dtype=idx, device=dev())
    off = torch.full((len(lengths) + 1,), -7, dtype=idx, device=dev())
    st = jca.new_status(dev())
    jca.jca_offsets_from_lengths(ln, off, st)
    jca.check_status(st)
    assert off.cpu().numpy().tolist() == oracle.offsets_from_lengths(lengths).tolist()


@pytest.mark.parametrize("idx", IDX)
def test_offsets_errors(idx):
    st = jca.new_status(dev())
    ln = torch.tensor([3, -1, 2], dtype=idx, device=dev())
    off = torch.zeros(4, dtype=idx, device=dev())
    jca.jca_offsets_from_lengths(ln, off, st)
    assert int(st.item()) == 1
    if idx == torch.int32:
        st.zero_()
        ln = torch.tensor([2 ** 30, 2 ** 30, 2 ** 30], dtype=idx, device=dev())
        jca.jca_offsets_from_lengths(ln, off, st)
        assert int(st.item()) == 1
    # an error already recorded stops later calls: offsets stay untouched
    off.fill_(-5)
    jca.jca_offsets_from_lengths(torch.tensor([1, 2, 3], dtype=idx, device=dev()), off, st)
    assert off.cpu().tolist() == [-5] * 4


def _seg_batch(name):
    if name == "tiny":
        b = synth.tiny()
        return b.row_lengths, b.cand_start, None
    if name == "three_users":
        b = synth.three_users()
        return b.row_lengths, b.cand_start, b.valid
    if name == "users256":
        n = synth.users256_history_lengths(0)
        rl = n + 4 + 64
        return rl, n + 4, None
    if name == "random_holes":
        rng = np.random.default_rng(11)
        rl = rng.integers(0, 300, size=400)
        rl[::37] = 0
        cs = np.array([rng.integers(0, L + 1) for L in rl])
        valid = (rng.random(int(rl.sum())) > 0.2).astype(np.uint8)
        return rl, cs, valid
    raise KeyError(name)


@pytest.mark.parametrize("idx", IDX)
@pytest.mark.parametrize("name", ["tiny", "three_users", "users256", "random_holes"])
@pytest.mark.parametrize("attend", [False, True])
def test_segment_ids_and_bounds_bit_exact(idx, name, attend):
    rl, cs, valid = _seg_batch(name)
    off_np = oracle.offsets_from_lengths(rl)
    T = int(off_np[-1])
    seg_ref = oracle.segment_ids(off_np, cs, valid, attend)
    off = torch.tensor(off_np, dtype=idx, device=dev())
    cst = torch.tensor(np.asarray(cs), dtype=idx, device=dev())
    vt = None if valid is None else torch.tensor(valid, dtype=torch.uint8, device=dev())
    seg = torch.full((T,), 9, dtype=torch.int8, device=dev())
    st = jca.new_status(dev())
    jca.jca_build_segment_ids(off, cst, vt, attend, seg, st)
    jca.check_status(st)
    assert np.array_equal(seg.cpu().numpy(), seg_ref)
    B = len(rl)
    outs = [torch.full((B,), -3, dtype=idx, device=dev()) for _ in range(4)]
    jca.jca_bounds_from_segment_ids(seg, off, *outs, st)
    jca.check_status(st)
    hl, hh, cl, ch, ok = oracle.bounds_from_segment_ids(seg_ref, off_np)
    assert ok.all()
    for got, ref in zip(outs, (hl, hh, cl, ch)):
        assert np.array_equal(got.cpu().numpy().astype(np.int64), ref)


def test_segment_and_bounds_errors():
    st = jca.new_status(dev())
    off = torch.tensor([0, 3, 2, 6], dtype=torch.int64, device=dev())       # decreasing
    cs = torch.tensor([1, 0, 1], dtype=torch.int64, device=dev())
    seg = torch.zeros(6, dtype=torch.int8, device=dev())
    jca.jca_build_segment_ids(off, cs, None, False, seg, st)
    assert int(st.item()) == 2
    st.zero_()
    off = torch.tensor([0, 3, 6], dtype=torch.int64, device=dev())
    jca.jca_build_segment_ids(off, torch.tensor([4, 0], dtype=torch.int64, device=dev()), None,
                              False, seg, st)
    assert int(st.item()) == 3                                            # cand_start > length
    st.zero_()
    bad_layout = torch.tensor([1, -1, 1, 1, 1, -1], dtype=torch.int8, device=dev())
    outs = [torch.zeros(2, dtype=torch.int64, device=dev()) for _ in range(4)]
    jca.jca_bounds_from_segment_ids(bad_layout, off, *outs, st)
    assert int(st.item()) == 4
    st.zero_()
    bad_value = torch.tensor([1, 2, -1, 1, 1, -1], dtype=torch.int8, device=dev())
    jca.jca_bounds_from_segment_ids(bad_value, off, *outs, st)
    assert int(st.item()) == 5
    st.zero_()
    jca.jca_bounds_from_segment_ids(bad_layout[:6], torch.tensor([0, 3, 5], dtype=torch.int64,
                                                                 device=dev()), *outs, st)
    assert int(st.item()) == 2                                            # off[B] != T


@pytest.mark.parametrize("idx", IDX)
@pytest.mark.parametrize("name", ["tiny", "three_users", "users256", "random_holes"])
def test_work_queue_matches_item_set(idx, name):
    rl, cs, valid = _seg_batch(name)
    H = 3
    off_np = oracle.offsets_from_lengths(rl)
    seg_np = oracle.segment_ids(off_np, cs, valid)
    hl, hh, _, _, _ = oracle.bounds_from_segment_ids(seg_np, off_np)
    T = int(off_np[-1])
    B = len(rl)
    cnt = np.array([int((seg_np[off_np[b]:off_np[b + 1]] == 1).sum()) for b in range(B)],
                   dtype=np.int32)
    ref = oracle.work_items(off_np, seg_np, H)
    max_items = jca.jca_max_work_items(B, T, H)
    items = torch.full((max_items * 4,), -1, dtype=torch.int32, device=dev())
    n = torch.zeros(1, dtype=torch.int32, device=dev())
    st = jca.new_status(dev())
    jca.jca_build_work_queue(torch.tensor(off_np, dtype=idx, device=dev()),
                             torch.tensor(hl, dtype=idx, device=dev()),
                             torch.tensor(hh, dtype=idx, device=dev()),
                             torch.tensor(cnt, device=dev()), T, T, H, items, n, st)
    jca.check_status(st)
    n = int(n.item())
    assert n == len(ref)
    got = items[: 4 * n].view(n, 4).cpu().numpy().astype(np.int64)
    costs = -(-(got[:, 3] & 0x7FFFFFFF) // 128)
    assert np.all(np.diff(costs) <= 0), "items must come largest cost first"
    # decode and compare as a set with the oracle's items
    users = np.searchsorted(off_np, got[:, 0], side="right") - 1
    tiles = (got[:, 0] - off_np[users]) // 256
    heads = got[:, 1] >> 9
    decoded = sorted(zip(users.tolist(), heads.tolist(), tiles.tolist(), costs.tolist()))
    assert decoded == sorted(ref)
    rows = got[:, 1] & 511
    L = (off_np[users + 1] - off_np[users])
    assert np.array_equal(rows, np.minimum(256, L - tiles * 256))
    assert np.array_equal(got[:, 2], hl[users])
    holes = (got[:, 3] >> 31) & 1
    assert np.array_equal(holes, (cnt[users] != (hh - hl)[users]).astype(np.int64))
