"""Host-side split of one batch's users over several GPUs (jca_shard_users), on the CPU.

Users never interact (no position reads across a user boundary: 候选隔离注意力掩码, section
段 ID：掩码的表达方式), so a batch is split by users with no exchange. The split is
longest-processing-time-first over each user's tile cost. Pinned here against what scheduling
theory fixes: Graham's list-scheduling bound (largest load <= total / m + (1 - 1/m) max cost) on
random batches, the 4/3 - 1/(3m) LPT guarantee against the exact optimum found by brute force on
small batches, a hand-worked instance, determinism, and the argument errors.
"""

import itertools

import numpy as np
import pytest

import synth
from candidate_isolated_jagged_b200 import jca


def _costs(rl, nk):
    return np.array([jca.user_tile_cost(a, b) for a, b in zip(rl, nk)], dtype=np.int64)


def test_tile_cost_hand_worked():
    # 68 rows, 4 keys: one query tile x one key tile; 4164 rows (4 prefix + 4096 + 64), 4100 keys:
    # 33 query tiles x 33 key tiles; an empty row costs nothing; keys = 0 still costs its tiles.
    assert jca.user_tile_cost(68, 4) == 1
    assert jca.user_tile_cost(4164, 4100) == 33 * 33
    assert jca.user_tile_cost(0, 0) == 0
    assert jca.user_tile_cost(129, 0) == 2
    assert jca.user_tile_cost(300, 200) == 3 * 2


def test_hand_worked_split():
    # costs 6, 6, 3, 2, 2 (users 0..4) over 2 shards: LPT puts 6 | 6, then 3 -> shard 0,
    # 2 -> shard 1, 2 -> shard 1: loads 9 and 10.
    rl = [6 * 128, 6 * 128, 3 * 128, 2 * 128, 2 * 128]
    nk = [1, 1, 1, 1, 1]
    shard, load = jca.shard_users(rl, nk, 2)
    assert shard.tolist() == [0, 1, 0, 1, 1]
    assert load.tolist() == [9, 10]


def _makespan(costs, assign, m):
    loads = np.zeros(m, dtype=np.int64)
    np.add.at(loads, assign, costs)
    return int(loads.max())


@pytest.mark.parametrize("m", [2, 3, 4])
def test_lpt_guarantee_against_brute_force(m):
    rng = np.random.default_rng(m)
    for _ in range(25):
        B = int(rng.integers(1, 8))
        rl = rng.integers(0, 1500, size=B)
        nk = np.minimum(rng.integers(0, 1500, size=B), rl)
        costs = _costs(rl, nk)
        shard, load = jca.shard_users(rl, nk, m)
        assert _makespan(costs, shard, m) == int(load.max())
        best = min(_makespan(costs, np.array(a), m) for a in itertools.product(range(m), repeat=B))
        assert load.max() <= (4.0 / 3.0 - 1.0 / (3 * m)) * best + 1e-9


@pytest.mark.parametrize("m", [1, 2, 8, 64])
def test_graham_bound_and_cover_on_lognormal_users(m):
    n = synth.lognormal_history_lengths(2048, seed=5)
    rl, nk = n + 68, n + 4
    costs = _costs(rl, nk)
    shard, load = jca.shard_users(rl, nk, m)
    assert shard.min() >= 0 and shard.max() < m
    assert int(load.sum()) == int(costs.sum())
    for s in range(m):
        assert int(costs[shard == s].sum()) == int(load[s])
    assert load.max() <= costs.sum() / m + (1 - 1 / m) * costs.max() + 1e-9
    # deterministic: the same lengths give the same split
    again, _ = jca.shard_users(rl, nk, m)
    assert np.array_equal(shard, again)


def test_more_shards_than_users_and_empty_batch():
    shard, load = jca.shard_users([200, 10], [100, 4], 4)
    assert sorted(shard.tolist()) == [0, 1] and load.tolist()[2:] == [0, 0]
    shard, load = jca.shard_users([], [], 3)
    assert shard.size == 0 and load.tolist() == [0, 0, 0]


def test_argument_errors():
    with pytest.raises(jca.JcaError):
        jca.shard_users([5], [6], 2)          # more keys than rows
    with pytest.raises(jca.JcaError):
        jca.shard_users([-1], [0], 2)
    with pytest.raises(jca.JcaError):
        jca.shard_users([5], [1], 0)
