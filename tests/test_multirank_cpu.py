"""The multi-rank paths on CPU: two gloo ranks agree on the max-over-ranks timings and on the
whole-job (weak-scaling) throughput, as the NCCL ranks do on GPUs; and two ranks that split one
batch by users (jca_shard_users) reproduce the unsharded batch's output from their shards."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        elapsed, kernel = 100.0 + 7.0 * rank, 50.0 - rank
        got = bench.max_over_ranks([elapsed, kernel], dist, "cpu")
        value = bench.weak_scaling_value(6.0e11, world, 10, got[0])
        out[rank] = torch.tensor([got[0], got[1], value], dtype=torch.float64)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank():
    world = 2
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    r0, r1 = out[0].tolist(), out[1].tolist()
    assert r0 == r1
    assert r0[0] == 107.0 and r0[1] == 50.0
    assert r0[2] == pytest.approx(2 * 6.0e11 * 10 / 0.107)


def test_single_process_is_a_no_op():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    assert bench.weak_scaling_value(10.0, 1, 2, 1000.0) == 20.0


HIST = [0, 3, 300, 17, 64, 129, 2, 500, 40, 1, 250, 7]
PREFIX, NCAND, H, D, SEED = 2, 5, 2, 16, 9


def _shard_rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import numpy as np
    import oracle
    import synth
    from candidate_isolated_jagged_b200 import jca
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        hist = np.asarray(HIST, dtype=np.int64)
        shard, load = jca.shard_users(hist + PREFIX + NCAND, hist + PREFIX, world)
        # every rank computed the same split from the same lengths
        mine = torch.from_numpy(shard.astype(np.int64))
        gathered = [torch.empty_like(mine) for _ in range(world)]
        dist.all_gather(gathered, mine)
        same = all(torch.equal(g, mine) for g in gathered)
        users = np.nonzero(shard == rank)[0].tolist()
        b = synth.users_batch(hist, users, PREFIX, NCAND, H, D, SEED)
        off = oracle.offsets_from_lengths(b.row_lengths)
        seg = oracle.segment_ids(off, b.cand_start)
        o = oracle.jagged_cand_attn(b.q, b.k, b.v, off, seg, b.scale)
        out[rank] = (same, users, torch.from_numpy(o), load.tolist())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_users_and_reproduce_the_whole_batch():
    """Each rank takes its users from the LPT split and computes only their rows (the oracle stands
    in for the kernels on CPU); the shards are disjoint, cover every user, stay within Graham's
    bound, and their outputs placed back at the users' rows equal the unsharded batch's output."""
    import sys
    sys.path.insert(0, ROOT)
    import numpy as np
    import oracle
    import synth
    from candidate_isolated_jagged_b200 import jca
    world = 2
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_shard_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    hist = np.asarray(HIST, dtype=np.int64)
    full = synth.users_batch(hist, range(len(hist)), PREFIX, NCAND, H, D, SEED)
    off = oracle.offsets_from_lengths(full.row_lengths)
    ref = oracle.jagged_cand_attn(full.q, full.k, full.v, off,
                                  oracle.segment_ids(off, full.cand_start), full.scale)
    seen = []
    for r in range(world):
        same, users, o, load = out[r]
        assert same
        seen += users
        rows = np.concatenate([np.arange(off[u], off[u + 1]) for u in users]) if users else []
        assert np.array_equal(o.numpy(), ref[rows])
    assert sorted(seen) == list(range(len(hist)))
    costs = np.array([jca.user_tile_cost(h + PREFIX + NCAND, h + PREFIX) for h in hist])
    loads = out[0][3]
    assert sum(loads) == costs.sum()
    assert max(loads) <= costs.sum() / world + (1 - 1 / world) * costs.max()
