"""Multi-rank host logic on the CPU (gloo, world size 2): length-balanced user
sharding reproduces the unsharded result, and the bench's max-over-ranks
timing reduction."""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

from generative_recommendation_ranking_b200 import shard  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_balance_users_partition_and_balance():
    import synth
    rng = np.random.default_rng(0)
    lens = synth.make_lengths(synth.WORKLOADS[3], rng, B=256)
    for world in (1, 2, 3, 8):
        shards = shard.balance_users(lens, world, 1024, 4096)
        allu = np.sort(np.concatenate(shards))
        np.testing.assert_array_equal(allu, np.arange(256))
        assert shard.imbalance(lens, shards, 1024, 4096) < 1.05


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import synth
        from generative_recommendation_ranking_b200 import shard as sh
        w = synth.make_workload(0, seed=5)
        lens = np.concatenate([w["lens"], np.array([[2, 40, 6, 3], [1, 10, 2, 9]], np.int32)])
        rng = np.random.default_rng(5)
        ts = synth.make_timestamps(lens, rng)
        x = synth.make_tokens(lens, w["d"], rng)
        # the shard the product path runs on this rank (bench.py --gpus N):
        # its users, their global rows and its own packed sub-batch
        mine, rows, lens_r, ts_r = sh.rank_shard(lens, ts, world, rank, w["d"], w["d_ff"])
        np.testing.assert_array_equal(lens_r, lens[mine])
        np.testing.assert_array_equal(ts_r, ts[rows])
        y = oracle.hstu_stack(x[rows], lens_r, ts_r, w["layers"], w["H"])
        gathered = [None] * world
        dist.all_gather_object(gathered, (mine, rows, y))
        # the bench's timing reduction: max over ranks
        t = torch.tensor([float(rank + 1)], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        if rank == 0:
            full = oracle.hstu_stack(x, lens, ts, w["layers"], w["H"])
            out = np.zeros_like(full)
            for _, r, yy in gathered:
                out[r] = yy
            q.put((float(np.max(np.abs(out - full))), float(t.item()),
                   sorted(int(u) for g in gathered for u in g[0])))
    finally:
        dist.destroy_process_group()


def test_two_rank_sharded_forward_matches_unsharded():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    err, tmax, users = q.get(timeout=240)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert err < 1e-9
    assert tmax == 2.0
    assert users == list(range(6))


def test_rank_shards_cover_the_global_batch_once():
    # the row maps every rank's sub-batch uses: disjoint, complete, each rank's
    # rows in its own packed order (users ascending, each user's rows in
    # order), and the packed sub-batch is exactly those rows
    import synth
    rng = np.random.default_rng(1)
    lens = synth.make_lengths(synth.WORKLOADS[2], rng, B=64)
    ts = synth.make_timestamps(lens, rng)
    T = int(lens.sum())
    for world in (1, 2, 3, 8):
        seen = np.zeros(T, np.int64)
        costs = []
        for r in range(world):
            mine, rows, lens_r, ts_r = shard.rank_shard(lens, ts, world, r, 512, 2048)
            assert np.all(np.diff(mine) > 0)
            assert len(rows) == int(lens_r.sum())
            np.testing.assert_array_equal(ts_r, ts[rows])
            np.testing.assert_array_equal(rows, shard.shard_rows(lens, mine))
            seen[rows] += 1
            costs.append(shard.user_cost(lens, 512, 2048)[mine].sum())
        assert (seen == 1).all()
        assert max(costs) / (sum(costs) / world) < 1.1
    with pytest.raises(ValueError):
        shard.rank_shard(lens, ts, 2, 2, 512, 2048)


def test_bench_rank_workloads_share_weights_and_split_one_batch():
    # bench.py's per-rank workload: same weights on every rank, users drawn
    # once globally and split by rank_shard
    import argparse
    sys.path.insert(0, ROOT)
    import bench
    args = argparse.Namespace(config=2, users=12, seed=0)
    parts = [bench.rank_workload(args, 3, r) for r in range(3)]
    assert all(p[1] == 36 for p in parts)
    assert sum(p[0]["lens"].shape[0] for p in parts) == 36
    for p in parts[1:]:
        for a, b in zip(p[0]["layers"], parts[0][0]["layers"]):
            for k in a:
                np.testing.assert_array_equal(a[k], b[k])
    one, b1 = bench.rank_workload(args, 1, 0)
    assert b1 == 12 and one["lens"].shape[0] == 12
