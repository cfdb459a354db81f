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
        shards = sh.balance_users(lens, world, w["d"], w["d_ff"])
        mine = shards[rank]
        rows = sh.shard_rows(lens, mine)
        y = oracle.hstu_stack(x[rows], lens[mine], ts[rows], w["layers"], w["H"])
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
