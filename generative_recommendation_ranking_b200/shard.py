"""Length-balanced sharding of users across GPUs (host logic).

Users are independent — packing never lets one user attend to another (MTGR
summary page, Method; chenhuiyu blog, the training-system list: "sequence
packing" and per-GPU batch sizes balanced by real sequence length) — so a
batch splits across data-parallel ranks by user, with the weights replicated
and no collective in the forward. Each user's cost is estimated from its
length and each user goes to the least-loaded rank, longest first
(longest-processing-time greedy).
"""

from __future__ import annotations

import heapq

import numpy as np


def user_cost(lens: np.ndarray, d: int, d_ff: int) -> np.ndarray:
    """Estimated forward FLOPs per user: the projections and MLP (2 (4 d^2 +
    2 d d_ff) per token) plus the attention at full visibility (4 d N^2)."""
    n = np.asarray(lens, np.int64).reshape(-1, 4).sum(axis=1).astype(np.float64)
    return 2.0 * (4 * d * d + 2 * d * d_ff) * n + 4.0 * d * n * n


def balance_users(lens: np.ndarray, world: int, d: int, d_ff: int) -> list:
    """Partition user indices into ``world`` shards of near-equal cost.
    Each shard lists its users in ascending order."""
    if world < 1:
        raise ValueError("world must be >= 1")
    cost = user_cost(lens, d, d_ff)
    order = sorted(range(len(cost)), key=lambda u: (-cost[u], u))
    heap = [(0.0, r) for r in range(world)]
    shards = [[] for _ in range(world)]
    for u in order:
        load, r = heapq.heappop(heap)
        shards[r].append(u)
        heapq.heappush(heap, (load + cost[u], r))
    return [np.asarray(sorted(s), dtype=np.int64) for s in shards]


def shard_rows(lens: np.ndarray, users: np.ndarray) -> np.ndarray:
    """Packed-row indices of the given users (in the given order)."""
    n = np.asarray(lens, np.int64).reshape(-1, 4).sum(axis=1)
    off = np.concatenate([[0], np.cumsum(n)])
    if len(users) == 0:
        return np.zeros(0, np.int64)
    return np.concatenate([np.arange(off[u], off[u + 1]) for u in users])


def imbalance(lens: np.ndarray, shards: list, d: int, d_ff: int) -> float:
    """max shard cost / mean shard cost (1.0 = perfect balance)."""
    cost = user_cost(lens, d, d_ff)
    loads = np.array([cost[s].sum() for s in shards])
    return float(loads.max() / max(loads.mean(), 1e-300))


def rank_shard(lens: np.ndarray, ts: np.ndarray, world: int, rank: int, d: int, d_ff: int):
    """This rank's share of one global batch, as the data-parallel forward runs
    it: the rank's users (ascending), their rows in the global packed layout,
    and the sub-batch (lens [n, 4], ts [rows]) the rank packs and processes on
    its own GPU. Every rank calls it with the same global ``lens`` and ``ts``,
    so the shards are disjoint and cover the batch; a rank's output rows go
    back to ``rows`` of the global output."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    lens = np.asarray(lens).reshape(-1, 4)
    mine = balance_users(lens, world, d, d_ff)[rank]
    rows = shard_rows(lens, mine)
    return (mine, rows, np.ascontiguousarray(lens[mine], dtype=np.int32),
            np.ascontiguousarray(np.asarray(ts)[rows], dtype=np.int64))
