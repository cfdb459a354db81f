"""Pins of the oracle's dynamic mask (fun-rec 7.3.4 Rules 1-3; summary page,
Method) against hand-derived matrices, a per-cell brute force and special cases."""

import numpy as np
import pytest

import oracle


def _golden_mask(golden, name):
    g = golden(name)
    n_u, n_s, n_r, n_k = g["lens"]
    return (n_u, n_s, n_r, n_k), np.asarray(g["ts"], np.int64), np.asarray(g["mask"], bool)


def test_leakage_example(golden):
    lens, ts, expected = _golden_mask(golden, "mask_leakage_example.txt")
    M = oracle.user_mask(*lens, ts)
    np.testing.assert_array_equal(M, expected)
    # the point of the example: candidate B (12:30) does not see the 13:00 click
    n_ctx = lens[0] + lens[1]
    b_row, rt_1300 = n_ctx + lens[2] + 1, n_ctx + 1
    assert not M[b_row, rt_1300]


def test_toy_layout(golden):
    lens, ts, expected = _golden_mask(golden, "mask_toy_layout.txt")
    np.testing.assert_array_equal(oracle.user_mask(*lens, ts), expected)


def _brute_force_mask(n_u, n_s, n_r, n_k, ts):
    """Per-cell evaluation of the three rules with plain if-statements."""
    N = n_u + n_s + n_r + n_k
    grp = []
    for g, n in enumerate((n_u, n_s, n_r, n_k)):
        grp += [g] * n
    M = np.zeros((N, N), bool)
    for i in range(N):
        for j in range(N):
            if grp[j] in (0, 1):              # rule 1: static keys
                M[i, j] = True
            elif grp[j] == 2:                 # rule 2: real-time keys, causal in time
                query_time_known = grp[i] != 0
                M[i, j] = (i == j) or (query_time_known and ts[j] < ts[i])
            else:                             # rule 3: a candidate sees only itself
                M[i, j] = i == j
    return M


@pytest.mark.parametrize("seed", range(20))
def test_brute_force_random(seed):
    rng = np.random.default_rng(1000 + seed)
    n_u, n_s, n_r, n_k = (int(v) for v in rng.integers(0, 6, size=4))
    N = n_u + n_s + n_r + n_k
    # small time range so that ties occur
    ts = rng.integers(0, 6, size=N).astype(np.int64)
    np.testing.assert_array_equal(oracle.user_mask(n_u, n_s, n_r, n_k, ts),
                                  _brute_force_mask(n_u, n_s, n_r, n_k, ts))


def test_rt_only_strictly_increasing_is_causal_triangle():
    # with only R tokens in strictly increasing time order the mask is the
    # textbook causal (lower-triangular, diagonal included) mask
    n = 9
    ts = np.arange(100, 100 + n, dtype=np.int64) * 7
    M = oracle.user_mask(0, 0, n, 0, ts)
    np.testing.assert_array_equal(M, np.tril(np.ones((n, n), bool)))


def test_tied_rt_timestamps_not_visible():
    ts = np.array([5, 5, 5], dtype=np.int64)
    M = oracle.user_mask(0, 0, 3, 0, ts)
    np.testing.assert_array_equal(M, np.eye(3, dtype=bool))


def test_candidates_block_is_diagonal_and_us_columns_full():
    rng = np.random.default_rng(3)
    n_u, n_s, n_r, n_k = 3, 5, 4, 6
    ts = np.concatenate([np.zeros(3), rng.integers(0, 1000, 5), np.sort(rng.integers(1000, 2000, 4)),
                         rng.integers(1000, 2000, 6)]).astype(np.int64)
    M = oracle.user_mask(n_u, n_s, n_r, n_k, ts)
    c0 = n_u + n_s + n_r
    np.testing.assert_array_equal(M[:, c0:][c0:], np.eye(n_k, dtype=bool))
    assert not M[:c0, c0:].any()          # no context token sees a candidate
    assert M[:, :n_u + n_s].all()         # rule 1 columns are all ones


def test_visible_pairs_counts_mask(golden):
    lens, ts, expected = _golden_mask(golden, "mask_leakage_example.txt")
    assert oracle.visible_pairs(np.array([lens]), ts) == int(expected.sum())
