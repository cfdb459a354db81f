"""Pins of the oracle's GroupLN (fun-rec 7.3.3) and masked SiLU attention
(summary page, Method) against library routines on special cases and invariants."""

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle


def _t(a):
    return torch.as_tensor(np.asarray(a, np.float64))


def test_gln_single_group_is_layer_norm():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((37, 48)) * 3 + 1
    gamma = rng.standard_normal((1, 48))
    beta = rng.standard_normal((1, 48))
    y = oracle.group_layernorm(x, np.zeros(37, np.int8), gamma, beta, eps=1e-5)
    ref = F.layer_norm(_t(x), (48,), _t(gamma[0]), _t(beta[0]), eps=1e-5).numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_gln_four_groups_is_layer_norm_per_subset():
    rng = np.random.default_rng(1)
    T, d = 60, 32
    x = rng.standard_normal((T, d)) * rng.uniform(0.1, 10, size=(T, 1))
    gid = rng.integers(0, 4, size=T).astype(np.int8)
    gamma = rng.standard_normal((4, d))
    beta = rng.standard_normal((4, d))
    y = oracle.group_layernorm(x, gid, gamma, beta, eps=1e-5)
    for g in range(4):
        rows = gid == g
        ref = F.layer_norm(_t(x[rows]), (d,), _t(gamma[g]), _t(beta[g]), eps=1e-5).numpy()
        np.testing.assert_allclose(y[rows], ref, rtol=1e-12, atol=1e-12)


def _rand_qkvu(rng, T, d):
    return rng.standard_normal((T, 4 * d))


def test_attention_static_only_user_is_dense_silu_attention():
    # a user with only U and S tokens has no masked cell: the attention is the
    # dense silu(Q K^T) V / N of the formula, computed here with torch routines
    rng = np.random.default_rng(2)
    n_u, n_s, d, H = 5, 11, 16, 2
    T = n_u + n_s
    qkvu = _rand_qkvu(rng, T, d)
    ts = np.concatenate([np.zeros(n_u), rng.integers(0, 1000, n_s)]).astype(np.int64)
    G = oracle.hstu_attention(qkvu, np.array([[n_u, n_s, 0, 0]]), ts, H)
    q, k, v, u = (_t(qkvu[:, i * d:(i + 1) * d]) for i in range(4))
    dh = d // H
    ref = torch.zeros(T, d, dtype=torch.float64)
    for h in range(H):
        c = slice(h * dh, (h + 1) * dh)
        ref[:, c] = F.silu(q[:, c] @ k[:, c].T) @ v[:, c] / T
    np.testing.assert_allclose(G, (ref * u).numpy(), rtol=1e-12, atol=1e-12)


def test_attention_score_orientation_query_row():
    # one query row that sees every key: its output uses q_0 . k_j (query row 0
    # against all keys), not k_0 . q_j
    rng = np.random.default_rng(3)
    d, H, T = 8, 1, 6
    qkvu = _rand_qkvu(rng, T, d)
    G = oracle.hstu_attention(qkvu, np.array([[T, 0, 0, 0]]), np.zeros(T, np.int64), H)
    q0, K, V, u0 = qkvu[0, :d], qkvu[:, d:2 * d], qkvu[:, 2 * d:3 * d], qkvu[0, 3 * d:]
    ref = (F.silu(_t(K @ q0)).numpy()[:, None] * V).sum(0) / T * u0
    np.testing.assert_allclose(G[0], ref, rtol=1e-12, atol=1e-12)


def test_attention_normaliser_override_scales_output():
    rng = np.random.default_rng(4)
    lens = np.array([[2, 6, 3, 4], [1, 5, 0, 2]], np.int32)
    T = int(lens.sum())
    ts = rng.integers(0, 50, size=T).astype(np.int64)
    qkvu = _rand_qkvu(rng, T, 16)
    G = oracle.hstu_attention(qkvu, lens, ts, 2)
    G2 = oracle.hstu_attention(qkvu, lens, ts, 2, norm=2.0 * lens.sum(1))
    np.testing.assert_allclose(G2, G / 2, rtol=1e-13, atol=1e-15)


def test_attention_heads_are_independent_column_slices():
    # head h of an H-head call equals a 1-head call on that head's columns
    rng = np.random.default_rng(5)
    lens = np.array([[2, 7, 4, 5]], np.int32)
    T, d, H = int(lens.sum()), 24, 3
    dh = d // H
    ts = np.concatenate([np.zeros(2), rng.integers(0, 100, 7), np.sort(rng.integers(100, 200, 4)),
                         rng.integers(100, 200, 5)]).astype(np.int64)
    qkvu = _rand_qkvu(rng, T, d)
    G = oracle.hstu_attention(qkvu, lens, ts, H)
    for h in range(H):
        cols = np.concatenate([np.arange(i * d + h * dh, i * d + (h + 1) * dh) for i in range(4)])
        Gh = oracle.hstu_attention(qkvu[:, cols], lens, ts, 1)
        np.testing.assert_allclose(G[:, h * dh:(h + 1) * dh], Gh, rtol=1e-13, atol=1e-15)


def test_attention_users_do_not_interact():
    rng = np.random.default_rng(6)
    lens = np.array([[2, 4, 3, 2], [1, 3, 2, 3]], np.int32)
    T = int(lens.sum())
    ts = rng.integers(0, 50, size=T).astype(np.int64)
    qkvu = _rand_qkvu(rng, T, 8)
    G = oracle.hstu_attention(qkvu, lens, ts, 1)
    n0 = int(lens[0].sum())
    G1 = oracle.hstu_attention(qkvu[n0:], lens[1:], ts[n0:], 1)
    np.testing.assert_allclose(G[n0:], G1, rtol=0, atol=0)
    qkvu2 = qkvu.copy()
    qkvu2[:n0] = rng.standard_normal((n0, 32))
    np.testing.assert_array_equal(oracle.hstu_attention(qkvu2, lens, ts, 1)[n0:], G[n0:])


def test_silu_values():
    x = np.array([-30.0, -1.0, 0.0, 0.5, 2.0, 40.0])
    np.testing.assert_allclose(oracle.silu(x), F.silu(_t(x)).numpy(), rtol=1e-14, atol=1e-300)
