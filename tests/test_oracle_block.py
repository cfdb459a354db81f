"""Pins of the oracle's whole HSTU block (summary page, Method): closed forms and
the invariants the pages imply (candidate independence, aggregation = expanded
rows, no temporal leakage)."""

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synth


def _small_user_batch(seed, B=2, d=16, d_ff=40):
    rng = np.random.default_rng(seed)
    lens = np.array([[2, 6, 4, 5], [3, 4, 2, 3]][:B], np.int32)
    ts = synth.make_timestamps(lens, rng)
    x = synth.make_tokens(lens, d, rng).astype(np.float64)
    p = synth.make_block_params(d, d_ff, rng, dtype="f32")
    return lens, ts, x, p


def _mlp_torch(z, p):
    h = F.silu(F.linear(torch.as_tensor(z), torch.as_tensor(p["w1"], dtype=torch.float64)))
    return F.linear(h, torch.as_tensor(p["w2"], dtype=torch.float64)).numpy()


def test_block_closed_form_zero_query_weights():
    # W_q = 0 -> every score is 0 -> silu(0) = 0 -> G = 0 -> GroupLN_2(0) = beta_2
    # of the token's group -> X_out = X + MLP(beta_2[g])
    lens, ts, x, p = _small_user_batch(0)
    d = x.shape[1]
    p = dict(p)
    p["w_qkvu"] = p["w_qkvu"].copy()
    p["w_qkvu"][:d] = 0.0
    y = oracle.hstu_block(x, lens, ts, p, H=2)
    _, _, gid = oracle.pack_offsets(lens)
    ref = x + _mlp_torch(np.asarray(p["gln2_beta"], np.float64)[gid], p)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_block_zero_output_weights_is_identity():
    lens, ts, x, p = _small_user_batch(1)
    p = dict(p)
    p["w2"] = np.zeros_like(p["w2"])
    np.testing.assert_array_equal(oracle.hstu_block(x, lens, ts, p, H=2), x)


def _one_user(seed, n_u=3, n_s=9, n_r=5, K=6, d=16, d_ff=32):
    rng = np.random.default_rng(seed)
    lens = np.array([[n_u, n_s, n_r, K]], np.int32)
    ts = synth.make_timestamps(lens, rng)
    x = synth.make_tokens(lens, d, rng).astype(np.float64)
    layers = synth.make_stack_params(2, d, d_ff, rng, dtype="f32")
    return lens, ts, x, layers


def test_candidate_permutation_permutes_outputs():
    lens, ts, x, layers = _one_user(2)
    c0 = int(lens[0, :3].sum())
    K = int(lens[0, 3])
    perm = np.random.default_rng(9).permutation(K)
    idx = np.concatenate([np.arange(c0), c0 + perm])
    y = oracle.hstu_stack(x, lens, ts, layers, H=2)
    yp = oracle.hstu_stack(x[idx], lens, ts[idx], layers, H=2)
    np.testing.assert_allclose(yp, y[idx], rtol=1e-12, atol=1e-12)


def test_candidate_removal_at_fixed_n_leaves_output_unchanged():
    lens, ts, x, layers = _one_user(3)
    N = int(lens.sum())
    c0 = int(lens[0, :3].sum())
    K = int(lens[0, 3])
    y = oracle.hstu_stack(x, lens, ts, layers, H=2)
    keep = [1, 4]
    idx = np.concatenate([np.arange(c0), c0 + np.array(keep)])
    lens2 = lens.copy()
    lens2[0, 3] = len(keep)
    y2 = oracle.hstu_stack(x[idx], lens2, ts[idx], layers, H=2, norm=np.array([N], float))
    np.testing.assert_allclose(y2, y[idx], rtol=1e-12, atol=1e-12)
    assert K > len(keep)


def test_aggregated_pass_equals_expanded_rows():
    lens, ts, x, layers = _one_user(4, K=5)
    wl = dict(lens=lens, ts=ts, x=x)
    ex = synth.sweep_expanded(wl)
    y = oracle.hstu_stack(x, lens, ts, layers, H=2)
    ye = oracle.hstu_stack(ex["x"], ex["lens"], ex["ts"], layers, H=2, norm=ex["norm"])
    n_ctx = int(lens[0, :3].sum())
    K = int(lens[0, 3])
    row = n_ctx + 1
    for i in range(K):
        np.testing.assert_allclose(ye[i * row + n_ctx], y[n_ctx + i], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(ye[i * row:i * row + n_ctx], y[:n_ctx], rtol=1e-12, atol=1e-12)


def test_temporal_replay_no_leakage():
    # perturbing R tokens stamped at or after a candidate's exposure time leaves
    # that candidate's output bit-for-bit unchanged
    lens, ts, x, layers = _one_user(5, n_r=8, K=6)
    c0 = int(lens[0, :3].sum())
    r0 = int(lens[0, :2].sum())
    y = oracle.hstu_stack(x, lens, ts, layers, H=2)
    for c in range(int(lens[0, 3])):
        tc = ts[c0 + c]
        late = [r0 + j for j in range(int(lens[0, 2])) if ts[r0 + j] >= tc]
        x2 = x.copy()
        x2[late] += 5.0
        y2 = oracle.hstu_stack(x2, lens, ts, layers, H=2)
        np.testing.assert_array_equal(y2[c0 + c], y[c0 + c])


def test_stack_of_identity_layers():
    lens, ts, x, layers = _one_user(6)
    layers = [dict(p, w2=np.zeros_like(p["w2"])) for p in layers]
    np.testing.assert_array_equal(oracle.hstu_stack(x, lens, ts, layers, H=2), x)


def test_block_bias_terms():
    lens, ts, x, p = _small_user_batch(7)
    d, d_ff = x.shape[1], p["w1"].shape[0]
    rng = np.random.default_rng(11)
    pb = dict(p, b_qkvu=np.zeros(4 * d), b1=np.zeros(d_ff), b2=rng.standard_normal(d))
    np.testing.assert_allclose(oracle.hstu_block(x, lens, ts, pb, H=2),
                               oracle.hstu_block(x, lens, ts, p, H=2) + pb["b2"], rtol=1e-12, atol=1e-12)
