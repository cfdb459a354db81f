"""GPU parity of the HSTU block's backward pass (training) against the
oracle's chain-rule gradients (oracle.hstu_block_backward): the fp32 path at
1e-4 x RMS, the bf16 tensor-core path at the gradient bars of tests/_util.py
(max-abs 5e-2 x RMS, RMS error 1e-2 x RMS), on small and ragged batches and
on the 512-user block workload, every gradient tensor compared element by
element against its own RMS."""

import numpy as np
import pytest
import torch

import oracle
import synth
from _util import (TOL_BF16_GRAD_PEAK, TOL_BF16_GRAD_RMS, TOL_F32, assert_grads_close,
                   oracle_backward_all_users, to_host, user_rows)

pytestmark = pytest.mark.gpu

mt = pytest.importorskip("generative_recommendation_ranking_b200")


def _gpu_backward(lens, ts, x, p, H, dtype, dy, norm=None):
    dev = torch.device("cuda")
    b = mt.PackedBatch(lens, ts, norm=norm)
    bw = mt.BlockWeights(p, H, dtype=dtype)
    xd = torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(dev)
    y, saved = mt.hstu_block_forward_train(bw, b, xd)
    y_inf = mt.hstu_block_forward(bw, b, xd)
    dx, grads = mt.hstu_block_backward(bw, b, xd, saved, torch.from_numpy(dy).to(dev))
    b.check()
    out = {k: to_host(v) for k, v in grads.items()}
    out["x"] = to_host(dx)
    return to_host(y), to_host(y_inf), out


def _compare(got, ref, tol, what):
    # fp32: largest error within 1e-4 of the largest element and RMS error
    # within 1e-4 of the RMS; bf16: the gradient bars of tests/_util.py
    if tol == TOL_F32:
        assert_grads_close(got, ref, TOL_F32, TOL_F32, what)
    else:
        assert_grads_close(got, ref, TOL_BF16_GRAD_PEAK, TOL_BF16_GRAD_RMS, what)


def test_fp32_block_backward_workload_full():
    w = synth.make_workload(0, seed=1)
    rng = np.random.default_rng(7)
    dy = rng.standard_normal(w["x"].shape).astype(np.float32)
    y, y_inf, g = _gpu_backward(w["lens"], w["ts"], w["x"], w["layers"][0], w["H"], "f32", dy)
    np.testing.assert_array_equal(y, y_inf)
    ref = oracle.hstu_block_backward(w["x"], w["lens"], w["ts"], w["layers"][0], w["H"], dy)
    _compare(g, ref, TOL_F32, "fp32 block")


def test_fp32_block_backward_with_biases_and_norm_override():
    w = synth.make_workload(0, seed=2)
    rng = np.random.default_rng(3)
    p = dict(w["layers"][0])
    d, dff = w["d"], w["d_ff"]
    p["b_qkvu"] = (0.1 * rng.standard_normal(4 * d)).astype(np.float32)
    p["b1"] = (0.1 * rng.standard_normal(dff)).astype(np.float32)
    p["b2"] = (0.1 * rng.standard_normal(d)).astype(np.float32)
    norm = (w["lens"].sum(1) * np.array([1.0, 2.0, 0.5, 1.5])).astype(np.float32)
    dy = rng.standard_normal(w["x"].shape).astype(np.float32)
    _, _, g = _gpu_backward(w["lens"], w["ts"], w["x"], p, w["H"], "f32", dy, norm=norm)
    ref = oracle.hstu_block_backward(w["x"], w["lens"], w["ts"], p, w["H"], dy, norm=norm)
    _compare(g, ref, TOL_F32, "fp32 block with biases")


def test_bf16_block_backward_small_batch():
    w = synth.make_workload(2, seed=5, B=6)
    dy = np.random.default_rng(11).standard_normal(w["x"].shape).astype(np.float32)
    y, y_inf, g = _gpu_backward(w["lens"], w["ts"], w["x"], w["layers"][0], w["H"], "bf16", dy)
    np.testing.assert_array_equal(y, y_inf)  # the training forward computes the same output
    ref = oracle.hstu_block_backward(w["x"], w["lens"], w["ts"], w["layers"][0], w["H"], dy)
    _compare(g, ref, "bf16", "bf16 block, 6 users")


# users of 1 token, U-only, S-only, R-only, candidate-only, lengths on and
# off the 128-row tile grid, an empty user
RAGGED = np.array([[1, 0, 0, 0], [0, 0, 1, 0], [0, 0, 0, 1], [0, 127, 0, 1], [64, 64, 0, 0],
                   [0, 0, 128, 0], [0, 0, 0, 129], [10, 100, 17, 129], [0, 0, 0, 0],
                   [3, 250, 5, 0], [24, 300, 60, 200]], np.int32)
# users whose every attention row reduces to a single weight (one token, no
# U/S keys): their block output is exact up to a scale that GroupLN_2 divides
# out, while their gradient carries 1/sigma(G) and with it the f16 SiLU
# weight's relative error (an absolute error of about 2^-11 |h| on a weight
# near zero) -- ill-conditioned at bf16, exact on the fp32 path
SINGLE_WEIGHT = [0, 1, 2, 5, 6, 8]


def _ragged_case(d, dff, dtype, rng):
    lens = RAGGED
    ts = rng.integers(0, 6, size=int(lens.sum())).astype(np.int64)  # many ties
    x = synth.make_tokens(lens, d, rng)
    p = synth.make_block_params(d, dff, rng, dtype=dtype)
    p["b_qkvu"] = (0.1 * rng.standard_normal(4 * d)).astype(np.float32)
    p["b1"] = (0.1 * rng.standard_normal(dff)).astype(np.float32)
    p["b2"] = (0.1 * rng.standard_normal(d)).astype(np.float32)
    dy = rng.standard_normal(x.shape).astype(np.float32)
    return lens, ts, x, p, dy


def test_fp32_block_backward_ragged_edge_users():
    # every edge user, the single-weight ones included, with biases and ties
    lens, ts, x, p, dy = _ragged_case(64, 256, "f32", np.random.default_rng(4))
    _, _, g = _gpu_backward(lens, ts, x, p, 2, "f32", dy)
    ref = oracle.hstu_block_backward(x, lens, ts, p, 2, dy)
    _compare(g, ref, TOL_F32, "fp32 block, ragged users")


def test_bf16_block_backward_ragged_edge_users():
    # the same layouts on the tensor-core path; the single-weight users get a
    # zero upstream gradient, so their gradient rows must come out exactly
    # zero (nothing leaks in from a neighbouring user) while their tiles still
    # run through every kernel
    lens, ts, x, p, dy = _ragged_case(128, 256, "bf16", np.random.default_rng(4))
    dy[user_rows(lens, SINGLE_WEIGHT)] = 0.0
    _, _, g = _gpu_backward(lens, ts, x, p, 2, "bf16", dy)
    rows = user_rows(lens, SINGLE_WEIGHT)
    assert np.count_nonzero(g["x"][rows]) == 0
    ref = oracle.hstu_block_backward(x, lens, ts, p, 2, dy)
    _compare(g, ref, "bf16", "bf16 block, ragged users")


def test_bf16_block_backward_full_workload():
    # the 512-user block workload (459k tokens): every input-gradient row and
    # every parameter gradient (sums over all tokens) against the oracle
    w = synth.make_workload(2)
    dy = np.random.default_rng(21).standard_normal(w["x"].shape).astype(np.float32)
    _, _, g = _gpu_backward(w["lens"], w["ts"], w["x"], w["layers"][0], w["H"], "bf16", dy)
    for k, v in g.items():
        assert np.isfinite(v).all(), k
    ref = oracle_backward_all_users(w, dy)
    _compare(g, ref, "bf16", "bf16 block, 512 users")
