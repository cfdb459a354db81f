"""GPU parity of GroupLN (vs the oracle) and of the tensor-core GEMM with the
block's epilogues (vs float64 products of the same bf16 operands)."""

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synth
from _util import TOL_BF16, TOL_F32, assert_close_bf16_out, assert_close_rms, to_host

pytestmark = pytest.mark.gpu

mt = pytest.importorskip("generative_recommendation_ranking_b200")


def _gln_case(T, d, seed):
    rng = np.random.default_rng(seed)
    gid = rng.integers(0, 4, T).astype(np.int8)
    x = (rng.standard_normal((T, d)) * np.asarray(synth.group_scales())[gid][:, None] + 0.5).astype(np.float32)
    gamma = (1 + 0.3 * rng.standard_normal((4, d))).astype(np.float32)
    beta = (0.3 * rng.standard_normal((4, d))).astype(np.float32)
    return x, gid, gamma, beta


@pytest.mark.parametrize("d", [64, 256, 512, 1024, 2048])
@pytest.mark.parametrize("mode", ["f32", "f32_bf16", "bf16"])
def test_group_layernorm(d, mode):
    T = 3001
    x, gid, gamma, beta = _gln_case(T, d, d)
    dev = torch.device("cuda")
    if mode == "bf16":
        x = synth.bf16_round(x)
    xt = torch.from_numpy(x).to(dev)
    if mode == "bf16":
        xt = xt.to(torch.bfloat16)
    out_dt = torch.float32 if mode == "f32" else torch.bfloat16
    y = mt.group_layernorm(xt, torch.from_numpy(gid).to(dev), torch.from_numpy(gamma).to(dev),
                           torch.from_numpy(beta).to(dev), 1e-5, out_dtype=out_dt)
    ref = oracle.group_layernorm(x, gid, gamma, beta, 1e-5)
    if mode == "f32":
        assert_close_rms(to_host(y), ref, TOL_F32, f"gln {mode} d={d}")
    else:  # bf16 output: one rounding of the exact value
        assert_close_bf16_out(to_host(y), ref, f"gln {mode} d={d}")


def _bf16(a):
    return synth.bf16_round(a.astype(np.float32))


@pytest.mark.parametrize("M,N,K", [(1, 256, 64), (129, 512, 512), (1000, 2048, 512),
                                   (4097, 512, 2048), (300, 96, 1024), (2000, 1024, 4096)])
def test_gemm_plain_f32_out(M, N, K):
    rng = np.random.default_rng(M + N + K)
    a = _bf16(rng.standard_normal((M, K)))
    b = _bf16(rng.standard_normal((N, K)) / np.sqrt(K))
    bias = rng.standard_normal(N).astype(np.float32)
    dev = torch.device("cuda")
    out = mt.gemm(torch.from_numpy(a).to(dev).bfloat16(), torch.from_numpy(b).to(dev).bfloat16(),
                  torch.from_numpy(bias).to(dev), out_dtype=torch.float32)
    ref = a.astype(np.float64) @ b.astype(np.float64).T + bias
    assert_close_rms(to_host(out), ref, TOL_F32, f"gemm {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(777, 2048, 512), (1200, 4096, 1024)])
def test_gemm_qkvu_epilogue_f16_with_halved_q(M, N, K):
    rng = np.random.default_rng(5)
    a = _bf16(rng.standard_normal((M, K)))
    b = _bf16(rng.standard_normal((N, K)) / np.sqrt(K))
    dev = torch.device("cuda")
    q_cols = N // 4
    out = mt.gemm(torch.from_numpy(a).to(dev).bfloat16(), torch.from_numpy(b).to(dev).bfloat16(),
                  q_cols=q_cols, out_dtype=torch.float16)
    ref = a.astype(np.float64) @ b.astype(np.float64).T
    ref[:, :q_cols] *= 0.5
    assert_close_rms(to_host(out), ref, 4e-3, "gemm f16 out")  # f16 rounding: 2^-11 x max|out|


@pytest.mark.parametrize("M,N", [(1, 32), (100, 288), (257, 512), (700, 96)])
@pytest.mark.parametrize("form", ["f16", "bf16", "silu_bf16"])
def test_gemm_16bit_pairs_ragged(M, N, form):
    # K = 512 runs on CTA pairs with eight epilogue warps, each on half of a
    # tile's columns: M below one pair tile or off the 256-row grid, N off
    # the 256-column grid (one warp group's columns all past N)
    rng = np.random.default_rng(M * 7 + N)
    K = 512
    a = _bf16(rng.standard_normal((M, K)))
    b = _bf16(rng.standard_normal((N, K)) / np.sqrt(K))
    bias = rng.standard_normal(N).astype(np.float32) * 0.1
    dev = torch.device("cuda")
    epi = mt.MTGR_EPI_SILU if form == "silu_bf16" else mt.MTGR_EPI_NONE
    dt = torch.float16 if form == "f16" else torch.bfloat16
    out = mt.gemm(torch.from_numpy(a).to(dev).bfloat16(), torch.from_numpy(b).to(dev).bfloat16(),
                  torch.from_numpy(bias).to(dev), epi=epi, out_dtype=dt)
    ref = a.astype(np.float64) @ b.astype(np.float64).T + bias
    if form == "silu_bf16":
        ref = oracle.silu(ref)
    if form == "f16":
        assert_close_rms(to_host(out), ref, 4e-3, f"gemm f16 {M}x{N}")  # 2^-11 x max|out|
    else:
        assert_close_bf16_out(to_host(out), ref, f"gemm {form} {M}x{N}")


def test_gemm_silu_and_residual_epilogues():
    rng = np.random.default_rng(6)
    M, d, dff = 1500, 512, 2048
    g = _bf16(rng.standard_normal((M, d)))
    w1 = _bf16(rng.uniform(-1, 1, (dff, d)) * np.sqrt(6 / (d + dff)))
    w2 = _bf16(rng.uniform(-1, 1, (d, dff)) * np.sqrt(6 / (d + dff)))
    x = rng.standard_normal((M, d)).astype(np.float32) * 3
    dev = torch.device("cuda")
    h = mt.gemm(torch.from_numpy(g).to(dev).bfloat16(), torch.from_numpy(w1).to(dev).bfloat16(),
                epi=mt.MTGR_EPI_SILU, out_dtype=torch.bfloat16)
    h_ref = oracle.silu(g.astype(np.float64) @ w1.astype(np.float64).T)
    assert_close_bf16_out(to_host(h), h_ref, "silu epilogue")
    y = mt.gemm(h, torch.from_numpy(w2).to(dev).bfloat16(), epi=mt.MTGR_EPI_RESID,
                resid=torch.from_numpy(x).to(dev), out_dtype=torch.float32)
    hb = to_host(h).astype(np.float64)
    y_ref = hb @ w2.astype(np.float64).T + x
    assert_close_rms(to_host(y), y_ref, TOL_F32, "residual epilogue")


def test_gemm_residual_single_cta_ragged():
    # the residual form on single CTAs (K < 1024) with M and N off the tile
    # grid: the residual ring skips rows past M and column blocks past N
    rng = np.random.default_rng(16)
    M, N, K = 700, 288, 512
    a = _bf16(rng.standard_normal((M, K)))
    b = _bf16(rng.uniform(-1, 1, (N, K)) * np.sqrt(3 / K))
    x = rng.standard_normal((M, N)).astype(np.float32) * 2
    dev = torch.device("cuda")
    y = mt.gemm(torch.from_numpy(a).to(dev).bfloat16(), torch.from_numpy(b).to(dev).bfloat16(),
                epi=mt.MTGR_EPI_RESID, resid=torch.from_numpy(x).to(dev), out_dtype=torch.float32)
    y_ref = a.astype(np.float64) @ b.astype(np.float64).T + x
    assert_close_rms(to_host(y), y_ref, TOL_F32, "residual epilogue, single CTAs")


def test_gemm_f32_simt_path():
    rng = np.random.default_rng(7)
    a = rng.standard_normal((208, 64)).astype(np.float32)
    b = rng.standard_normal((256, 64)).astype(np.float32)
    dev = torch.device("cuda")
    out = mt.gemm(torch.from_numpy(a).to(dev), torch.from_numpy(b).to(dev), epi=mt.MTGR_EPI_SILU)
    ref = oracle.silu(a.astype(np.float64) @ b.astype(np.float64).T)
    assert_close_rms(to_host(out), ref, TOL_F32, "f32 gemm")
