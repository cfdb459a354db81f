"""GPU parity of the weight-gradient GEMM (mtgr_gemm_wgrad): out = a^T b summed
over tokens, against float64 products of the same bf16 operands. The shapes
reach every branch of the kernel's schedule on 74 resident CTA pairs: the
balanced slab schedule (tiles x slabs a multiple of the pairs), the fallback
slab count when the tokens are too few for it, slabs with no token block,
stream-K when the output has too many tiles, and pair tiles whose second CTA
half lies partly or wholly past M or N."""

import numpy as np
import pytest
import torch

import synth
from _util import TOL_F32, assert_close_rms, to_host

pytestmark = pytest.mark.gpu

mt = pytest.importorskip("generative_recommendation_ranking_b200")


def _operands(T, M, N, seed, lda=None, ldb=None):
    rng = np.random.default_rng(seed)
    a = synth.bf16_round(rng.standard_normal((T, lda or M)).astype(np.float32))
    b = synth.bf16_round(rng.standard_normal((T, ldb or N)).astype(np.float32))
    return a, b


def _dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda().bfloat16()


@pytest.mark.parametrize("M,N,T", [
    (192, 384, 5000),   # 2 pair tiles: rank 1 holds rows 128-191 of 256, columns 384-511 are past N
    (512, 2048, 3001),  # the block's dW2 shape; 37 slabs of one or two 64-token blocks
    (2048, 512, 1000),  # too few tokens for 37 slabs: 4 slabs on 64 pairs
    (64, 32, 200),      # one tile, 74 slabs over 4 token blocks: most units empty
    (4096, 1024, 700),  # 64 pair tiles: stream-K ranges across tiles
])
def test_wgrad_matches_float64(M, N, T):
    a, b = _operands(T, M, N, M + N + T)
    out = mt.gemm_wgrad(_dev(a), _dev(b))
    ref = a.astype(np.float64).T @ b.astype(np.float64)
    assert_close_rms(to_host(out), ref, TOL_F32, f"wgrad {M}x{N} over {T} tokens")


def test_wgrad_strided_operands_and_accumulate():
    # a and b are column slices of wider token-major rows (lda, ldb > M, N);
    # the second call adds onto the first call's sums
    M, N, T = 320, 136, 4100
    a, b = _operands(T, M, N, 9, lda=512, ldb=256)
    ad, bd = _dev(a), _dev(b)
    out = mt.gemm_wgrad(ad[:, :M], bd[:, :N])
    out = mt.gemm_wgrad(ad[:, 64:64 + M], bd[:, 8:8 + N], out=out)
    ref = (a[:, :M].astype(np.float64).T @ b[:, :N].astype(np.float64)
           + a[:, 64:64 + M].astype(np.float64).T @ b[:, 8:8 + N].astype(np.float64))
    assert_close_rms(to_host(out), ref, TOL_F32, "wgrad strided, accumulated")


def test_wgrad_no_tokens_gives_zeros():
    a = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    b = torch.empty(0, 512, dtype=torch.bfloat16, device="cuda")
    out = mt.gemm_wgrad(a, b)
    assert out.shape == (256, 512)
    assert int(torch.count_nonzero(out).item()) == 0
