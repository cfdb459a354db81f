"""GPU parity of the masked SiLU attention (tensor-core and fp32 paths) against
the oracle, on small ragged batches, edge cases and the full 256-user
attention workload (sampled users)."""

import numpy as np
import pytest
import torch

import oracle
import synth
from _util import (TOL_BF16, TOL_F32, assert_close_bf16_out, assert_close_rms, sample_users,
                   to_host, user_rows)

pytestmark = pytest.mark.gpu

mt = pytest.importorskip("generative_recommendation_ranking_b200")


def _run(lens, ts, qkvu, d, H, in_dtype, out_dtype, norm=None):
    dev = torch.device("cuda")
    b = mt.PackedBatch(lens, ts, norm=norm)
    q = torch.from_numpy(qkvu).to(dev).to(in_dtype)
    g = mt.hstu_attention(b, q, d, H, out_dtype=out_dtype)
    b.check()
    return to_host(g)


def _random_case(seed, B, d, scale=1.0 / np.sqrt(8.0)):
    rng = np.random.default_rng(seed)
    lens = np.stack([rng.integers(0, 20, B), rng.integers(0, 500, B), rng.integers(0, 120, B),
                     rng.integers(0, 200, B)], 1).astype(np.int32)
    ts = synth.make_timestamps(lens, rng)
    qkvu = synth.bf16_round((rng.standard_normal((int(lens.sum()), 4 * d)) * scale).astype(np.float32))
    return lens, ts, qkvu


@pytest.mark.parametrize("in_dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_tc_small_ragged_batch(in_dtype, out_dtype):
    d, H = 256, 4
    lens, ts, qkvu = _random_case(11, 9, d)
    if in_dtype == torch.float16:
        qkvu = torch.from_numpy(qkvu).half().float().numpy()
    g = _run(lens, ts, qkvu, d, H, in_dtype, out_dtype)
    ref = oracle.hstu_attention(qkvu, lens, ts, H)
    if out_dtype == torch.float32:
        assert_close_rms(g, ref, TOL_BF16, f"attention {in_dtype} -> f32")
    else:  # bf16 output: one rounding of the exact value on top
        assert_close_bf16_out(g, ref, f"attention {in_dtype} -> bf16")


@pytest.mark.parametrize("dh", [32, 64])
def test_f32_path(dh):
    H = 2
    d = H * dh
    rng = np.random.default_rng(dh)
    lens = np.array([[4, 32, 8, 8]] * 3 + [[2, 200, 30, 40]], np.int32)
    ts = synth.make_timestamps(lens, rng)
    qkvu = rng.standard_normal((int(lens.sum()), 4 * d)).astype(np.float32) * 0.5
    g = _run(lens, ts, qkvu, d, H, torch.float32, torch.float32)
    assert_close_rms(g, oracle.hstu_attention(qkvu, lens, ts, H), TOL_F32, "f32 attention")


def test_edge_users():
    d, H = 128, 2
    lens = np.array([[1, 0, 0, 0], [0, 0, 1, 0], [0, 0, 0, 1], [0, 127, 0, 1], [64, 64, 0, 0],
                     [0, 0, 128, 0], [0, 0, 0, 129], [10, 100, 17, 129], [0, 0, 0, 0],
                     [3, 250, 5, 0]], np.int32)
    rng = np.random.default_rng(2)
    ts = rng.integers(0, 4, size=int(lens.sum())).astype(np.int64)  # many ties
    qkvu = synth.bf16_round(rng.standard_normal((int(lens.sum()), 4 * d)).astype(np.float32) * 0.4)
    g = _run(lens, ts, qkvu, d, H, torch.bfloat16, torch.float32)
    assert_close_rms(g, oracle.hstu_attention(qkvu, lens, ts, H), TOL_BF16, "edge users")


def test_normaliser_override():
    d, H = 128, 2
    lens, ts, qkvu = _random_case(5, 4, d)
    norm = lens.sum(1).astype(np.float32) * np.array([1.0, 2.0, 0.5, 3.0], np.float32)
    g = _run(lens, ts, qkvu, d, H, torch.bfloat16, torch.float32, norm=norm)
    assert_close_rms(g, oracle.hstu_attention(qkvu, lens, ts, H, norm=norm), TOL_BF16, "norm override")


@pytest.fixture(scope="module")
def attn_workload():
    return synth.make_workload(1)


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_full_attention_workload_sampled_users(attn_workload, out_dtype):
    w = attn_workload
    d, H = w["d"], w["H"]
    g = _run(w["lens"], w["ts"], w["qkvu"], d, H, torch.bfloat16, out_dtype)
    users = sample_users(w["lens"], k=4)
    rows = user_rows(w["lens"], users)
    sub_lens = w["lens"][users]
    ref = oracle.hstu_attention(w["qkvu"][rows], sub_lens, w["ts"][rows], H)
    if out_dtype == torch.float32:
        assert_close_rms(g[rows], ref, TOL_BF16, "full attention workload")
    else:
        assert_close_bf16_out(g[rows], ref, "full attention workload, bf16 out")
    assert np.isfinite(g).all()
