"""GPU parity of the block variants against the oracle: GroupLN with pooled
(user, group) statistics (the practice article's 3.1 GLN pseudocode) and SiLU
on the Q|K|V|U projections (HSTU's pointwise SiLU), alone and together."""

import numpy as np
import pytest
import torch

import oracle
import synth
from _util import TOL_BF16, assert_close_bf16_out, assert_close_rms, sample_users, to_host, user_rows

pytestmark = pytest.mark.gpu

mt = pytest.importorskip("generative_recommendation_ranking_b200")

RAGGED = np.array([[24, 300, 50, 70], [24, 0, 0, 1], [0, 0, 0, 0], [3, 129, 0, 0],
                   [24, 1000, 100, 256], [1, 1, 1, 1]], np.int32)


@pytest.mark.parametrize("dt_in,dt_out", [("f32", "bf16"), ("bf16", "bf16"), ("f32", "f32")])
def test_pooled_gln_matches_oracle(dt_in, dt_out):
    rng = np.random.default_rng(0)
    lens = RAGGED
    d = 512
    x = synth.make_tokens(lens, d, rng)
    if dt_in == "bf16":
        x = synth.bf16_round(x)
    gamma = (1.0 + 0.3 * rng.standard_normal((4, d))).astype(np.float32)
    beta = (0.3 * rng.standard_normal((4, d))).astype(np.float32)
    b = mt.PackedBatch(lens, synth.make_timestamps(lens, rng))
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16}
    xd = torch.from_numpy(x).cuda().to(tdt[dt_in])
    y = mt.group_layernorm_pooled(b, xd, torch.from_numpy(gamma).cuda(), torch.from_numpy(beta).cuda(),
                                  out_dtype=tdt[dt_out])
    b.check()
    ref = oracle.group_layernorm_pooled(x, lens, gamma, beta)
    if dt_out == "bf16":
        assert_close_bf16_out(to_host(y), ref, "pooled GroupLN", tol=1e-4)
    else:
        assert_close_rms(to_host(y), ref, 1e-5, "pooled GroupLN f32")


@pytest.mark.parametrize("variant", [mt.MTGR_VARIANT_POOLED_GLN, mt.MTGR_VARIANT_SILU_QKVU,
                                     mt.MTGR_VARIANT_POOLED_GLN | mt.MTGR_VARIANT_SILU_QKVU])
def test_block_variant_matches_oracle(variant):
    w = synth.make_workload(2, B=6, seed=1)
    b = mt.PackedBatch(w["lens"], w["ts"])
    ws = [mt.BlockWeights(p, w["H"], variant=variant) for p in w["layers"]]
    y = to_host(mt.hstu_stack_forward(ws, b, torch.from_numpy(w["x"]).cuda()))
    b.check()
    ref = oracle.hstu_stack(w["x"], w["lens"], w["ts"], w["layers"], w["H"], variant=variant)
    assert_close_rms(y, ref, TOL_BF16, f"block variant {variant}")
    # the variant changes the block's update: it is not the plain block
    plain = oracle.hstu_stack(w["x"], w["lens"], w["ts"], w["layers"], w["H"]) - w["x"]
    upd = ref - w["x"]
    assert np.abs(plain - upd).max() > 0.1 * np.sqrt(np.mean(plain ** 2))


def test_block_variants_full_workload_sampled_users():
    w = synth.make_workload(2)
    v = mt.MTGR_VARIANT_POOLED_GLN | mt.MTGR_VARIANT_SILU_QKVU
    b = mt.PackedBatch(w["lens"], w["ts"])
    ws = [mt.BlockWeights(p, w["H"], variant=v) for p in w["layers"]]
    y = to_host(mt.hstu_stack_forward(ws, b, torch.from_numpy(w["x"]).cuda()))
    b.check()
    users = sample_users(w["lens"], k=2)
    rows = user_rows(w["lens"], users)
    ref = oracle.hstu_stack(w["x"][rows], w["lens"][users], w["ts"][rows], w["layers"], w["H"],
                            variant=v)
    assert_close_rms(y[rows], ref, TOL_BF16, "both variants, 512 users")


def test_pooled_variant_rejected_on_candidate_rows():
    w = synth.make_workload(4, k_override=8)
    n_ctx = int(w["lens"][0, :3].sum())
    ws = [mt.BlockWeights(p, w["H"], variant=mt.MTGR_VARIANT_POOLED_GLN) for p in w["layers"]]
    x = torch.from_numpy(w["x"]).cuda()
    cc = mt.ContextCache(ws, 24, 1000, 64, w["ts"][:n_ctx], x[:n_ctx], 8, 8)
    with pytest.raises(mt.MTGRError) as e:
        cc.score(w["ts"][n_ctx:], x[n_ctx:])
    assert e.value.status == mt._lib.MTGR_ERR_UNSUPPORTED


def _with_rab(w, seed=5):
    rng = np.random.default_rng(seed)
    layers = []
    for p in w["layers"]:
        q = dict(p)
        q["rab_pos"], q["rab_time"] = synth.make_rab_tables(w["H"], rng)
        layers.append(q)
    return layers


@pytest.mark.parametrize("variant", [mt.MTGR_VARIANT_RAB, mt.MTGR_VARIANT_RAB | mt.MTGR_VARIANT_SILU_QKVU])
def test_block_relative_attention_bias_matches_oracle(variant):
    # ragged users (a 1000-token S run, tiles off the grid, a U-only user)
    # and timestamp ties: every bucket and clip path of the bias
    rng = np.random.default_rng(2)
    lens = RAGGED
    d, H, dff = 512, 8, 2048
    ts = synth.make_timestamps(lens, rng)
    x = synth.make_tokens(lens, d, rng)
    w = dict(lens=lens, ts=ts, x=x, H=H, layers=[synth.make_block_params(d, dff, rng)])
    layers = _with_rab(w)
    b = mt.PackedBatch(lens, ts)
    ws = [mt.BlockWeights(p, H, variant=variant) for p in layers]
    y = to_host(mt.hstu_stack_forward(ws, b, torch.from_numpy(x).cuda()))
    b.check()
    ref = oracle.hstu_stack(x, lens, ts, layers, H, variant=variant)
    assert_close_rms(y, ref, TOL_BF16, f"bias variant {variant}")
    plain = oracle.hstu_stack(x, lens, ts, layers, H, variant=variant & ~mt.MTGR_VARIANT_RAB) - x
    assert np.abs(plain - (ref - x)).max() > 0.1 * np.sqrt(np.mean(plain ** 2))


def test_block_relative_attention_bias_full_workload_sampled_users():
    w = synth.make_workload(2)
    layers = _with_rab(w)
    b = mt.PackedBatch(w["lens"], w["ts"])
    ws = [mt.BlockWeights(p, w["H"], variant=mt.MTGR_VARIANT_RAB) for p in layers]
    y = to_host(mt.hstu_stack_forward(ws, b, torch.from_numpy(w["x"]).cuda()))
    b.check()
    users = sample_users(w["lens"], k=2)
    rows = user_rows(w["lens"], users)
    ref = oracle.hstu_stack(w["x"][rows], w["lens"][users], w["ts"][rows], layers, w["H"],
                            variant=mt.MTGR_VARIANT_RAB)
    assert_close_rms(y[rows], ref, TOL_BF16, "bias variant, 512 users")


def test_relative_attention_bias_needs_its_tables():
    w = synth.make_workload(2, B=2)
    b = mt.PackedBatch(w["lens"], w["ts"])
    ws = [mt.BlockWeights(p, w["H"], variant=mt.MTGR_VARIANT_RAB) for p in w["layers"]]
    with pytest.raises(mt.MTGRError) as e:
        mt.hstu_stack_forward(ws, b, torch.from_numpy(w["x"]).cuda())
    assert e.value.status == mt._lib.MTGR_ERR_INVALID_ARG
