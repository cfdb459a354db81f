"""GPU parity of the token MLPs and the CTR/CTCVR heads against the oracle
(blog posts, "Converting heterogeneous features into tokens"; summary page,
Method; fun-rec 7.3.3): U rows bit-exact, MLP rows within the bf16 tolerance,
on small ragged batches, the 512-user block workload (sampled users) and the
whole pipeline tokens -> stack -> heads."""

import numpy as np
import pytest
import torch

import oracle
import synth
from _util import TOL_BF16, assert_close_rms, sample_users, to_host, user_rows

pytestmark = pytest.mark.gpu

mt = pytest.importorskip("generative_recommendation_ranking_b200")


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda().to(torch.bfloat16)


def _domain_rows(lens, users):
    """Rows of each domain input that belong to the given users."""
    lens = np.asarray(lens, np.int64)
    out = []
    for g in range(4):
        off = np.concatenate([[0], np.cumsum(lens[:, g])])
        out.append(np.concatenate([np.arange(off[u], off[u + 1]) for u in users])
                   if len(users) else np.zeros(0, np.int64))
    return out


def _tokenize_gpu(lens, e, p, ts=None):
    rng = np.random.default_rng(0)
    ts = synth.make_timestamps(lens, rng) if ts is None else ts
    b = mt.PackedBatch(lens, ts)
    x = mt.tokenize(mt.TokenMLPs(p), b, [_dev(a) for a in e])
    b.check()
    return b, x


@pytest.mark.parametrize("seed", [0, 1])
def test_tokenize_small_ragged_batches(seed):
    rng = np.random.default_rng(seed)
    lens = np.array([[24, 300, 50, 70], [24, 0, 0, 1], [0, 0, 0, 0], [3, 129, 0, 0],
                     [24, 1000, 100, 256], [1, 1, 1, 1]], np.int32)
    d = 512
    e = synth.make_token_inputs(lens, d, rng)
    p = synth.make_token_params(d, rng)
    b, x = _tokenize_gpu(lens, e, p)
    x = to_host(x)
    ref = oracle.tokenize(lens, e, p)
    _, _, gid = oracle.pack_offsets(lens)
    np.testing.assert_array_equal(x[gid == 0], ref[gid == 0])
    for g in (1, 2, 3):
        assert_close_rms(x[gid == g], ref[gid == g], TOL_BF16, f"domain {g}")


def test_tokenize_block_workload_sampled_users():
    w = synth.make_workload(2)
    rng = np.random.default_rng(7)
    e = synth.make_token_inputs(w["lens"], w["d"], rng)
    p = synth.make_token_params(w["d"], rng)
    _, x = _tokenize_gpu(w["lens"], e, p, ts=w["ts"])
    x = to_host(x)
    users = sample_users(w["lens"], k=3)
    rows = user_rows(w["lens"], users)
    dr = _domain_rows(w["lens"], users)
    ref = oracle.tokenize(w["lens"][users], [e[g][dr[g]] for g in range(4)], p)
    assert_close_rms(x[rows], ref, TOL_BF16, "tokens, 512 users")


def test_heads_match_oracle():
    rng = np.random.default_rng(3)
    lens = np.array([[24, 300, 50, 70], [24, 10, 0, 1], [0, 0, 0, 0], [3, 129, 0, 0],
                     [24, 500, 100, 256]], np.int32)
    d = 512
    T = int(lens.sum())
    x = rng.standard_normal((T, d), dtype=np.float32) * 2.0
    hp = synth.make_head_params(d, rng)
    b = mt.PackedBatch(lens, synth.make_timestamps(lens, rng))
    out = mt.candidate_heads(mt.CandidateHeads(hp), b, torch.from_numpy(x).cuda())
    b.check()
    # the heads read x in bf16: the oracle takes the same rounded rows
    ref = oracle.candidate_heads(synth.bf16_round(x), lens, hp)
    assert out.shape == (int(lens[:, 3].sum()), 2)
    assert_close_rms(to_host(out), ref, TOL_BF16, "heads")


def test_heads_block_workload_sampled_users():
    w = synth.make_workload(2)
    rng = np.random.default_rng(11)
    hp = synth.make_head_params(w["d"], rng)
    b = mt.PackedBatch(w["lens"], w["ts"])
    x = w["x"]
    out = to_host(mt.candidate_heads(mt.CandidateHeads(hp), b, torch.from_numpy(x).cuda()))
    b.check()
    users = sample_users(w["lens"], k=3)
    koff = np.concatenate([[0], np.cumsum(w["lens"][:, 3].astype(np.int64))])
    cand = np.concatenate([np.arange(koff[u], koff[u + 1]) for u in users])
    rows = user_rows(w["lens"], users)
    ref = oracle.candidate_heads(synth.bf16_round(x[rows]), w["lens"][users], hp)
    assert_close_rms(out[cand], ref, TOL_BF16, "heads, 512 users")


def test_pipeline_tokens_stack_heads():
    w = synth.make_workload(2, B=5, seed=2)
    rng = np.random.default_rng(5)
    e = synth.make_token_inputs(w["lens"], w["d"], rng)
    tp = synth.make_token_params(w["d"], rng)
    hp = synth.make_head_params(w["d"], rng)
    layers = synth.make_stack_params(2, w["d"], w["d_ff"], rng)
    b = mt.PackedBatch(w["lens"], w["ts"])
    x = mt.tokenize(mt.TokenMLPs(tp), b, [_dev(a) for a in e])
    y = mt.hstu_stack_forward([mt.BlockWeights(p, w["H"]) for p in layers], b, x)
    logits = mt.candidate_heads(mt.CandidateHeads(hp), b, y)
    b.check()
    x_ref = oracle.tokenize(w["lens"], e, tp)
    y_ref = oracle.hstu_stack(x_ref, w["lens"], w["ts"], layers, w["H"])
    ref = oracle.candidate_heads(y_ref, w["lens"], hp)
    assert_close_rms(to_host(logits), ref, 2 * TOL_BF16, "tokens -> 2 blocks -> heads")


def test_domain_count_mismatch_sets_device_status():
    # per-domain totals that sum to T but disagree with the batch: a device
    # validation error, every access still inside the given buffers
    lens = np.array([[4, 10, 2, 3], [2, 5, 1, 6]], np.int32)
    rng = np.random.default_rng(0)
    d = 512
    p = synth.make_token_params(d, rng)
    mlps = mt.TokenMLPs(p)
    b = mt.PackedBatch(lens, synth.make_timestamps(lens, rng))
    n_rows = [6, 16, 3, 8]  # true totals are 6, 15, 3, 9
    widths = (d,) + synth.TOKEN_F
    e = [torch.zeros(n_rows[g], widths[g], dtype=torch.bfloat16, device="cuda") for g in range(4)]
    x = torch.zeros(b.T, d, device="cuda")
    ws = torch.empty(mt.mtgr_tokenize_workspace_bytes(b.B, d, n_rows), dtype=torch.uint8, device="cuda")
    mt.mtgr_tokenize(b.c, d, n_rows, e, mlps.c, x, ws)
    torch.cuda.synchronize()
    assert int(b.status.item()) == mt._lib.MTGR_ERR_DEVICE_VALIDATION
    assert torch.isfinite(x).all()
