"""GPU parity of candidate-incremental scoring: one user's context (U, S, R)
run once with every layer's Q|K|V|U cached, then candidates scored in chunks
over the cached keys. The candidates' outputs must equal their rows of the
aggregated pass over [U, S, R, all candidates] (same normaliser N) and the
oracle's; the context rows must equal the aggregated pass's bit for bit
(a context token never sees a candidate: fun-rec 7.3.4, mask rules 1-3)."""

import numpy as np
import pytest
import torch

import oracle
import synth
from _util import TOL_BF16, assert_close_rms, to_host

pytestmark = pytest.mark.gpu

mt = pytest.importorskip("generative_recommendation_ranking_b200")

# candidate rows differ from the aggregated pass only by where each
# candidate's own key term enters the P V sum (its k-tile and column move
# with the chunk), i.e. by rounding order
TOL_REORDER = 2e-3


def _user(n_s, K, L=2, seed=0):
    """The one-user candidate workload (N_U=24, R=64, d=512, 8 heads) with
    S = n_s, K candidates and an L-layer bf16 stack."""
    w = synth.make_workload(4, seed=seed, k_override=K)
    rng = np.random.default_rng(1000 + seed)
    lens = np.array([[24, n_s, 64, K]], dtype=np.int64)
    ts = synth.make_timestamps(lens, rng)
    x = synth.make_tokens(lens, w["d"], rng)
    layers = synth.make_stack_params(L, w["d"], w["d_ff"], rng)
    return dict(lens=lens, ts=ts, x=x, layers=layers, H=w["H"], d=w["d"])


def _aggregated(u):
    dev = torch.device("cuda")
    b = mt.PackedBatch(u["lens"], u["ts"])
    ws = [mt.BlockWeights(p, u["H"]) for p in u["layers"]]
    y = mt.hstu_stack_forward(ws, b, torch.from_numpy(u["x"]).to(dev))
    b.check()
    return to_host(y)


def _incremental(u, chunks, dirty=True):
    dev = torch.device("cuda")
    n_u, n_s, n_r, K = (int(v) for v in u["lens"][0])
    assert sum(chunks) == K
    n_ctx = n_u + n_s + n_r
    ws = [mt.BlockWeights(p, u["H"]) for p in u["layers"]]
    x = torch.from_numpy(u["x"]).to(dev)
    cc = mt.ContextCache(ws, n_u, n_s, n_r, u["ts"][:n_ctx], x[:n_ctx], K, max(chunks))
    outs, c0 = [], 0
    for k in chunks:
        sl = slice(n_ctx + c0, n_ctx + c0 + k)
        if dirty:  # NaN bit patterns: nothing may read stale workspace
            batch = cc.candidate_batch(u["ts"][sl])
            scratch = cc.workspace(k).fill_(0xFF)
            outs.append(to_host(cc.score(None, x[sl], ws=scratch, batch=batch)))
            batch.check()
        else:      # the one-call form
            outs.append(to_host(cc.score(u["ts"][sl], x[sl])))
        c0 += k
    return to_host(cc.out), np.concatenate(outs)


@pytest.mark.parametrize("n_s,K,chunks", [
    (1000, 64, [40, 24]),        # candidates start mid q-tile 8; chunks inside one tile
    (1100, 300, [130, 170]),     # candidates start in odd q-tile 9; chunks span tiles
    (1000, 8, [1, 1, 6]),        # single-candidate chunks
    (232, 512, [256, 256]),      # context of 2.5 tiles, chunks of two full tiles
])
def test_incremental_matches_aggregated_and_oracle(n_s, K, chunks):
    u = _user(n_s, K)
    n_ctx = 24 + n_s + 64
    ya = _aggregated(u)
    yc, yk = _incremental(u, chunks)
    np.testing.assert_array_equal(yc, ya[:n_ctx])
    assert_close_rms(yk, ya[n_ctx:], TOL_REORDER, f"incremental vs aggregated, chunks {chunks}")
    ref = oracle.hstu_stack(u["x"], u["lens"], u["ts"], u["layers"], u["H"])
    assert_close_rms(yk, ref[n_ctx:], TOL_BF16, f"incremental vs oracle, chunks {chunks}")


def test_one_chunk_equals_aggregated_bit_exact():
    # a single chunk of all K candidates puts every row, key and tile where
    # the aggregated pass has it: same arithmetic in the same order
    u = _user(1000, 64, L=3, seed=5)
    ya = _aggregated(u)
    yc, yk = _incremental(u, [64], dirty=False)
    np.testing.assert_array_equal(yc, ya[:24 + 1000 + 64])
    np.testing.assert_array_equal(yk, ya[24 + 1000 + 64:])


def test_chunk_bounds_and_batch_shape_rejected():
    u = _user(300, 16)
    dev = torch.device("cuda")
    ws = [mt.BlockWeights(p, u["H"]) for p in u["layers"]]
    x = torch.from_numpy(u["x"]).to(dev)
    cc = mt.ContextCache(ws, 24, 300, 64, u["ts"][:388], x[:388], 16, 8)
    with pytest.raises(ValueError):
        cc.candidate_batch(u["ts"][388:388 + 9])
    # rows [row0, T) must belong to one user
    two = mt.PackedBatch(np.array([[24, 300, 64, 8], [24, 300, 64, 8]]),
                         np.concatenate([u["ts"][:396], u["ts"][:396]]))
    out = torch.empty(8, u["d"], device=dev)
    big = torch.empty(2, 792, 4 * u["d"], dtype=torch.float16, device=dev)
    with pytest.raises(mt.MTGRError) as e:
        mt.mtgr_stack_fwd_rows([l.c for l in ws], two.c, 784, big, 792, x[:8], out,
                               cc.workspace(8))
    assert e.value.status == mt._lib.MTGR_ERR_UNSUPPORTED
    # a cache shorter than the batch
    b = cc.candidate_batch(u["ts"][388:396])
    with pytest.raises(mt.MTGRError) as e:
        mt.mtgr_stack_fwd_rows([l.c for l in ws], b.c, 388, cc.cache, 390, x[388:396], out,
                               cc.workspace(8))
    assert e.value.status == mt._lib.MTGR_ERR_INVALID_ARG


def _restricted_want(lens, m, ref, q_first):
    """The oracle's q-tile pairs (in work order) cut to the q-tiles holding a
    row at or after q_first[b]; a pair whose first q-tile ends before it
    keeps only the second."""
    seg_off, _, _ = oracle.pack_offsets(lens)
    order, desc, rp, ent = ref["order"], ref["qtile_desc"], ref["row_ptr"], ref["entries"]
    want, i = [], 0
    while i < len(order):
        qa = order[i]
        b, qt = (int(v) for v in desc[qa])
        two = i + 1 < len(order) and desc[order[i + 1]][0] == b and qt % 2 == 0
        qs = [qa, order[i + 1]] if two else [qa]
        i += len(qs)
        so = seg_off[4 * b:4 * b + 5].astype(np.int64)
        n = int(so[4] - so[0])
        keep = [q for q in qs if (int(desc[q][1]) + 1) * 128 > q_first[b] and n > q_first[b]]
        if not keep:
            continue
        ks = set()
        for q in keep:
            ks |= set((ent[rp[q]:rp[q + 1]] >> 1).tolist())
        qa2 = keep[0]
        qb2 = keep[1] if len(keep) == 2 else None
        want.append([so[0], n, so[1] - so[0], so[2] - so[0], so[3] - so[0], int(desc[qa2][1]), b,
                     len(keep), rp[qa2], rp[qa2 + 1], rp[qb2] if qb2 is not None else rp[qa2 + 1],
                     rp[qb2 + 1] if qb2 is not None else rp[qa2 + 1], len(ks), 0])
    return want


@pytest.mark.parametrize("seed", [0, 1])
def test_restricted_work_list(seed):
    rng = np.random.default_rng(seed)
    B = 9
    lens = np.stack([np.full(B, 24), rng.integers(0, 1200, B), rng.integers(0, 100, B),
                     rng.integers(0, 300, B)], axis=1).astype(np.int64)
    lens[0] = [24, 1000, 64, 0]  # nothing at or after q_first
    lens[1] = [0, 0, 0, 0]       # empty user
    ts = synth.make_timestamps(lens, rng)
    n = lens.sum(1)
    q_first = np.minimum(lens[:, :3].sum(1), n).astype(np.int32)
    q_first[2] = 0                # every tile of user 2
    b = mt.PackedBatch(lens, ts)
    b.check()
    mt.mtgr_restrict_work(b.c, torch.from_numpy(q_first).cuda())
    b.check()
    m = b.meta()
    want = _restricted_want(lens, m, oracle.mask_meta(lens, ts), q_first)
    assert m["P"] == len(want)
    for got, exp in zip(m["work"], want):
        np.testing.assert_array_equal(got[:14], exp)
        assert int(got[14]) | (int(got[15]) << 32) == int(m["rt_off"][exp[6]])


# ---- batched: the contexts of many users cached, candidates scored in one call


def _batched(lens, ts, x, ws, scramble=True):
    """Context pass with the candidate rows scrambled (features 0, times 0),
    then the candidate pass with the real ones."""
    _, _, gid = oracle.pack_offsets(lens)
    cand = gid == 3
    x0, ts0 = x.copy(), ts.copy()
    if scramble:
        x0[cand] = 0.0
        ts0[cand] = 0
    cc = mt.BatchContextCache(ws, lens, ts0, torch.from_numpy(x0).cuda())
    batch = cc.candidate_batch(ts)
    scratch = cc.workspace().fill_(0xFF)  # NaN bit patterns: nothing may read stale workspace
    yk = cc.score(None, torch.from_numpy(np.ascontiguousarray(x[cand])).cuda(), ws=scratch, batch=batch)
    batch.check()
    return to_host(cc.out), to_host(yk), cand


@pytest.mark.parametrize("variant", [0, 2])
def test_batched_candidate_pass_bit_exact_against_aggregated(variant):
    rng = np.random.default_rng(3)
    lens = np.array([[24, 300, 50, 70], [24, 10, 0, 1], [0, 0, 0, 0], [3, 129, 0, 0],
                     [24, 1000, 100, 256], [1, 1, 1, 130], [24, 230, 30, 0]], np.int32)
    d, H = 512, 8
    ts = synth.make_timestamps(lens, rng)
    x = synth.make_tokens(lens, d, rng)
    layers = synth.make_stack_params(2, d, 2048, rng)
    ws = [mt.BlockWeights(p, H, variant=variant) for p in layers]
    b = mt.PackedBatch(lens, ts)
    ya = to_host(mt.hstu_stack_forward(ws, b, torch.from_numpy(x).cuda()))
    b.check()
    yc, yk, cand = _batched(lens, ts, x, ws)
    np.testing.assert_array_equal(yc[~cand], ya[~cand])
    np.testing.assert_array_equal(yk, ya[cand])
    ref = oracle.hstu_stack(x, lens, ts, layers, H, variant=variant)
    assert_close_rms(yk, ref[cand], TOL_BF16, "batched candidates vs oracle")


def test_batched_candidate_pass_block_workload():
    # the 512-user block workload: every candidate row bit-exact against the
    # aggregated pass, sampled users against the oracle
    w = synth.make_workload(2)
    ws = [mt.BlockWeights(p, w["H"]) for p in w["layers"]]
    b = mt.PackedBatch(w["lens"], w["ts"])
    ya = to_host(mt.hstu_stack_forward(ws, b, torch.from_numpy(w["x"]).cuda()))
    b.check()
    yc, yk, cand = _batched(w["lens"], w["ts"], w["x"], ws)
    np.testing.assert_array_equal(yk, ya[cand])
    np.testing.assert_array_equal(yc[~cand], ya[~cand])


def test_batched_candidate_pass_refuses_pooled_gln():
    rng = np.random.default_rng(4)
    lens = np.array([[24, 100, 20, 10], [24, 50, 5, 3]], np.int32)
    ts = synth.make_timestamps(lens, rng)
    x = synth.make_tokens(lens, 512, rng)
    layers = synth.make_stack_params(1, 512, 2048, rng)
    ws = [mt.BlockWeights(p, 8, variant=mt.MTGR_VARIANT_POOLED_GLN) for p in layers]
    cc = mt.BatchContextCache(ws, lens, ts, torch.from_numpy(x).cuda())  # the context pass runs
    _, _, gid = oracle.pack_offsets(lens)
    with pytest.raises(mt.MTGRError) as e:
        cc.score(ts, torch.from_numpy(np.ascontiguousarray(x[gid == 3])).cuda())
    assert e.value.status == mt._lib.MTGR_ERR_UNSUPPORTED
