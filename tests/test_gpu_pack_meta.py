"""GPU parity of jagged packing and mask metadata: bit-exact against the oracle."""

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

mt = pytest.importorskip("generative_recommendation_ranking_b200")


def _check_batch(lens, ts):
    b = mt.PackedBatch(lens, ts)
    b.check()
    # rebuild over dirty buffers: nothing may depend on pre-cleared memory
    for t in (b.meta_ws, b.qtile_desc, b.row_ptr, b.entries, b.order, b.counts, b.seg_off,
              b.user_off, b.group_id, b.rt_cnt, b.rt_off, b.rt_mask, b.work):
        t.view(torch.uint8).fill_(0xA7)
    b.pack()
    b.build_meta()
    b.check()
    m = b.meta()
    seg_off, user_off, gid = oracle.pack_offsets(lens)
    np.testing.assert_array_equal(m["seg_off"], seg_off)
    np.testing.assert_array_equal(m["user_off"], user_off)
    np.testing.assert_array_equal(m["group_id"], gid)
    ref = oracle.mask_meta(lens, ts)
    np.testing.assert_array_equal(m["qtile_desc"], ref["qtile_desc"])
    np.testing.assert_array_equal(m["row_ptr"], ref["row_ptr"])
    np.testing.assert_array_equal(m["entries"], ref["entries"])
    np.testing.assert_array_equal(m["order"], ref["order"])
    assert m["visible_pairs"] == ref["visible_pairs"]
    _check_rank_tables(lens, ts, m)
    _check_work_list(lens, m, ref)
    return b


def _check_rank_tables(lens, ts, m):
    """Rule 2 as tables: for every query row i and every 64-column group g
    holding R keys, the table entry at cnt_i must equal the R columns of that
    group visible to i in the oracle's explicit M, the diagonal excluded."""
    _, user_off, _ = oracle.pack_offsets(lens)
    for b, (n_u, n_s, n_r, n_k) in enumerate(np.asarray(lens, np.int64)):
        s, e = int(user_off[b]), int(user_off[b + 1])
        if n_r == 0 or e == s:
            continue
        n_us, c_lo = n_u + n_s, n_u + n_s + n_r
        M = oracle.user_mask(int(n_u), int(n_s), int(n_r), int(n_k), ts[s:e]).copy()
        np.fill_diagonal(M, False)
        cnt = m["rt_cnt"][s:e].astype(np.int64)
        g0, g1 = n_us // 64, (c_lo - 1) // 64
        for g in range(g1 - g0 + 1):
            tab = m["rt_mask"][m["rt_off"][b] + g * (n_r + 1): m["rt_off"][b] + (g + 1) * (n_r + 1)]
            assert tab.shape[0] == n_r + 1
            cols = np.arange((g0 + g) * 64, (g0 + g + 1) * 64)
            in_r = (cols >= n_us) & (cols < c_lo)
            sub = M[:, np.clip(cols, 0, e - s - 1)] & in_r[None, :]
            weights = np.left_shift(np.uint64(1), np.arange(64, dtype=np.uint64))
            want = (sub.astype(np.uint64) * weights[None, :]).sum(axis=1, dtype=np.uint64)
            np.testing.assert_array_equal(tab[cnt], want)


def _check_work_list(lens, m, ref):
    """The work list restates, in work order, each user's q-tiles in pairs
    (qt 0-1, 2-3, ...) with the user offsets, both CSR ranges and the size of
    the union of the two k-tile lists."""
    seg_off, _, _ = oracle.pack_offsets(lens)
    order, desc, rp, ent = ref["order"], ref["qtile_desc"], ref["row_ptr"], ref["entries"]
    want = []
    i = 0
    while i < len(order):
        qa = order[i]
        b, qt = desc[qa]
        two = i + 1 < len(order) and desc[order[i + 1]][0] == b and qt % 2 == 0
        qb = order[i + 1] if two else None
        so = seg_off[4 * b:4 * b + 5].astype(np.int64)
        ka = set((ent[rp[qa]:rp[qa + 1]] >> 1).tolist())
        kb = set((ent[rp[qb]:rp[qb + 1]] >> 1).tolist()) if two else set()
        want.append([so[0], so[4] - so[0], so[1] - so[0], so[2] - so[0], so[3] - so[0], qt, b,
                     2 if two else 1, rp[qa], rp[qa + 1], rp[qb] if two else rp[qa + 1],
                     rp[qb + 1] if two else rp[qa + 1], len(ka | kb), 0, int(m["rt_off"][b])])
        i += 2 if two else 1
    w = m["work"]
    assert m["P"] == len(want) == w.shape[0]
    for got, exp in zip(w, want):
        np.testing.assert_array_equal(got[:14], exp[:14])
        assert int(got[14]) | (int(got[15]) << 32) == exp[14]


@pytest.mark.parametrize("idx", [0, 1, 2, 3])
def test_full_workload_metadata_bit_exact(idx):
    w = synth.make_workload(idx) if idx != 1 else None
    if w is None:  # the attention workload's features are not needed here
        rng = np.random.default_rng(0)
        lens = synth.make_lengths(synth.WORKLOADS[1], rng)
        ts = synth.make_timestamps(lens, rng)
    else:
        lens, ts = w["lens"], w["ts"]
    _check_batch(lens, ts)


@pytest.mark.parametrize("K", [1, 8, 64, 512])
def test_candidate_sweep_metadata(K):
    w = synth.make_workload(4, k_override=K)
    _check_batch(w["lens"], w["ts"])
    ex = synth.sweep_expanded(w)
    _check_batch(ex["lens"], ex["ts"])


@pytest.mark.parametrize("seed", range(6))
def test_random_ragged_batches(seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 40))
    lens = np.stack([rng.integers(0, 40, B), rng.integers(0, 400, B), rng.integers(0, 150, B),
                     rng.integers(0, 300, B)], 1).astype(np.int32)
    lens[rng.integers(0, B)] = 0  # an empty user
    T = int(lens.sum())
    ts = rng.integers(0, 50, size=T).astype(np.int64)  # dense ties
    _check_batch(lens, ts)


def test_edge_lengths():
    lens = np.array([[1, 0, 0, 0], [0, 0, 1, 0], [0, 0, 0, 1], [0, 127, 0, 1], [64, 64, 0, 0],
                     [0, 0, 128, 0], [0, 0, 0, 129], [10, 100, 17, 129], [0, 0, 0, 0]], np.int32)
    rng = np.random.default_rng(1)
    ts = rng.integers(0, 3, size=int(lens.sum())).astype(np.int64)
    _check_batch(lens, ts)


def test_empty_batch():
    b = mt.PackedBatch(np.zeros((0, 4), np.int32), np.zeros(0, np.int64))
    b.check()
    m = b.meta()
    assert m["Q"] == 0 and m["E"] == 0 and m["seg_off"].tolist() == [0]


def test_length_mismatch_sets_device_status():
    lens = np.array([[2, 3, 1, 1]], np.int32)
    dev = torch.device("cuda")
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    seg = torch.empty(5, dtype=torch.int32, device=dev)
    uo = torch.empty(2, dtype=torch.int32, device=dev)
    gid = torch.empty(9, dtype=torch.int8, device=dev)
    mt.mtgr_pack_offsets(1, torch.from_numpy(lens).to(dev), 9, seg, uo, gid, st)
    torch.cuda.synchronize()
    assert int(st.item()) == mt._lib.MTGR_ERR_DEVICE_VALIDATION
    st.zero_()
    bad = torch.tensor([[2, -1, 1, 1]], dtype=torch.int32, device=dev)
    mt.mtgr_pack_offsets(1, bad, 3, seg, uo, gid, st)
    torch.cuda.synchronize()
    assert int(st.item()) == mt._lib.MTGR_ERR_DEVICE_VALIDATION


def test_capacity_overflow_sets_device_status():
    lens = np.array([[4, 300, 8, 8]], np.int32)
    ts = np.arange(int(lens.sum()), dtype=np.int64)
    b = mt.PackedBatch(lens, ts)
    b.check()
    dev = torch.device("cuda")
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    i32 = dict(dtype=torch.int32, device=dev)
    ws = torch.empty(mt.mtgr_mask_meta_workspace_bytes(3, 3), dtype=torch.uint8, device=dev)
    i64 = dict(dtype=torch.int64, device=dev)
    # e_capacity 2 < the 9 tiles this user has
    mt.mtgr_build_mask_meta(1, b.seg_off, b.d_ts, 3, 3, 2, b.rt_cap, torch.empty(3, 2, **i32),
                            torch.empty(4, **i32), torch.empty(2, **i32), torch.empty(3, **i32),
                            torch.zeros(4, **i64), torch.empty(b.T, **i32), torch.empty(2, **i64),
                            torch.empty(max(b.rt_cap, 1), **i64),
                            torch.empty(3 * 64, dtype=torch.uint8, device=dev), ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == mt._lib.MTGR_ERR_CAPACITY
