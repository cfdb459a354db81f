"""Pins of the oracle's jagged packing and canonical tile metadata."""

import numpy as np
import pytest

import oracle


def test_pack_golden(golden):
    g = golden("pack_small.txt")
    seg_off, user_off, gid = oracle.pack_offsets(np.asarray(g["lens"]))
    np.testing.assert_array_equal(seg_off, g["seg_off"])
    np.testing.assert_array_equal(user_off, g["user_off"])
    np.testing.assert_array_equal(gid, g["group_id"])


def test_pack_empty_batch():
    seg_off, user_off, gid = oracle.pack_offsets(np.zeros((0, 4), np.int32))
    assert seg_off.tolist() == [0] and user_off.tolist() == [0] and gid.size == 0


def test_mask_meta_golden(golden):
    g = golden("mask_meta_two_tiles.txt")
    n_u, n_s, n_r, n_k = g["lens"]
    ts = np.concatenate([np.zeros(n_u), np.arange(n_s), 1000 + np.arange(n_r),
                         np.full(n_k, 1500)]).astype(np.int64)
    mm = oracle.mask_meta(np.array([g["lens"]]), ts)
    np.testing.assert_array_equal(mm["qtile_desc"].reshape(-1), g["qtile_desc"])
    np.testing.assert_array_equal(mm["row_ptr"], g["row_ptr"])
    np.testing.assert_array_equal(mm["entries"], g["entries"])


def _brute_tiles(M, bm, bn):
    """Tile classification by explicit per-cell enumeration."""
    N = M.shape[0]
    out = []
    for qt in range(-(-N // bm)):
        row = []
        for kt in range(-(-N // bn)):
            any_vis, all_vis = False, True
            for i in range(qt * bm, min(N, (qt + 1) * bm)):
                for j in range(kt * bn, min(N, (kt + 1) * bn)):
                    any_vis |= bool(M[i, j])
                    all_vis &= bool(M[i, j])
            if any_vis:
                row.append((kt << 1) | (0 if all_vis else 1))
        out.append(row)
    return out


@pytest.mark.parametrize("seed", range(8))
def test_mask_meta_brute_force_small_tiles(seed):
    rng = np.random.default_rng(seed)
    B = 3
    lens = rng.integers(0, 7, size=(B, 4)).astype(np.int32)
    lens[0] = [1, 2, 5, 4]
    T = int(lens.sum())
    ts = rng.integers(0, 8, size=T).astype(np.int64)
    bm, bn = 4, 3
    mm = oracle.mask_meta(lens, ts, bm, bn)
    _, user_off, _ = oracle.pack_offsets(lens)
    rows, desc = [], []
    for b in range(B):
        s, e = user_off[b], user_off[b + 1]
        if e == s:
            continue
        M = oracle.user_mask(*(int(v) for v in lens[b]), ts[s:e])
        tiles = _brute_tiles(M, bm, bn)
        rows += tiles
        desc += [(b, qt) for qt in range(len(tiles))]
    np.testing.assert_array_equal(mm["qtile_desc"], np.asarray(desc, np.int32).reshape(-1, 2))
    flat = [e for r in rows for e in r]
    np.testing.assert_array_equal(mm["entries"], flat)
    np.testing.assert_array_equal(np.diff(mm["row_ptr"]), [len(r) for r in rows])
    # order: users by descending length (ties by index), q-tiles ascending
    order = mm["order"]
    assert sorted(order.tolist()) == list(range(len(rows)))
    n_user = lens.sum(1)
    key = [(-int(n_user[desc[q][0]]), desc[q][0], desc[q][1]) for q in order]
    assert key == sorted(key)
    assert mm["visible_pairs"] == oracle.visible_pairs(lens, ts)


def test_diagonal_tile_always_present():
    rng = np.random.default_rng(7)
    lens = np.array([[3, 300, 50, 90]], np.int32)
    ts = np.concatenate([np.zeros(3), rng.integers(0, 1000, 300), np.sort(rng.integers(1000, 2000, 50)),
                         rng.integers(1000, 2000, 90)]).astype(np.int64)
    mm = oracle.mask_meta(lens, ts)
    for q in range(mm["qtile_desc"].shape[0]):
        qt = mm["qtile_desc"][q, 1]
        kts = mm["entries"][mm["row_ptr"][q]:mm["row_ptr"][q + 1]] >> 1
        assert qt in kts
