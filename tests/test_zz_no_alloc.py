"""mtgr_build_mask_meta_static: the mask-metadata builder for callers that
cannot allocate device memory (for example a serving process that gives all
of its device memory to its own pool at start-up and forbids later
cudaMalloc/cudaFree calls). It keeps its scratch in a fixed array inside the
library instead of a caller workspace. Its results must equal those of
mtgr_build_mask_meta, call after call, since the shared array keeps the
previous call's contents.

Kept in a file of its own that pytest collects last."""

import numpy as np
import pytest
import torch

import synth
from generative_recommendation_ranking_b200 import _lib, api


def _buffers(lens, dev):
    q_cap, kt_cap, e_cap, rt_cap = api.capacities(lens)
    B, T = int(lens.shape[0]), int(lens.sum())
    i32 = dict(dtype=torch.int32, device=dev)
    i64 = dict(dtype=torch.int64, device=dev)
    return dict(
        q_cap=q_cap, kt_cap=kt_cap, e_cap=e_cap, rt_cap=rt_cap,
        qtile_desc=torch.full((max(q_cap, 1), 2), -7, **i32),
        row_ptr=torch.full((q_cap + 1,), -7, **i32),
        entries=torch.full((max(e_cap, 1),), -7, **i32),
        order=torch.full((max(q_cap, 1),), -7, **i32),
        counts=torch.full((4,), -7, **i64),
        rt_cnt=torch.full((max(T, 1),), -7, **i32),
        rt_off=torch.full((B + 1,), -7, **i64),
        rt_mask=torch.full((max(rt_cap, 1),), -7, **i64),
        work=torch.full((max(q_cap, 1) * _lib.WORK_ITEM_BYTES,), 0xA5, dtype=torch.uint8, device=dev),
        status=torch.zeros(1, **i32))


def _results(bf):
    torch.cuda.synchronize()
    Q, E, P = int(bf["counts"][0]), int(bf["counts"][1]), int(bf["counts"][3])
    return dict(
        counts=bf["counts"].cpu().numpy(), qtile_desc=bf["qtile_desc"][:Q].cpu().numpy(),
        row_ptr=bf["row_ptr"][:Q + 1].cpu().numpy(), entries=bf["entries"][:E].cpu().numpy(),
        order=bf["order"][:Q].cpu().numpy(), rt_cnt=bf["rt_cnt"].cpu().numpy(),
        rt_off=bf["rt_off"].cpu().numpy(), rt_mask=bf["rt_mask"][:bf["rt_cap"]].cpu().numpy(),
        work=bf["work"][:P * _lib.WORK_ITEM_BYTES].cpu().numpy(),
        status=int(bf["status"].item()))


def _build(batch, lens, static, check_free=True):
    dev = batch.device
    bf = _buffers(lens, dev)
    args = (batch.B, batch.seg_off, batch.d_ts, bf["q_cap"], bf["kt_cap"], bf["e_cap"],
            bf["rt_cap"], bf["qtile_desc"], bf["row_ptr"], bf["entries"], bf["order"],
            bf["counts"], bf["rt_cnt"], bf["rt_off"], bf["rt_mask"], bf["work"])
    if static:
        # every buffer exists before the call: once the fixed array has been
        # committed (by the first call in the process, under lazy module
        # loading), the device's free memory must not move across a call
        torch.cuda.synchronize(dev)
        free0 = torch.cuda.mem_get_info(dev)[0]
        _lib.mtgr_build_mask_meta_static(*args, bf["status"])
        torch.cuda.synchronize(dev)
        if check_free:
            assert torch.cuda.mem_get_info(dev)[0] == free0, "the static builder changed free device memory"
    else:
        ws = torch.full((max(_lib.mtgr_mask_meta_workspace_bytes(bf["q_cap"], bf["kt_cap"]), 1),),
                        0x5A, dtype=torch.uint8, device=dev)
        _lib.mtgr_build_mask_meta(*args, ws, bf["status"])
    return _results(bf)


def test_static_builder_rejects_oversized_batches_on_the_host():
    # q_capacity x kt_capacity above the fixed 4 MiB scratch: a clear error, no device work
    lib = _lib.load()
    rc = lib.mtgr_build_mask_meta_static(1, None, None, 1 << 20, 8, 1, 1, None, None, None, None,
                                         None, None, None, None, None, None, None)
    assert rc == _lib.MTGR_ERR_CAPACITY
    assert _lib.STATIC_META_SCRATCH_BYTES == 4 << 20


@pytest.mark.gpu
def test_static_builder_matches_workspace_builder_on_consecutive_calls():
    # calls in a row with different shapes: no call may see anything an
    # earlier one left in the shared scratch array
    cases = []
    for idx, seed in ((3, 1), (2, 2)):
        rng = np.random.default_rng(seed)
        lens = synth.make_lengths(synth.WORKLOADS[idx], rng)
        ts = synth.make_timestamps(lens, rng)
        cases.append((lens, ts))
    rng = np.random.default_rng(9)
    lens = rng.integers(0, 300, size=(37, 4)).astype(np.int32)
    cases.append((lens, rng.integers(0, 40, size=int(lens.sum())).astype(np.int64)))
    # a first call on a larger, different batch commits the array on this
    # device (the one call allowed to change free memory) and leaves it
    # dirty, so every compared call starts from another call's tile codes,
    # never from zeros
    rng = np.random.default_rng(11)
    warm_lens = synth.make_lengths(synth.WORKLOADS[3], rng)
    warm = api.PackedBatch(warm_lens, synth.make_timestamps(warm_lens, rng))
    warm.check()
    assert _build(warm, warm_lens, static=True, check_free=False)["status"] == 0
    for lens, ts in cases:
        batch = api.PackedBatch(lens, ts)
        batch.check()
        got = _build(batch, lens, static=True)
        want = _build(batch, lens, static=False)
        assert got["status"] == 0 and want["status"] == 0
        for k in want:
            np.testing.assert_array_equal(got[k], want[k], err_msg=k)
