"""Failure handling on the GPU, without faulting it.

* The bounded waits: a self-test kernel shaped like the library's tensor-core
  kernels waits on barriers that nothing completes, under a 1 ms limit; every
  role must give up, record MTGR_ERR_TIMEOUT, free the tensor memory and
  return, and the next launches must run normally.
* Ranges of the 16-bit intermediates: inputs whose Q|K|V|U projection or whose
  silu weights leave the f16 range are reported (MTGR_ERR_RANGE), and inputs
  that stay inside it match the oracle; the library never hands back a silent
  NaN with an ok status.
"""

import numpy as np
import pytest
import torch

import oracle
import synth
from _util import TOL_BF16, assert_close_rms, to_host

pytestmark = pytest.mark.gpu

mt = pytest.importorskip("generative_recommendation_ranking_b200")
from generative_recommendation_ranking_b200 import _lib  # noqa: E402


def _small_block(seed=3, B=6):
    return synth.make_workload(2, seed=seed, B=B)


def _run_block(w, layers=None):
    dev = torch.device("cuda")
    layers = w["layers"] if layers is None else layers
    b = mt.PackedBatch(w["lens"], w["ts"])
    ws = [mt.BlockWeights(p, w["H"], dtype="bf16") for p in layers]
    y = mt.hstu_stack_forward(ws, b, torch.from_numpy(w["x"]).to(dev))
    torch.cuda.synchronize()
    return to_host(y), int(b.status.item())


def test_bounded_wait_runs_out_and_the_device_stays_usable():
    dev = torch.device("cuda")
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    for _ in range(2):  # twice: the first wind-down freed everything it held
        st.zero_()
        _lib.mtgr_selftest_bounded_wait(1_000_000, st)
        torch.cuda.synchronize()
        assert int(st.item()) == _lib.MTGR_ERR_TIMEOUT
    # the next normal launches (tensor-memory allocation included) still run and match
    w = _small_block()
    y, status = _run_block(w)
    assert status == 0
    ref = oracle.hstu_stack(w["x"], w["lens"], w["ts"], w["layers"], w["H"])
    assert_close_rms(y, ref, TOL_BF16, "block after the bounded-wait self-test")


def test_bounded_wait_limits_are_checked_on_the_host():
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for bad in (0, 999, 2_000_000_000):
        with pytest.raises(_lib.MTGRError):
            _lib.mtgr_selftest_bounded_wait(bad, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0


def _scaled(w, c):
    # GroupLN_1's gamma and beta scaled by c: Q, K, V and U scale by c, the
    # scores by c^2
    layers = []
    for p in w["layers"]:
        q = dict(p)
        q["gln1_gamma"] = np.asarray(p["gln1_gamma"], np.float32) * c
        q["gln1_beta"] = np.asarray(p["gln1_beta"], np.float32) * c
        layers.append(q)
    return layers


@pytest.mark.parametrize("c", [1.0, 16.0])
def test_large_scores_inside_the_f16_range_match_the_oracle(c):
    # c = 16: scores up to ~1e4 (h = s/2 accumulates in fp32, P = silu(s) in f16)
    w = _small_block()
    layers = _scaled(w, c)
    y, status = _run_block(w, layers)
    assert status == 0
    assert np.isfinite(y).all()
    ref = oracle.hstu_stack(w["x"], w["lens"], w["ts"], layers, w["H"])
    assert_close_rms(y, ref, TOL_BF16, f"block with GroupLN_1 scaled by {c}")


@pytest.mark.parametrize("c", [256.0, 30000.0])
def test_values_beyond_the_f16_range_are_reported(c):
    # c = 256: silu weights far above 65504 (the attention's P overflows);
    # c = 30000: the Q|K|V|U projection itself leaves the f16 range
    w = _small_block()
    y, status = _run_block(w, _scaled(w, c))
    assert status == _lib.MTGR_ERR_RANGE, status
