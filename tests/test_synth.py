"""The seeded generators: determinism, shapes and value ranges of each workload."""

import numpy as np
import torch

import synth


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(0)
    a = (rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))).astype(np.float32)
    a[:4] = [0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8]  # ties
    ref = torch.from_numpy(a).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(synth.bf16_round(a), ref)


def test_workloads_deterministic_and_shaped():
    for idx in (0, 1):
        a = synth.make_workload(idx, seed=3, B=8)
        b = synth.make_workload(idx, seed=3, B=8)
        np.testing.assert_array_equal(a["lens"], b["lens"])
        np.testing.assert_array_equal(a["ts"], b["ts"])
        feats = "x" if idx == 0 else "qkvu"
        np.testing.assert_array_equal(a[feats], b[feats])
    w0 = synth.make_workload(0)
    assert w0["lens"].tolist() == [[4, 32, 8, 8]] * 4
    assert w0["x"].shape == (208, 64) and len(w0["layers"]) == 1
    assert w0["layers"][0]["w_qkvu"].shape == (256, 64)


def test_length_and_time_ranges():
    for idx, wl in synth.WORKLOADS.items():
        if idx == 4:
            continue
        rng = np.random.default_rng(1)
        lens = synth.make_lengths(wl, rng, B=2000)
        for col, spec in zip((1, 2, 3), (wl.s_len, wl.r_len, wl.k_len)):
            if spec[0] != "fixed":
                assert lens[:, col].min() >= spec[1] and lens[:, col].max() <= spec[2]
        ts = synth.make_timestamps(lens[:50], rng)
        off = np.concatenate([[0], np.cumsum(lens[:50].reshape(-1))])
        for b in range(50):
            s_ts = ts[off[4 * b + 1]:off[4 * b + 2]]
            r_ts = ts[off[4 * b + 2]:off[4 * b + 3]]
            c_ts = ts[off[4 * b + 3]:off[4 * b + 4]]
            assert (s_ts < 1000).all() and (s_ts >= 0).all()
            assert (r_ts >= 1000).all() and (np.diff(r_ts) >= 0).all()
            assert (c_ts >= 1000).all() and (c_ts < 2000).all()


def test_sweep_expanded_layout():
    w = synth.make_workload(4, k_override=8)
    ex = synth.sweep_expanded(w)
    assert ex["lens"].shape == (8, 4) and (ex["lens"][:, 3] == 1).all()
    assert ex["x"].shape[0] == 8 * 1089
    assert np.allclose(ex["norm"], 1096)
    np.testing.assert_array_equal(ex["x"][1089 + 1088], w["x"][1088 + 1])
