"""Host logic of bench.py on the CPU: the ncu traffic record is used only
while the kernel source matches the capture, the peaks come from the measured
file (else the fallback), the workload description, and the default flags."""

import hashlib
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


def _fake_root(tmp_path, src_text, recorded_sha):
    csrc = tmp_path / "generative_recommendation_ranking_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "attn_tc.cu").write_text(src_text)
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps(
        {"attention": {"bytes_per_launch": 12345, "src_sha": recorded_sha,
                       "workload": "block_bf16_b512_d512", "users": 512}}))
    return str(tmp_path)


def test_traffic_only_while_the_source_matches(tmp_path, monkeypatch):
    text = "// kernel source\n"
    sha = hashlib.sha256(text.encode()).hexdigest()[:16]
    monkeypatch.setattr(bench, "ROOT", _fake_root(tmp_path / "a", text, sha))
    assert bench.ncu_traffic("attention") == 12345
    monkeypatch.setattr(bench, "ROOT", _fake_root(tmp_path / "b", text + "// changed\n", sha))
    assert bench.ncu_traffic("attention") is None
    monkeypatch.setattr(bench, "ROOT", str(tmp_path / "missing"))
    assert bench.ncu_traffic("attention") is None


def test_traffic_only_for_the_captured_workload(tmp_path, monkeypatch):
    text = "// kernel source\n"
    sha = hashlib.sha256(text.encode()).hexdigest()[:16]
    monkeypatch.setattr(bench, "ROOT", _fake_root(tmp_path / "a", text, sha))
    assert bench.ncu_traffic("attention", "block_bf16_b512_d512") == 12345
    assert bench.ncu_traffic("attention", "attn_bf16_b256_d256") is None
    # a --users override keeps the workload's name: the user count decides
    assert bench.ncu_traffic("attention", "block_bf16_b512_d512", 512) == 12345
    assert bench.ncu_traffic("attention", "block_bf16_b512_d512", 128) is None


def test_committed_traffic_record_names_a_kernel_class_with_a_source():
    with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
        rec = json.load(f)
    for cls, e in rec.items():
        assert cls in bench.KERNEL_SRC, cls
        assert e["bytes_per_launch"] > 0 and len(e["src_sha"]) == 16 and e["users"] > 0
        assert os.path.exists(os.path.join(ROOT, "profiles", os.path.basename(e["source"])))


def test_peaks_measured_else_fallback(tmp_path, monkeypatch):
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(
        {"hbm_gbs": 7000.0, "bf16_tflops": 1700.0, "bf16_tflops_sustained": 1500.0, "other": 1}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.load_peaks()
    assert src == "measured" and peaks == {"hbm_gbs": 7000.0, "bf16_tflops": 1700.0,
                                           "bf16_tflops_sustained": 1500.0}
    monkeypatch.setattr(bench, "ROOT", str(tmp_path / "nowhere"))
    peaks, src = bench.load_peaks()
    assert src == "fallback" and peaks == bench.FALLBACK_PEAKS


def test_workload_config_describes_the_block_workload():
    wl = synth.make_workload(2)
    c = bench.workload_config(wl, 4)
    assert c["workload"] == "block_bf16_b512_d512" and c["users_per_gpu"] == 512
    assert c["tokens_per_gpu"] == int(np.asarray(wl["lens"]).sum())
    assert (c["d_model"], c["heads"], c["d_ff"], c["layers"]) == (512, 8, 2048, 1)
    assert c["parallelism"].startswith("dp4")
    assert "larger than L2" in c["l2"]


def test_small_workloads_flush_l2():
    # a workload whose inputs fit in L2 is timed with the L2 flushed between
    # steps, and its config says so; the 512-user block workload is not
    small, big = synth.make_workload(0), synth.make_workload(2)
    assert bench.needs_flush(small) and not bench.needs_flush(big)
    assert bench.input_bytes(big) == int(np.asarray(big["lens"]).sum()) * 512 * 4
    assert bench.FLUSH_BYTES > bench.L2_BYTES
    assert "flushed" in bench.workload_config(small, 1)["l2"]


def test_default_flags(monkeypatch):
    monkeypatch.setattr(sys, "argv", ["bench.py"])
    a = bench.parse_args()
    assert (a.gpus, a.config, a.impl) == (1, 2, "ours")
    assert a.warmup >= 3 and a.steps > 0
    assert not (a.pipeline or a.serving or a.no_e2e or a.no_cpu_baseline)


def test_cpu_baseline_thread_cap():
    # the oracle timing runs on the fp32 block workload and reports its
    # threads; capped at one thread it reports one
    wl = synth.make_workload(0)
    r = bench.oracle_users_per_s(wl, 0.05)
    assert r["users"] >= 1 and r["value"] > 0 and r["threads"] >= 1
    r1 = bench.oracle_users_per_s(wl, 0.05, max_threads=1)
    assert r1["threads"] == 1 and r1["value"] > 0


def test_tensor_peak_follows_the_timed_region_length():
    # a short timed region runs at the burst clock: divide by the burst peak;
    # only seconds-long regions settle at the sustained (power-capped) figure
    import bench
    assert bench.tensor_peak_key(0.09) == "bf16_tflops"
    assert bench.tensor_peak_key(bench.SUSTAINED_AFTER_S - 1e-3) == "bf16_tflops"
    assert bench.tensor_peak_key(bench.SUSTAINED_AFTER_S) == "bf16_tflops_sustained"
    assert bench.tensor_peak_key(30.0) == "bf16_tflops_sustained"


def test_expanded_rows_of_a_many_user_sweep_batch():
    # row r is user r // K's context with its candidate r % K, at the
    # aggregated user's normaliser
    import bench
    import synth
    K, B = 8, 3
    agg = synth.make_workload(4, seed=1, k_override=K, B=B)
    ex = bench.expanded_rows(agg, 11)
    n_ctx, n = 1088, 1088 + K
    assert ex["lens"].shape == (11, 4) and (ex["lens"][:, 3] == 1).all()
    assert (ex["norm"] == n).all()
    for r in (0, 7, 8, 10):
        b, c = divmod(r, K)
        row = ex["x"][r * (n_ctx + 1):(r + 1) * (n_ctx + 1)]
        np.testing.assert_array_equal(row[:n_ctx], agg["x"][b * n:b * n + n_ctx])
        np.testing.assert_array_equal(row[n_ctx], agg["x"][b * n + n_ctx + c])
        np.testing.assert_array_equal(ex["ts"][r * (n_ctx + 1) + n_ctx], agg["ts"][b * n + n_ctx + c])
