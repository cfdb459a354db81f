#!/usr/bin/env python
"""Benchmark of the MTGR HSTU-block forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 2] [--impl ours|reference]

One step = one pass of the whole hot path over one batch: jagged packing, mask
metadata, then the HSTU block (or stack) forward — GroupLN, Q|K|V|U
projection, masked SiLU attention with gate, GroupLN, MLP with residual —
through the C ABI (libmtgr.so). Default workload: the full HSTU block at
d_model 512, 8 heads x 64, MLP 512->2048->512, bf16, 512 users per GPU.

N > 1 runs one process per GPU (torchrun): users are independent, so each rank
processes its own batch of users with replicated weights and no collective in
the data path (weak scaling); only the timing is reduced (max over ranks).

Rank 0 prints one JSON line. `--impl reference` times the CPU oracle instead
(the reference arm: a plain float64 implementation of the same step).
"""

from __future__ import annotations

import os
import sys

_CORES = len(os.sched_getaffinity(0))
for _v in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
    os.environ.setdefault(_v, str(_CORES))

import argparse  # noqa: E402
import datetime  # noqa: E402
import hashlib  # noqa: E402
import json  # noqa: E402
import statistics  # noqa: E402
import subprocess  # noqa: E402
import time  # noqa: E402

import numpy as np  # noqa: E402
import torch  # noqa: E402

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "HSTU-block fwd user-samples/s & masked-attn TFLOP/s (% of B200 BF16 peak)"
UNIT = "user-samples/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=2, help="workload index (0-3)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="CPU-baseline sample budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------- clocks ------
class ClockSampler:
    """nvidia-smi samples of this GPU's SM clock and throttle reasons."""

    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: torch.device):
        self.proc = None
        self.lines = []
        try:
            self.uuid = str(torch.cuda.get_device_properties(device).uuid).lower().replace("gpu-", "")
        except Exception:
            self.uuid = ""

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            if self.uuid and self.uuid not in f[0].lower():
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------- distributed -------
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int, device) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------- CPU oracle --------
def oracle_users_per_s(wl: dict, budget_s: float, min_users: int = 1) -> dict:
    """Time the CPU oracle on the first n users of the workload (n sized to the budget)."""
    import oracle
    from threadpoolctl import threadpool_info

    def run(n):
        rows = np.arange(int(wl["lens"][:n].sum()))
        t0 = time.perf_counter()
        if wl["kind"] == "attention":
            oracle.hstu_attention(wl["qkvu"][rows], wl["lens"][:n], wl["ts"][rows], wl["H"])
        else:
            oracle.hstu_stack(wl["x"][rows], wl["lens"][:n], wl["ts"][rows], wl["layers"], wl["H"])
        return time.perf_counter() - t0

    t1 = run(1)
    n = int(max(min_users, min(wl["lens"].shape[0], budget_s / max(t1, 1e-6))))
    dt = run(n)
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    return {"users": n, "seconds": dt, "value": n / dt, "threads": threads}


def run_reference(args, world, rank):
    """The reference arm: the CPU oracle timed on bounded samples of the workload."""
    if rank != 0:
        return
    wl = synth.make_workload(args.config, seed=args.seed)
    per_step = max(0.5, 150.0 / max(1, args.steps + args.warmup))
    import oracle  # noqa: F401
    for _ in range(args.warmup):
        oracle_users_per_s(wl, per_step)
    vals, users = [], []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        r = oracle_users_per_s(wl, per_step)
        vals.append(r["seconds"])
        users.append(r["users"])
        threads = r["threads"]
    total = time.perf_counter() - t0
    value = sum(users) / sum(vals)
    sample = f"first {min(users)}-{max(users)} users of {wl['name']} per step, float64 NumPy"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(wl, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(wl: dict, n_gpus: int) -> dict:
    t = int(wl["lens"].sum())
    return {"workload": wl["name"], "users_per_gpu": int(wl["lens"].shape[0]),
            "tokens_per_gpu": t, "d_model": wl["d"], "heads": wl["H"], "d_ff": wl["d_ff"],
            "layers": wl["L"], "parallelism": f"dp{n_gpus} (users sharded, weights replicated)",
            "l2": "inputs larger than L2 (fp32 token features %.2f GB per GPU)" % (t * wl["d"] * 4 / 1e9)}


# ------------------------------------------------------------ our arm --------
def src_sha(name: str) -> str:
    p = os.path.join(ROOT, "generative_recommendation_ranking_b200", "csrc", name)
    with open(p, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


KERNEL_SRC = {"attention": "attn_tc.cu", "gemm_qkvu": "gemm_tc.cu", "gemm_mlp1": "gemm_tc.cu",
              "gemm_mlp2": "gemm_tc.cu", "gln": "gln.cu", "pack": "pack_meta.cu",
              "mask_meta": "pack_meta.cu"}


def ncu_traffic(cls: str):
    """Per-launch DRAM bytes of a kernel class from the committed ncu summary,
    or None when absent or when the kernel source changed since the capture."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(cls)
    if not e or e.get("src_sha") != src_sha(KERNEL_SRC[cls]):
        return None
    return e.get("bytes_per_launch")


def run_ours(args, world, rank, local):
    import generative_recommendation_ranking_b200 as mt
    from generative_recommendation_ranking_b200 import _lib

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = synth.make_workload(args.config, seed=args.seed + rank)
    if wl["kind"] not in ("block", "stack"):
        raise SystemExit("bench.py times the block/stack workloads (configs 0, 2, 3)")
    B, T, d, H, dff, L = (int(wl["lens"].shape[0]), int(wl["lens"].sum()), wl["d"], wl["H"],
                          wl["d_ff"], wl["L"])
    stream = torch.cuda.current_stream(dev)

    # inputs resident in HBM
    x = torch.from_numpy(wl["x"]).to(dev)
    batch = mt.PackedBatch(wl["lens"], wl["ts"], device=dev)
    layers = [mt.BlockWeights(p, H, dtype=wl["dtype"], device=dev) for p in wl["layers"]]
    ws = mt.stack_workspace(layers, batch)
    out = torch.empty_like(x)
    batch.check()

    def step(lens_d, ts_d, x_d, out_d):
        batch.pack(stream, d_lens=lens_d)
        batch.build_meta(stream, d_ts=ts_d)
        _lib.mtgr_stack_fwd([l.c for l in layers], batch.c, x_d, out_d, ws, stream)

    for _ in range(args.warmup):
        step(batch.d_lens, batch.d_ts, x, out)
    batch.check()

    timer = _lib.Timer()
    clocks = ClockSampler(dev)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize(dev)
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    timer.attach()
    t_start.record(stream)
    for _ in range(args.steps):
        step(batch.d_lens, batch.d_ts, x, out)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    timer.detach()
    barrier(world)
    clk = clocks.stop()
    ms = t_start.elapsed_time(t_end)
    ms_max = max_over_ranks(ms, world, dev)
    batch.check()
    per_class = timer.read()
    Q, E, V = (int(v) for v in batch.counts.cpu())

    # e2e: host (pinned) inputs -> device -> step -> host output, through the C ABI
    e2e = None
    if not args.no_e2e:
        hx = torch.from_numpy(wl["x"]).pin_memory()
        hl = torch.from_numpy(np.ascontiguousarray(wl["lens"])).pin_memory()
        ht = torch.from_numpy(np.ascontiguousarray(wl["ts"])).pin_memory()
        hout = torch.empty(T, d, dtype=torch.float32).pin_memory()
        dx, dl, dts = torch.empty_like(x), torch.empty_like(batch.d_lens), torch.empty_like(batch.d_ts)
        h2d = hx.numel() * 4 + hl.numel() * 4 + ht.numel() * 8
        d2h = hout.numel() * 4

        def e2e_step():
            dx.copy_(hx, non_blocking=True)
            dl.copy_(hl, non_blocking=True)
            dts.copy_(ht, non_blocking=True)
            step(dl, dts, dx, out)
            hout.copy_(out, non_blocking=True)

        for _ in range(2):
            e2e_step()
        barrier(world)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ems = max_over_ranks(e0.elapsed_time(e1), world, dev)
        batch.check()
        assert torch.equal(hout, out.cpu()), "e2e output mismatch"
        e2e = {"value": B * world * args.e2e_steps / (ems / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": ems / args.e2e_steps}

    if rank != 0:
        return
    peaks, peak_src = load_peaks()
    # algorithmic work per launch of each class
    work = {
        "gemm_qkvu": ("tensor", 2.0 * T * 4 * d * d),
        "attention": ("tensor", 4.0 * d * V),
        "gemm_mlp1": ("tensor", 2.0 * T * dff * d),
        "gemm_mlp2": ("tensor", 2.0 * T * d * dff),
        # GroupLN_1 reads f32 and writes bf16 (6d bytes/token); GroupLN_2 reads and
        # writes bf16 (4d bytes/token): 5d bytes/token per launch on average
        "gln": ("hbm", 5.0 * d * T),
    }
    kernels = {}
    for cls, (bound, w) in work.items():
        t_ms, n = per_class[cls]
        if n == 0:
            continue
        avg_ms = t_ms / n
        if bound == "tensor":
            ach = w / (avg_ms * 1e-3) / 1e12
            kernels[cls] = {"bound": "tensor", "achieved": ach, "unit": "TFLOP/s",
                            "peak": peaks["bf16_tflops_sustained"], "avg_ms": avg_ms, "launches": n,
                            "share": t_ms / ms}
        else:
            ach = w / (avg_ms * 1e-3) / 1e9
            kernels[cls] = {"bound": "hbm", "achieved": ach, "unit": "GB/s", "peak": peaks["hbm_gbs"],
                            "avg_ms": avg_ms, "launches": n, "share": t_ms / ms}
        kernels[cls]["frac"] = kernels[cls]["achieved"] / kernels[cls]["peak"]
    for cls in ("pack", "mask_meta"):
        t_ms, n = per_class[cls]
        if n:
            kernels[cls] = {"avg_ms_per_call": t_ms / args.steps, "launches": n, "share": t_ms / ms}
    dom = max((c for c in work if c in kernels), key=lambda c: kernels[c]["share"])
    k = kernels[dom]
    traffic = ncu_traffic(dom)
    roofline = {"bound": k["bound"], "achieved": k["achieved"], "peak": k["peak"], "unit": k["unit"],
                "frac": k["frac"], "traffic": traffic, "kernel": dom,
                "peak_source": f"{peak_src} ({'bf16_tflops_sustained' if k['bound'] == 'tensor' else 'hbm_gbs'})"}
    att = kernels.get("attention", {})
    value = B * world * args.steps / (ms_max / 1e3)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        r = oracle_users_per_s(wl, args.cpu_seconds)
        cpu = {"value": r["value"], "unit": UNIT, "cores": r["threads"], "kind": "oracle",
               "sample": f"first {r['users']} users of {wl['name']} (seed {args.seed}), "
                         f"float64 NumPy, {r['seconds']:.1f} s"}
    launches = int(sum(n for _, n in per_class.values()))
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(wl, world),
        "masked_attn": {"tflops": att.get("achieved"),
                        "frac_of_bf16_peak": att.get("frac"),
                        "visible_pairs_per_gpu": V, "q_tiles": Q, "tile_entries": E},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clk,
        "gpu_launches": launches, "kernels": kernels,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    world, rank, local = dist_setup(args) if args.impl == "ours" else (
        int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if args.impl == "ours" and world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
