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
    ap.add_argument("--users", type=int, default=None,
                    help="run only the first N users of the workload (profiling a smaller case)")
    ap.add_argument("--config", type=int, default=2,
                    help="workload: 0 fp32 block, 1 attention only, 2 block (default), "
                         "3 8-layer stack, 4 candidate sweep")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="CPU-baseline sample budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--serving", action="store_true",
                    help="cached-context candidate scoring on the 512-user block workload: the "
                         "candidate pass against the aggregated pass (one JSON line)")
    ap.add_argument("--sweep-users", type=int, default=0,
                    help="with --config 4: run the candidate sweep over this many users per "
                         "launch (aggregated, cached-context and expanded legs), so that the "
                         "cost per added candidate is not launch latency")
    ap.add_argument("--backward", action="store_true",
                    help="one training step of the block on the 512-user block workload: the "
                         "forward keeping its activations, then the backward (one JSON line, "
                         "each backward kernel class with its roofline)")
    ap.add_argument("--pipeline", action="store_true",
                    help="time token MLPs -> block -> CTR/CTCVR heads on the 512-user block "
                         "workload, each part with its roofline (one JSON line)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# A tensor kernel timed inside a short region runs at the burst clock; only a
# timed region of seconds settles at the power-capped sustained clock.
SUSTAINED_AFTER_S = 2.0


def tensor_peak_key(timed_s: float) -> str:
    """Which measured bf16 peak a tensor kernel's fraction divides by: the
    burst figure for a timed region shorter than SUSTAINED_AFTER_S seconds,
    the sustained one for longer regions."""
    return "bf16_tflops_sustained" if timed_s >= SUSTAINED_AFTER_S else "bf16_tflops"


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
def oracle_users_per_s(wl: dict, budget_s: float, min_users: int = 1,
                       max_threads: int | None = None) -> dict:
    """Time the CPU oracle on the first n users of the workload (n sized to
    the budget); ``max_threads`` caps the BLAS thread pools while it runs."""
    import oracle
    from threadpoolctl import threadpool_info, threadpool_limits

    if max_threads is not None:
        with threadpool_limits(limits=max_threads):
            return oracle_users_per_s(wl, budget_s, min_users)

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
    wl = synth.make_workload(args.config, seed=args.seed, B=args.users)
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
        "data": "synthetic",
        "config": workload_config(wl, args.gpus,
                                  (args.users or synth.WORKLOADS[args.config].B) * args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def dtype_label(wl: dict) -> str:
    """The arithmetic the step computes in. bf16 blocks: bf16 GEMM operands
    with fp32 accumulation and an fp32 residual stream; the attention takes
    Q|K|V|U and its silu weights P in f16, sums Q K^T in f16 (an overflow
    sets MTGR_ERR_RANGE) and P V in fp32."""
    if wl["dtype"] == "f32":
        return "f32"
    if wl["kind"] == "attention":
        return "bf16 (attention: Q|K|V|U bf16, P and V f16, fp32 accumulate)"
    return ("bf16 (GEMMs bf16 -> fp32 accumulate; attention: Q|K|V|U f16, Q.K^T f16 accumulate "
            "(overflow reported), P f16, P.V fp32 accumulate)")


def rank_workload(args, world: int, rank: int):
    """This rank's workload and the global user count. One GPU: the workload
    itself. N GPUs: one global batch of N x B users drawn with the same seed
    on every rank (lengths and timestamps), split by length-balanced
    sharding; each rank draws the token features of its own users only, and
    the weights from one seed shared by all ranks (replicated). Per-GPU work
    stays at about B users as N grows (weak scaling)."""
    spec = synth.WORKLOADS[args.config]
    b = args.users or spec.B
    if world == 1:
        return synth.make_workload(args.config, seed=args.seed, B=args.users), b
    from generative_recommendation_ranking_b200 import shard
    rng = np.random.default_rng(args.seed)
    lens = synth.make_lengths(spec, rng, B=b * world)
    ts = synth.make_timestamps(lens, rng)
    _, _, lens_r, ts_r = shard.rank_shard(lens, ts, world, rank, spec.d, spec.d_ff)
    wl = synth.assemble_workload(args.config, lens_r, ts_r,
                                 token_rng=np.random.default_rng([args.seed, 1, rank]),
                                 weight_rng=np.random.default_rng([args.seed, 2]))
    return wl, b * world


L2_BYTES = 126 * 10**6   # the B200's L2
FLUSH_BYTES = 256 * 2**20
E2E_STREAMS = 3  # host-buffer leg: streams (and workspaces) the steps rotate over


def input_bytes(wl: dict) -> int:
    """Bytes a step reads as input: the token features (fp32) of a block
    workload, or Q|K|V|U (bf16) of an attention-only one."""
    t = int(wl["lens"].sum())
    return t * 4 * wl["d"] * 2 if wl["kind"] == "attention" else t * wl["d"] * 4


def needs_flush(wl: dict) -> bool:
    return input_bytes(wl) <= L2_BYTES


def workload_config(wl: dict, n_gpus: int, users_total: int | None = None) -> dict:
    t = int(wl["lens"].sum())
    par = ("dp1" if n_gpus == 1 else
           f"dp{n_gpus} (one global batch of {users_total} users in length-balanced user "
           "shards, weights replicated, no collective in the data path)")
    what = "Q|K|V|U bf16" if wl["kind"] == "attention" else "fp32 token features"
    gb = input_bytes(wl) / 1e9
    l2 = (f"L2 flushed between timed steps ({FLUSH_BYTES >> 20} MB written outside the timed "
          f"events; {what} {gb:.3f} GB per GPU fit in L2)" if needs_flush(wl) else
          f"inputs larger than L2 ({what} {gb:.2f} GB per GPU)")
    return {"workload": wl["name"], "users_per_gpu": int(wl["lens"].shape[0]),
            "tokens_per_gpu": t, "d_model": wl["d"], "heads": wl["H"], "d_ff": wl["d_ff"],
            "layers": wl["L"], "parallelism": par, "l2": l2}


# ------------------------------------------------------------ our arm --------
def src_sha(name: str) -> str:
    p = os.path.join(ROOT, "generative_recommendation_ranking_b200", "csrc", name)
    with open(p, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


KERNEL_SRC = {"attention": "attn_tc.cu", "gemm_qkvu": "gemm_tc.cu", "gemm_mlp1": "gemm_tc.cu",
              "gemm_mlp2": "gemm_tc.cu", "gln": "gln.cu", "pack": "pack_meta.cu",
              "mask_meta": "pack_meta.cu", "bwd_attention": "attn_bwd_tc.cu",
              "bwd_wgrad": "gemm_wgrad.cu"}


def ncu_traffic(cls: str, workload: str = None, users: int = None):
    """Per-launch DRAM bytes of a kernel class from the committed ncu summary,
    or None when absent, when the kernel source changed since the capture, or
    when the record is for another workload than `workload` or another user
    count than `users` (a --users override keeps the workload's name)."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(cls)
    if not e or e.get("src_sha") != src_sha(KERNEL_SRC[cls]):
        return None
    if workload is not None and e.get("workload") != workload:
        return None
    if users is not None and e.get("users") != users:
        return None
    return e.get("bytes_per_launch")


class Workspace:
    """Device-side state of one workload: inputs, batch metadata, weights and
    workspace; ``step`` runs one pass of the hot path through the C ABI."""

    def __init__(self, wl, dev, stream):
        import generative_recommendation_ranking_b200 as mt
        from generative_recommendation_ranking_b200 import _lib
        self.wl, self.dev, self.stream, self._lib = wl, dev, stream, _lib
        self.kind = wl["kind"]
        self.d, self.H = wl["d"], wl["H"]
        if self.kind == "attention":
            self.x = torch.from_numpy(wl["qkvu"]).to(dev).to(torch.bfloat16)
            self.out = torch.empty(int(wl["lens"].sum()), self.d, dtype=torch.float32, device=dev)
        else:
            self.x = torch.from_numpy(wl["x"]).to(dev)
            self.out = torch.empty_like(self.x)
        self.batch = mt.PackedBatch(wl["lens"], wl["ts"], device=dev, norm=wl.get("norm"))
        self.layers = [mt.BlockWeights(p, self.H, dtype=wl["dtype"], device=dev)
                       for p in wl["layers"]]
        self.ws = mt.stack_workspace(self.layers, self.batch) if self.layers else None
        self.batch.check()

    def step(self, lens_d=None, ts_d=None, x_d=None, out_d=None, stream=None):
        s = self.stream if stream is None else stream
        b = self.batch
        b.pack(s, d_lens=b.d_lens if lens_d is None else lens_d)
        b.build_meta(s, d_ts=b.d_ts if ts_d is None else ts_d)
        x_d = self.x if x_d is None else x_d
        out_d = self.out if out_d is None else out_d
        if self.kind == "attention":
            self._lib.mtgr_hstu_attention_fwd(b.c, self.d, self.H, x_d, out_d, s)
        else:
            self._lib.mtgr_stack_fwd([l.c for l in self.layers], b.c, x_d, out_d, self.ws, s)


def graph_steps_ms(fn, n: int, warmup: int) -> float:
    """Device milliseconds per replay of fn(stream) captured once into a CUDA
    graph: the launch cost of a step made of short kernels drops out."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(warmup):
            fn(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        fn(side)
    cur = torch.cuda.current_stream()
    for _ in range(warmup):
        g.replay()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cur)
    for _ in range(n):
        g.replay()
    e1.record(cur)
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) / n


def time_steps(fn, n, stream, flush=None) -> float:
    """Device milliseconds of n calls of fn on `stream` (CUDA events). With
    `flush` (a buffer larger than L2), each call is timed alone and the
    buffer is overwritten on the stream between calls, outside the events."""
    if flush is None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(n)]
    with torch.cuda.stream(stream):
        for i in range(n):
            flush.add_(1)
            ev[i][0].record(stream)
            fn()
            ev[i][1].record(stream)
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in ev)


def run_e2e(wsp: Workspace, steps: int, world: int, dev, users_total: int):
    """The same step end to end through the C ABI's host-buffer entry
    (mtgr_stack_fwd_host): every call copies the step's lengths, timestamps
    and token features from pinned host memory into the device workspace,
    packs, builds the mask metadata, runs the stack and copies the whole
    output and the status word back. Steps rotate over E2E_STREAMS streams,
    each with its own workspace and output buffer. On one stream a step's
    input copy waits for the output copy of the step before it there, so
    with three streams one step's input copy, another's kernels and a third's
    output copy run at once and both directions of the (full-duplex) PCIe
    link stay busy; two leave each direction idle while a stream turns
    around. Attention-only workloads keep the device-pointer path (the host
    entry runs the block stack)."""
    import generative_recommendation_ranking_b200 as mt
    from generative_recommendation_ranking_b200 import _lib
    wl = wsp.wl
    if wsp.kind == "attention":
        return None
    hl = torch.from_numpy(np.ascontiguousarray(wl["lens"], np.int32)).pin_memory()
    ht = torch.from_numpy(np.ascontiguousarray(wl["ts"], np.int64)).pin_memory()
    hn = (torch.from_numpy(np.ascontiguousarray(wl["norm"], np.float32)).pin_memory()
          if wl.get("norm") is not None else None)
    hx = torch.from_numpy(np.ascontiguousarray(wl["x"], np.float32)).pin_memory()
    hout = [torch.empty_like(hx).pin_memory() for _ in range(E2E_STREAMS)]
    hst = [torch.zeros(1, dtype=torch.int32).pin_memory() for _ in range(E2E_STREAMS)]
    c_layers = [l.c for l in wsp.layers]
    nbytes = _lib.mtgr_stack_fwd_host_workspace_bytes(hl, c_layers)
    dws = [torch.empty(nbytes, dtype=torch.uint8, device=dev) for _ in range(E2E_STREAMS)]
    streams = [torch.cuda.Stream(dev) for _ in range(E2E_STREAMS)]
    h2d = hl.numel() * 4 + ht.numel() * 8 + hx.numel() * 4 + (hn.numel() * 4 if hn is not None else 0)
    d2h = hout[0].numel() * 4 + 4

    def run(n):
        for k in range(n):
            i = k % E2E_STREAMS
            _lib.mtgr_stack_fwd_host(c_layers, hl, ht, hn, hx, hout[i], hst[i], dws[i], streams[i])

    run(E2E_STREAMS)
    torch.cuda.synchronize(dev)
    barrier(world)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    cur = torch.cuda.current_stream(dev)
    ev[0].record(cur)
    for st in streams:
        st.wait_stream(cur)
    run(steps)
    for st in streams:
        cur.wait_stream(st)
    ev[1].record(cur)
    torch.cuda.synchronize(dev)
    ems = max_over_ranks(ev[0].elapsed_time(ev[1]), world, dev)
    assert all(int(h.item()) == 0 for h in hst), "e2e device status"
    wsp.step()
    torch.cuda.synchronize(dev)
    assert torch.equal(hout[(steps - 1) % E2E_STREAMS], wsp.out.cpu()), "e2e output mismatch"
    return {"value": users_total * steps / (ems / 1e3), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": ems / steps,
            "path": "C ABI mtgr_stack_fwd_host (host buffers in, host buffers out)",
            "pipelining": f"{E2E_STREAMS} streams, {E2E_STREAMS} workspaces: one step's input copy, "
                          "another's kernels and a third's output copy overlap"}


def run_ours(args, world, rank, local):
    from generative_recommendation_ranking_b200 import _lib

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if synth.WORKLOADS[args.config].kind == "sweep":
        raise SystemExit("use --config 4 through run_sweep")
    wl, B_global = rank_workload(args, world, rank)
    B, T, d, H, dff, L = (int(wl["lens"].shape[0]), int(wl["lens"].sum()), wl["d"], wl["H"],
                          wl["d_ff"], wl["L"])
    stream = torch.cuda.current_stream(dev)
    wsp = Workspace(wl, dev, stream)
    batch = wsp.batch
    for _ in range(args.warmup):
        wsp.step()
    batch.check()

    timer = _lib.Timer()
    clocks = ClockSampler(dev)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize(dev)
    flush = (torch.zeros(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
             if needs_flush(wl) else None)
    timer.attach()
    ms = time_steps(wsp.step, args.steps, stream, flush)
    timer.detach()
    barrier(world)
    clk = clocks.stop()
    ms_max = max_over_ranks(ms, world, dev)
    batch.check()
    per_class = timer.read()
    Q, E, V, P = (int(v) for v in batch.counts.cpu())
    e2e = None if args.no_e2e else run_e2e(wsp, args.e2e_steps, world, dev, B_global)

    if rank != 0:
        return
    peaks, peak_src = load_peaks()
    tensor_key = tensor_peak_key(ms_max / 1e3)
    f32 = wl["dtype"] == "f32"
    # algorithmic work per launch of each class
    gln_bytes = (8.0 if f32 else 5.0) * d * T  # bf16 path: GroupLN_1 6d, GroupLN_2 4d bytes/token
    work = {
        "gemm_qkvu": ("tensor", 2.0 * T * 4 * d * d),
        "attention": ("tensor", 4.0 * d * V),
        "gemm_mlp1": ("tensor", 2.0 * T * dff * d),
        "gemm_mlp2": ("tensor", 2.0 * T * d * dff),
        "gln": ("hbm", gln_bytes),
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
                            "peak": peaks[tensor_key], "avg_ms": avg_ms, "launches": n,
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
    # The attention's binding pipe is the MUFU, not the tensor pipe: every score
    # needs one tanh, and the SM evaluates 16 per clock (8 tanh.approx.f16x2
    # instructions; measured on this part at 4-16 warps per SM), against
    # 128x128x64 x 2 MMAs per 16384 scores that the tensor pipe clears in
    # fewer cycles. Algorithmic work: one silu per visible (query, key) pair
    # and head; peak: 16 x SMs x the SM clock sampled during the timed region.
    if "attention" in kernels and not f32:
        sm_mhz = (clk or {}).get("sm_mhz") or (clk or {}).get("sm_max_mhz") or 1965.0
        n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
        att_t = kernels["attention"]
        sfu_ach = V * H / (att_t["avg_ms"] * 1e-3) / 1e9
        sfu_peak = 16.0 * n_sm * sm_mhz * 1e6 / 1e9
        kernels["attention"]["sfu"] = {"bound": "alu", "achieved": sfu_ach, "unit": "Gsilu/s",
                                       "peak": sfu_peak, "frac": sfu_ach / sfu_peak,
                                       "peak_source": f"MUFU tanh 16/clk/SM x {n_sm} SMs x {sm_mhz:.0f} MHz"}
    dom = max((c for c in work if c in kernels), key=lambda c: kernels[c]["share"])
    k = kernels[dom]
    traffic = ncu_traffic(dom, wl["name"], int(wl["lens"].shape[0]))
    roofline = {"bound": k["bound"], "achieved": k["achieved"], "peak": k["peak"], "unit": k["unit"],
                "frac": k["frac"], "traffic": traffic, "kernel": dom,
                "peak_source": f"{peak_src} ({tensor_key if k['bound'] == 'tensor' else 'hbm_gbs'}; "
                               f"timed region {ms_max / 1e3:.2f} s)"}
    if "sfu" in k:  # the attention's binding pipe, beside the tensor view
        roofline["sfu"] = k["sfu"]
    att = kernels.get("attention", {})
    value = B_global * args.steps / (ms_max / 1e3)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        r = oracle_users_per_s(wl, args.cpu_seconds)
        r1 = oracle_users_per_s(wl, args.cpu_seconds / 3, max_threads=1)
        cpu = {"value": r["value"], "unit": UNIT, "cores": r["threads"], "kind": "oracle",
               "sample": f"first {r['users']} users of {wl['name']} (seed {args.seed}), "
                         f"float64 NumPy, {r['seconds']:.1f} s",
               "single_thread": {"value": r1["value"], "unit": UNIT,
                                 "sample": f"first {r1['users']} users, {r1['seconds']:.1f} s"}}
    launches = int(sum(n for _, n in per_class.values()))
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": dtype_label(wl), "data": "synthetic",
        "config": workload_config(wl, world, B_global),
        "masked_attn": {"tflops": att.get("achieved"),
                        "frac_of_bf16_peak": att.get("frac"),
                        "visible_pairs_per_gpu": V, "q_tiles": Q, "tile_entries": E,
                        "work_items": P},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clk,
        "gpu_launches": launches, "kernels": kernels,
    }
    print(json.dumps(line), flush=True)


def incremental_leg(agg: dict, dev, stream, args) -> dict:
    """The same user served with its context cached: the context pass (U, S,
    R through the block, Q|K|V|U kept) timed once per request of new context,
    and the candidate pass (all K candidates over the cached keys) timed as
    the per-request work once the context is cached. Both include their
    packing and mask metadata."""
    import generative_recommendation_ranking_b200 as mt
    from generative_recommendation_ranking_b200 import _lib
    n_u, n_s, n_r, K = (int(v) for v in agg["lens"][0])
    n_ctx = n_u + n_s + n_r
    layers = [mt.BlockWeights(p, agg["H"], dtype="bf16", device=dev) for p in agg["layers"]]
    x = torch.from_numpy(agg["x"]).to(dev)
    xc, xk = x[:n_ctx], x[n_ctx:]
    cc = mt.ContextCache(layers, n_u, n_s, n_r, agg["ts"][:n_ctx], xc, K, K, stream=stream)
    cb = cc.ctx_batch
    batch = cc.candidate_batch(agg["ts"][n_ctx:], stream)
    ws = cc.workspace(K)
    out = torch.empty(K, agg["d"], dtype=torch.float32, device=dev)

    def ctx_step(s=stream):
        cb.pack(s)
        cb.build_meta(s)
        _lib.mtgr_stack_fwd_rows(cc.c_layers, cb.c, 0, cc.cache, cc.cache_rows, xc, cc.out,
                                 cc.ctx_ws, s)

    def cand_step(s=stream):
        batch.pack(s)
        batch.build_meta(s)
        _lib.mtgr_restrict_work(batch.c, cc.q_first, s)
        cc.score(None, xk, out=out, ws=ws, batch=batch, stream=s)

    res = {}
    n = max(5, min(args.steps, 50))
    for name, fn in (("context", ctx_step), ("incremental", cand_step)):
        for _ in range(max(3, args.warmup)):
            fn()
        ms = time_steps(fn, n, stream) / n
        batch.check()
        res[f"{name}_ms"] = ms
        res[f"{name}_graph_ms"] = graph_steps_ms(fn, n, max(3, args.warmup))
        batch.check()
    res["incremental_ms_per_candidate"] = res["incremental_ms"] / K
    res["incremental_graph_ms_per_candidate"] = res["incremental_graph_ms"] / K
    return res


def run_sweep(args, local):
    """Candidate scaling for one user (d_model 512, 8 heads, one block): the
    aggregated sample [U, S, R, c_1..c_K] against K expanded rows [U, S, R, c_i]
    at the same normaliser, for K in 1, 8, 64, 512."""
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    rows = []
    for K in synth.WORKLOADS[4].sweep_k:
        agg = synth.make_workload(4, seed=args.seed, k_override=K)
        res = {"K": K}
        for name, wl in (("aggregated", agg), ("expanded", synth.sweep_expanded(agg))):
            wsp = Workspace(wl, dev, stream)
            for _ in range(max(3, args.warmup)):
                wsp.step()
            wsp.batch.check()
            n = max(5, min(args.steps, 50))
            ms = time_steps(wsp.step, n, stream) / n
            wsp.batch.check()
            res[f"{name}_ms"] = ms
            res[f"{name}_ms_per_candidate"] = ms / K
            res[f"{name}_graph_ms"] = graph_steps_ms(lambda s: wsp.step(stream=s), n,
                                                     max(3, args.warmup))
            wsp.batch.check()
            del wsp
            torch.cuda.empty_cache()
        res.update(incremental_leg(agg, dev, stream, args))
        rows.append(res)
    marginal = (rows[-1]["aggregated_ms"] - rows[0]["aggregated_ms"]) / (rows[-1]["K"] - rows[0]["K"])
    line = {"metric": "candidate sweep: HSTU-block fwd ms per candidate, aggregated vs expanded rows vs cached context",
            "unit": "ms", "higher_is_better": False, "data": "synthetic", "dtype": "bf16",
            "config": {"workload": "sweep_b1_d512", "d_model": 512, "heads": 8, "d_ff": 2048,
                       "n_u": 24, "s": 1000, "r": 64},
            "l2": "not flushed: one user's inputs and weights fit in L2",
            "sweep": rows, "aggregated_marginal_ms_per_added_candidate": marginal,
            "incremental_ms_per_candidate_at_k512": rows[-1]["incremental_ms_per_candidate"],
            "graph": "*_graph_ms: the same step captured once into a CUDA graph and replayed",
            "expanded_ms_per_row_at_k512": rows[-1]["expanded_ms_per_candidate"]}
    print(json.dumps(line), flush=True)


def expanded_rows(agg: dict, rows: int) -> dict:
    """`rows` expanded rows [U, S, R, c] taken user by user, candidate by
    candidate, from a many-user aggregated sweep batch: each row repeats its
    user's U, S, R tokens and holds one of its candidates, with the
    aggregated user's normaliser N = N_U + N_S + N_R + K."""
    lens = np.asarray(agg["lens"])
    n_u, n_s, n_r, K = (int(v) for v in lens[0])
    n_ctx, n = n_u + n_s + n_r, n_u + n_s + n_r + K
    xs, tss = [], []
    for r in range(rows):
        b, c = divmod(r, K)
        s0 = b * n
        xs += [agg["x"][s0:s0 + n_ctx], agg["x"][s0 + n_ctx + c:s0 + n_ctx + c + 1]]
        tss += [agg["ts"][s0:s0 + n_ctx], agg["ts"][s0 + n_ctx + c:s0 + n_ctx + c + 1]]
    out = dict(agg)
    out["lens"] = np.tile(np.array([[n_u, n_s, n_r, 1]], np.int32), (rows, 1))
    out["x"] = np.concatenate(xs, axis=0)
    out["ts"] = np.concatenate(tss)
    out["norm"] = np.full(rows, float(n), np.float32)
    out["kind"] = "sweep_expanded"
    return out


def run_sweep_batched(args, local):
    """The candidate sweep with many users per launch: B users of the sweep's
    shape (N_U 24, S 1000, R 64, d_model 512, one block), each with K
    candidates, K in 1, 8, 64, 512. Legs per K:
      aggregated: pack + metadata + block over the B samples [U, S, R, c_1..c_K];
      cached: the cached-context candidate pass (the B contexts computed once,
        every layer's Q|K|V|U kept; per request only the candidate rows);
      expanded: B K rows [U, S, R, c_i] at the same normaliser, timed on up to
        4096 rows and scaled by the row count (rows are independent users of
        equal length, so their cost is linear in the row count).
    Reported: ms per step and per candidate for each leg, and the aggregated
    pass's marginal cost per added candidate between K = 1 and K = 512."""
    import generative_recommendation_ranking_b200 as mt
    from generative_recommendation_ranking_b200 import _lib
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    B = args.sweep_users
    n = max(5, min(args.steps, 30))
    rows_out = []
    for K in synth.WORKLOADS[4].sweep_k:
        agg = synth.make_workload(4, seed=args.seed, k_override=K, B=B)
        res = {"K": K, "candidates": B * K}
        wsp = Workspace(agg, dev, stream)
        for _ in range(max(3, args.warmup)):
            wsp.step()
        wsp.batch.check()
        ms = time_steps(wsp.step, n, stream) / n
        wsp.batch.check()
        res["aggregated_ms"] = ms
        res["aggregated_ms_per_candidate"] = ms / (B * K)
        # cached contexts: the candidate pass over all B users
        lens = agg["lens"]
        x = wsp.x
        gid = torch.from_numpy(np.repeat(np.tile(np.arange(4), B), lens.reshape(-1).astype(np.int64))).to(dev)
        x_cand = x[gid == 3].contiguous()
        cc = mt.BatchContextCache(wsp.layers, lens, agg["ts"], x, stream=stream)
        cbatch = cc.candidate_batch(agg["ts"], stream)
        cws = cc.workspace()
        out = torch.empty(cc.k_total, agg["d"], dtype=torch.float32, device=dev)
        c_layers = [l.c for l in wsp.layers]

        def cand_step():
            cbatch.pack(stream)
            cbatch.build_meta(stream)
            _lib.mtgr_stack_fwd_candidates(c_layers, cbatch.c, cc.k_total, cc.cache, cc.T, x_cand,
                                           out, cws, stream)

        for _ in range(max(3, args.warmup)):
            cand_step()
        cbatch.check()
        ms = time_steps(cand_step, n, stream) / n
        cbatch.check()
        res["cached_ms"] = ms
        res["cached_ms_per_candidate"] = ms / (B * K)
        del cc, cbatch, cws, out, x_cand, wsp
        torch.cuda.empty_cache()
        # expanded rows, scaled linearly from at most 4096 rows
        rows = min(B * K, 4096)
        ex = Workspace(expanded_rows(agg, rows), dev, stream)
        for _ in range(max(3, args.warmup)):
            ex.step()
        ex.batch.check()
        ms = time_steps(ex.step, n, stream) / n
        ex.batch.check()
        res["expanded_rows_timed"] = rows
        res["expanded_ms_per_candidate"] = ms / rows
        res["expanded_ms"] = ms / rows * B * K
        del ex
        torch.cuda.empty_cache()
        rows_out.append(res)
    first, last = rows_out[0], rows_out[-1]
    marginal = (last["aggregated_ms"] - first["aggregated_ms"]) / (B * (last["K"] - first["K"]))
    line = {"metric": "candidate sweep, many users per launch: HSTU-block fwd ms per candidate, "
                      "aggregated vs cached context vs expanded rows",
            "unit": "ms", "higher_is_better": False, "data": "synthetic", "dtype": "bf16",
            "config": {"workload": f"sweep_b{B}_d512", "users": B, "d_model": 512, "heads": 8,
                       "d_ff": 2048, "n_u": 24, "s": 1000, "r": 64},
            "sweep": rows_out,
            "aggregated_marginal_ms_per_added_candidate": marginal,
            "expanded_ms_per_candidate_at_k512": last["expanded_ms_per_candidate"],
            "marginal_vs_expanded": marginal / last["expanded_ms_per_candidate"]}
    print(json.dumps(line), flush=True)


def run_serving(args, local):
    """Serving with cached contexts on the 512-user block workload: the
    contexts (U, S, R) of all users run once with every layer's Q|K|V|U kept;
    each candidate request then recomputes the candidate rows only. Timed:
    the aggregated pass (pack + metadata + block over every row), the context
    pass, and the candidate pass (pack + metadata + the candidate rows)."""
    import generative_recommendation_ranking_b200 as mt
    from generative_recommendation_ranking_b200 import _lib
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    wl = synth.make_workload(2, seed=args.seed, B=args.users)
    lens = wl["lens"]
    wsp = Workspace(wl, dev, stream)
    layers = wsp.layers
    x = wsp.x
    gid = torch.from_numpy(np.repeat(np.tile(np.arange(4), lens.shape[0]),
                                     lens.reshape(-1).astype(np.int64)).astype(np.int64)).to(dev)
    cand = gid == 3
    x_cand = x[cand].contiguous()
    cc = mt.BatchContextCache(layers, lens, wl["ts"], x, stream=stream)
    cb = cc.batch
    cws = cc.ctx_ws
    batch = cc.candidate_batch(wl["ts"], stream)
    ws = cc.workspace()
    out = torch.empty(cc.k_total, wl["d"], dtype=torch.float32, device=dev)
    c_layers = [l.c for l in layers]

    def ctx_step():
        cb.pack(stream)
        cb.build_meta(stream)
        _lib.mtgr_stack_fwd_rows(c_layers, cb.c, 0, cc.cache, cc.T, x, cc.out, cws, stream)

    def cand_step():
        batch.pack(stream)
        batch.build_meta(stream)
        _lib.mtgr_stack_fwd_candidates(c_layers, batch.c, cc.k_total, cc.cache, cc.T, x_cand, out, ws,
                                       stream)

    n = max(5, min(args.steps, 100))
    res = {}
    for name, fn in (("aggregated", wsp.step), ("context", ctx_step), ("candidates", cand_step)):
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize(dev)
        timer = _lib.Timer()
        timer.attach()
        ms = time_steps(fn, n, stream) / n
        timer.detach()
        batch.check()
        per = timer.read()
        res[name] = {"ms_per_step": ms,
                     "kernels_ms": {c: round(t / n, 4) for c, (t, k) in per.items() if k}}
    K = cc.k_total
    line = {"metric": "cached-context candidate scoring: candidate pass vs aggregated pass",
            "value": lens.shape[0] / (res["candidates"]["ms_per_step"] * 1e-3),
            "unit": "user-samples/s", "ms_per_step": res["candidates"]["ms_per_step"],
            "steps": n, "higher_is_better": True, "n_gpus": 1, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl["name"], "users": int(lens.shape[0]), "tokens": cc.T,
                       "candidates": K, "l2": "inputs 0.9 GB > L2"},
            "candidates_per_s": K / (res["candidates"]["ms_per_step"] * 1e-3),
            "speedup_vs_aggregated": res["aggregated"]["ms_per_step"] / res["candidates"]["ms_per_step"],
            "parts": res}
    print(json.dumps(line), flush=True)


def run_pipeline(args, local):
    """The ranking forward around the block on the 512-user block workload:
    the per-domain token MLPs build X, the HSTU block runs, the task heads
    score the candidates. Each part is timed with the library's event timer;
    the step is the three calls back to back (pack and mask metadata once)."""
    import generative_recommendation_ranking_b200 as mt
    from generative_recommendation_ranking_b200 import _lib
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    wl = synth.make_workload(2, seed=args.seed, B=args.users)
    lens, d = wl["lens"], wl["d"]
    rng = np.random.default_rng(args.seed + 1)
    e = [torch.from_numpy(a).to(dev).to(torch.bfloat16) for a in synth.make_token_inputs(lens, d, rng)]
    mlps = mt.TokenMLPs(synth.make_token_params(d, rng), device=dev)
    heads = mt.CandidateHeads(synth.make_head_params(d, rng), device=dev)
    batch = mt.PackedBatch(lens, wl["ts"], device=dev)
    layers = [mt.BlockWeights(p, wl["H"], device=dev) for p in wl["layers"]]
    T = batch.T
    n_rows = [int(lens[:, g].sum()) for g in range(4)]
    K = n_rows[3]
    x = torch.empty(T, d, dtype=torch.float32, device=dev)
    y = torch.empty_like(x)
    logits = torch.empty(K, heads.n_tasks, dtype=torch.float32, device=dev)
    tws = torch.empty(_lib.mtgr_tokenize_workspace_bytes(batch.B, d, n_rows), dtype=torch.uint8,
                      device=dev)
    hws = torch.empty(_lib.mtgr_heads_workspace_bytes(batch.B, K, heads.c), dtype=torch.uint8,
                      device=dev)
    sws = mt.stack_workspace(layers, batch)

    def step():
        _lib.mtgr_tokenize(batch.c, d, n_rows, e, mlps.c, x, tws, stream)
        _lib.mtgr_stack_fwd([l.c for l in layers], batch.c, x, y, sws, stream)
        _lib.mtgr_candidate_heads(heads.c, batch.c, K, y, logits, hws, stream)

    for _ in range(max(3, args.warmup)):
        step()
    batch.check()
    n = max(5, min(args.steps, 100))
    timer = _lib.Timer()
    clocks = ClockSampler(dev)
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize(dev)
    timer.attach()
    ms = time_steps(step, n, stream) / n
    timer.detach()
    clk = clocks.stop()
    batch.check()
    per = timer.read()
    peaks, _ = load_peaks()
    tkey = tensor_peak_key(ms * n / 1e3)
    f = synth.TOKEN_F
    tok_flop = 2.0 * sum(n_rows[g] * (f[g - 1] * d + d * d) for g in (1, 2, 3))
    head_flop = 2.0 * K * d * heads.n_tasks * synth.HEAD_DH
    parts = {}
    for cls, flop in (("token_mlp", tok_flop), ("head_mlp", head_flop)):
        t_ms, cnt = per[cls]
        avg = t_ms / n
        ach = flop / (avg * 1e-3) / 1e12
        parts[cls] = {"bound": "tensor", "ms_per_step": avg, "launches_per_step": cnt / n,
                      "achieved": ach, "unit": "TFLOP/s", "peak": peaks[tkey],
                      "frac": ach / peaks[tkey], "peak_source": tkey}
    block_ms = sum(per[c][0] for c in ("pack", "mask_meta", "gln", "gemm_qkvu", "attention",
                                       "gemm_mlp1", "gemm_mlp2")) / n
    parts["block"] = {"ms_per_step": block_ms}
    rows_ms = per["rows"][0] / n
    # row bookkeeping: U rows bf16 in -> fp32 out; candidate rows fp32 in -> bf16
    # out; the heads' last layer reads the hidden rows (bf16) once
    rows_bytes = (n_rows[0] * d * 6 + K * d * 6 + K * heads.n_tasks * synth.HEAD_DH * 2
                  + 4 * (T + K))
    parts["rows"] = {"bound": "hbm", "ms_per_step": rows_ms, "launches_per_step": per["rows"][1] / n,
                     "achieved": rows_bytes / (rows_ms * 1e-3) / 1e9, "unit": "GB/s",
                     "peak": peaks["hbm_gbs"]}
    parts["rows"]["frac"] = parts["rows"]["achieved"] / parts["rows"]["peak"]
    line = {"metric": "ranking forward: token MLPs -> HSTU block -> CTR/CTCVR heads",
            "value": batch.B / (ms * 1e-3), "unit": "user-samples/s", "ms_per_step": ms,
            "steps": n, "warmup": max(3, args.warmup), "higher_is_better": True, "n_gpus": 1,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl["name"], "users": batch.B, "tokens": T, "candidates": K,
                       "token_f": list(f), "head_dh": synth.HEAD_DH, "tasks": heads.n_tasks,
                       "l2": "inputs 0.9 GB > L2"},
            "parts": parts, "clocks": clk}
    print(json.dumps(line), flush=True)


def run_backward(args, local):
    """Training step of one bf16 block: pack, mask metadata, the forward that
    keeps the backward's activations, and the backward (dX and every
    parameter gradient), all through the C ABI, inputs and upstream gradient
    resident in HBM."""
    import generative_recommendation_ranking_b200 as mt
    from generative_recommendation_ranking_b200 import _lib
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = synth.make_workload(2, seed=args.seed, B=args.users)
    lens = wl["lens"]
    B, T, d, H, dff = int(lens.shape[0]), int(lens.sum()), wl["d"], wl["H"], wl["d_ff"]
    stream = torch.cuda.current_stream(dev)
    batch = mt.PackedBatch(lens, wl["ts"], device=dev)
    bw = mt.BlockWeights(wl["layers"][0], H, device=dev)
    x = torch.from_numpy(wl["x"]).to(dev)
    dy = torch.from_numpy(np.random.default_rng(args.seed + 1).standard_normal(
        wl["x"].shape, dtype=np.float32)).to(dev)
    y = torch.empty_like(x)
    dx = torch.empty_like(x)
    saved = torch.empty(_lib.mtgr_block_saved_bytes(T, bw.c), dtype=torch.uint8, device=dev)
    bws = torch.empty(_lib.mtgr_block_bwd_workspace_bytes(T, bw.c, batch.c), dtype=torch.uint8,
                      device=dev)
    shapes = {"gln1_gamma": (4, d), "gln1_beta": (4, d), "w_qkvu": (4 * d, d),
              "gln2_gamma": (4, d), "gln2_beta": (4, d), "w1": (dff, d), "w2": (d, dff)}
    grads = {k: torch.empty(v, dtype=torch.float32, device=dev) for k, v in shapes.items()}
    gc = _lib.MtgrBlockGrads(**{k: v.data_ptr() for k, v in grads.items()})

    def step():
        batch.pack(stream)
        batch.build_meta(stream)
        _lib.mtgr_hstu_block_fwd_train(bw.c, batch.c, x, y, saved, stream)
        _lib.mtgr_hstu_block_bwd(bw.c, batch.c, x, saved, dy, dx, gc, bws, stream)

    for _ in range(max(3, args.warmup)):
        step()
    batch.check()
    n = max(3, min(args.steps, 50))
    timer = _lib.Timer()
    clocks = ClockSampler(dev)
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize(dev)
    timer.attach()
    ms = time_steps(step, n, stream) / n
    timer.detach()
    clk = clocks.stop()
    batch.check()
    per = timer.read()
    V = int(batch.counts[2].item())
    peaks, peak_src = load_peaks()
    tkey = tensor_peak_key(ms * n / 1e3)
    # algorithmic work per step of each class (bf16 block, dh = 64):
    #   forward: projections 2 T (4 d^2 + 2 d d_ff), attention 4 d V
    #   backward GEMMs dH, dG~, dX~: 2 T (d d_ff + d_ff d + 4 d^2); weight
    #   gradients the same count; attention backward 10 d V (S, dP, dV, dK,
    #   dQ: 2 dh FLOP each per visible pair and head)
    gemm_flop = 2.0 * T * (d * dff + dff * d + 4 * d * d)
    work = {"bwd_gemm": ("tensor", gemm_flop), "bwd_wgrad": ("tensor", gemm_flop),
            "bwd_attention": ("tensor", 10.0 * d * V),
            "attention": ("tensor", 4.0 * d * V),
            "gemm_qkvu": ("tensor", 2.0 * T * 4 * d * d), "gemm_mlp1": ("tensor", 2.0 * T * d * dff),
            "gemm_mlp2": ("tensor", 2.0 * T * d * dff),
            # GroupLN backward, bytes per token: GLN_1 reads x (fp32), dX~
            # (bf16), dY (fp32) and writes dX (fp32): 14 d; GLN_2 with the
            # gate reads G (bf16), dG~ (bf16), U (f16), O/N (bf16) and writes
            # dO~ (f16), dU (bf16): 12 d
            "bwd_gln": ("hbm", T * d * (14.0 + 12.0))}
    kernels = {}
    for cls, (bound, w) in work.items():
        t_ms, cnt = per[cls]
        if cnt == 0:
            continue
        avg = t_ms / n
        ach = w / (avg * 1e-3) / (1e12 if bound == "tensor" else 1e9)
        peak = peaks[tkey] if bound == "tensor" else peaks["hbm_gbs"]
        kernels[cls] = {"bound": bound, "ms_per_step": avg, "launches_per_step": cnt / n,
                        "achieved": ach, "unit": "TFLOP/s" if bound == "tensor" else "GB/s",
                        "peak": peak, "frac": ach / peak, "share": t_ms / (ms * n)}
    for cls in ("pack", "mask_meta", "gln", "bwd_rows"):
        t_ms, cnt = per[cls]
        if cnt:
            kernels[cls] = {"ms_per_step": t_ms / n, "launches_per_step": cnt / n,
                            "share": t_ms / (ms * n)}
    bwd = [c for c in ("bwd_gemm", "bwd_wgrad", "bwd_attention", "bwd_gln") if c in kernels]
    dom = max(bwd, key=lambda c: kernels[c]["share"])
    k = kernels[dom]
    total_flop = 3 * gemm_flop + 14.0 * d * V
    line = {"metric": "HSTU-block training step (fwd + bwd) user-samples/s",
            "value": B / (ms * 1e-3), "unit": "user-samples/s", "ms_per_step": ms, "steps": n,
            "warmup": max(3, args.warmup), "higher_is_better": True, "n_gpus": 1,
            "dtype": "bf16 (attention operands f16, fp32 accumulate)", "data": "synthetic",
            "config": {"workload": wl["name"], "users": B, "tokens": T, "d_model": d, "heads": H,
                       "d_ff": dff, "layers": 1, "visible_pairs": V,
                       "l2": "inputs larger than L2 (fp32 token features and gradient, 1.9 GB)"},
            "step_tflops": total_flop / (ms * 1e-3) / 1e12,
            "roofline": {"bound": k["bound"], "achieved": k["achieved"], "peak": k["peak"],
                         "unit": k["unit"], "frac": k["frac"],
                         "traffic": ncu_traffic(dom, wl["name"], B) if dom in KERNEL_SRC else None,
                         "kernel": dom,
                         "peak_source": f"{peak_src} ({tkey if k['bound'] == 'tensor' else 'hbm_gbs'})"},
            "kernels": kernels, "gpu_launches": int(sum(c for _, c in per.values()) / n),
            "clocks": clk}
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    world, rank, local = dist_setup(args) if args.impl == "ours" else (
        int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        elif args.serving:
            if rank == 0:
                run_serving(args, local)
        elif args.pipeline:
            if rank == 0:
                run_pipeline(args, local)
        elif args.backward:
            if rank == 0:
                run_backward(args, local)
        elif synth.WORKLOADS[args.config].kind == "sweep":
            if rank == 0:
                if args.sweep_users > 0:
                    run_sweep_batched(args, local)
                else:
                    run_sweep(args, local)
        else:
            run_ours(args, world, rank, local)
    finally:
        if args.impl == "ours" and world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
