"""Helpers shared by the GPU parity tests (no method arithmetic here)."""

from __future__ import annotations

import numpy as np
import torch

TOL_F32 = 1e-4   # max-abs error / RMS(oracle output), fp32 path
TOL_BF16 = 2e-2  # max-abs error / RMS(oracle output), bf16 path


def assert_close_rms(gpu, ref, tol, what=""):
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite GPU values"
    rms = float(np.sqrt(np.mean(r ** 2))) if r.size else 0.0
    err = float(np.max(np.abs(g - r))) if r.size else 0.0
    assert err <= tol * rms + 1e-30, f"{what}: max|err| {err:.3e} > {tol} x RMS {rms:.3e} ({err / max(rms, 1e-300):.2e})"
    return err / max(rms, 1e-300)


def assert_close_bf16_out(gpu, ref, what="", tol=1e-2):
    """Bar for an intermediate tensor stored in bf16: within one bf16 rounding
    of the exact value (|rounded - x| <= 2^-8 |x| for round-to-nearest) plus a
    computation error of ``tol`` x RMS."""
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite GPU values"
    rms = float(np.sqrt(np.mean(r ** 2))) if r.size else 0.0
    excess = np.abs(g - r) - 2.0 ** -8 * np.abs(r)
    worst = float(excess.max()) if r.size else 0.0
    assert worst <= tol * rms, f"{what}: error beyond bf16 rounding {worst:.3e} > {tol} x RMS {rms:.3e}"
    return worst / max(rms, 1e-300)


def user_rows(lens, users):
    """Row indices (in the packed layout) of the given users, in order."""
    n = np.asarray(lens, np.int64).reshape(-1, 4).sum(1)
    off = np.concatenate([[0], np.cumsum(n)])
    return np.concatenate([np.arange(off[u], off[u + 1]) for u in users]) if len(users) else np.zeros(0, np.int64)


def sample_users(lens, k=4, seed=0):
    """First, last, longest, shortest and a few random users."""
    n = np.asarray(lens, np.int64).reshape(-1, 4).sum(1)
    rng = np.random.default_rng(seed)
    pick = {0, len(n) - 1, int(np.argmax(n)), int(np.argmin(n))}
    pick |= set(rng.choice(len(n), size=min(k, len(n)), replace=False).tolist())
    return sorted(pick)


def to_host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def _oracle_stack_chunk(args):
    import oracle
    x, lens, ts, layers, H, variant = args
    return oracle.hstu_stack(x, lens, ts, layers, H, variant=variant)


def oracle_stack_all_users(w, procs=None, chunk=8, variant=0):
    """The oracle's stack output for every user of workload ``w``, computed in
    chunks of users by a pool of single-threaded worker processes. The pool is
    started with ``spawn`` (a forked child of a process that has used the GPU
    can hang), and users are independent, so the chunks concatenate to the
    whole batch's output."""
    import multiprocessing as mp
    import os
    lens = np.asarray(w["lens"]).reshape(-1, 4)
    n = lens.sum(1)
    off = np.concatenate([[0], np.cumsum(n)])
    jobs = []
    for u0 in range(0, lens.shape[0], chunk):
        u1 = min(lens.shape[0], u0 + chunk)
        r0, r1 = int(off[u0]), int(off[u1])
        jobs.append((w["x"][r0:r1], lens[u0:u1], w["ts"][r0:r1], w["layers"], w["H"], variant))
    procs = procs or max(1, len(os.sched_getaffinity(0)))
    saved = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
    for k in saved:
        os.environ[k] = "1"  # inherited by the spawned workers: one BLAS thread each
    try:
        with mp.get_context("spawn").Pool(procs) as pool:
            parts = pool.map(_oracle_stack_chunk, jobs)
    finally:
        for k, v in saved.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
    return np.concatenate(parts, axis=0)


def _oracle_backward_chunk(args):
    import oracle
    x, lens, ts, p, H, dy = args
    return oracle.hstu_block_backward(x, lens, ts, p, H, dy)


def oracle_backward_all_users(w, dy, procs=None, chunk=8):
    """The oracle's block backward over every user of workload ``w`` (one
    block): per-user chunks on a spawned pool of single-threaded workers; the
    input gradient rows concatenate and the parameter gradients, sums over
    tokens, add up across chunks."""
    import multiprocessing as mp
    import os
    lens = np.asarray(w["lens"]).reshape(-1, 4)
    off = np.concatenate([[0], np.cumsum(lens.sum(1))])
    jobs = []
    for u0 in range(0, lens.shape[0], chunk):
        u1 = min(lens.shape[0], u0 + chunk)
        r0, r1 = int(off[u0]), int(off[u1])
        jobs.append((w["x"][r0:r1], lens[u0:u1], w["ts"][r0:r1], w["layers"][0], w["H"], dy[r0:r1]))
    procs = procs or max(1, len(os.sched_getaffinity(0)))
    saved = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
    for k in saved:
        os.environ[k] = "1"
    try:
        with mp.get_context("spawn").Pool(procs) as pool:
            parts = pool.map(_oracle_backward_chunk, jobs)
    finally:
        for k, v in saved.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
    out = {"x": np.concatenate([p["x"] for p in parts], axis=0)}
    for k in parts[0]:
        if k != "x":
            out[k] = sum(p[k] for p in parts)
    return out

# bf16 backward: gradient tensors inherit the per-element error of the
# forward's saved bf16/f16 activations (about 0.5% of an element), which sums
# over tokens do not dilute. Bars: the RMS error of a tensor within 1e-2 of
# its RMS (the bulk, about 2 sigma), and its largest error within 2e-2 of its
# largest element (the tail: gradient tensors are heavy-tailed, their largest
# elements 10-20 x RMS, and each element carries its own relative error)
TOL_BF16_GRAD_RMS = 1e-2
TOL_BF16_GRAD_PEAK = 2e-2


def grad_errors(gpu, ref):
    """(max-abs error / max|ref|, RMS error / RMS(ref), max-abs error / RMS(ref))."""
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    if not r.size:
        return 0.0, 0.0, 0.0
    rms = float(np.sqrt(np.mean(r ** 2)))
    peak = float(np.max(np.abs(r)))
    d = g - r
    mx = float(np.max(np.abs(d)))
    return (mx / max(peak, 1e-300), float(np.sqrt(np.mean(d ** 2))) / max(rms, 1e-300),
            mx / max(rms, 1e-300))


def assert_grads_close(got: dict, ref: dict, peak_tol: float, rms_tol: float, what: str):
    """Every gradient tensor of ``ref`` against ``got``: finite, largest error
    <= peak_tol x its largest element and RMS error <= rms_tol x its RMS;
    prints each tensor's errors (also the largest error over the RMS) so the
    margins stay on record."""
    report = []
    for k in ref:
        g = np.asarray(got[k], np.float64)
        assert g.shape == np.shape(ref[k]), (k, g.shape, np.shape(ref[k]))
        assert np.isfinite(g).all(), f"{what}: d{k} has non-finite values"
        pk, rm, mx = grad_errors(g, ref[k])
        report.append(f"d{k} peak {pk:.2e} rms {rm:.2e} max/rms {mx:.2e}")
    print(f"{what}: " + "; ".join(report))
    for k in ref:
        pk, rm, _ = grad_errors(got[k], ref[k])
        assert pk <= peak_tol and rm <= rms_tol, \
            f"{what}: d{k} peak {pk:.2e} (<= {peak_tol}) rms {rm:.2e} (<= {rms_tol})"
