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
