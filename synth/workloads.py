"""Seeded synthetic inputs shaped like the MTGR pages' workloads.

The Meituan dataset the paper trains on is not public, so these generators stand
in for it. Every user request is D = [U, S, R, [C,I]_1..K] (MTGR paper, "Method",
the user-aggregated sample D): N_U scalar-feature tokens, N_S long-term
behaviour tokens, N_R real-time tokens and K candidate tokens, each a d_model
vector. Lengths follow the pages' caps (S up to ~1000, R up to ~100; "System"
section) except the long-tailed stack workload, which pushes S to 3000.

Random-draw recipe (numpy ``default_rng(seed)``, always in this order):
  1. per-user S lengths, then R lengths, then K lengths (vectorised over B);
  2. S timestamps (uniform int in [0, 1000)), then R timestamps (uniform int in
     [1000, 2000), sorted ascending within each user), then candidate exposure
     timestamps (uniform int in [1000, 2000), unsorted); U tokens carry 0,
     which the method ignores;
  3. token features N(0,1) times the group scale (U 1, S 3, R 0.3, C 10), or,
     for the attention-only workload, Q|K|V|U ~ N(0, variance 1/8);
  4. per layer: GroupLN-1 gamma = 1 + N(0, var 0.1), beta = N(0, var 0.1),
     then GroupLN-2 the same way, then W_qkvu as four stacked d x d
     Xavier-uniform blocks, then W1 [d_ff, d] and W2 [d, d_ff] Xavier-uniform.

Inputs of the steps around the stack, drawn on their own generator: per-domain
token inputs (E_U [sum N_U, d], E_S, E_R, E_C at the TOKEN_F widths, N(0, 1)),
then the token MLPs (per domain: W1 Xavier, b1, W2 Xavier, b2 N(0, var 0.01)),
then the task heads (W1 Xavier, b1, w2 Xavier, b2).

"N(0, x)" in the workload descriptions is read as variance x (the candidate
features of the sweep are written N(0, 10^2), i.e. standard deviation 10).

Nothing here computes any part of the method.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# group ids of the four token kinds
G_U, G_S, G_R, G_C = 0, 1, 2, 3

# per-group feature scales (U, S, R, candidate)
_SCALES = (1.0, 3.0, 0.3, 10.0)


def group_scales() -> tuple:
    return _SCALES


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str  # "block", "attention", "stack" or "sweep"
    B: int
    d: int
    H: int
    d_ff: int
    L: int
    dtype: str  # "f32" or "bf16"
    n_u: int
    s_len: tuple  # ("fixed", v) | ("uniform", lo, hi) inclusive | ("loguniform", lo, hi)
    r_len: tuple
    k_len: tuple
    sweep_k: tuple = field(default=())


WORKLOADS = {
    0: Workload("block_f32_b4_d64", "block", B=4, d=64, H=2, d_ff=256, L=1, dtype="f32",
                n_u=4, s_len=("fixed", 32), r_len=("fixed", 8), k_len=("fixed", 8)),
    1: Workload("attn_bf16_b256_d256", "attention", B=256, d=256, H=4, d_ff=0, L=1,
                dtype="bf16", n_u=16, s_len=("uniform", 200, 1000),
                r_len=("uniform", 10, 100), k_len=("uniform", 16, 128)),
    2: Workload("block_bf16_b512_d512", "block", B=512, d=512, H=8, d_ff=2048, L=1,
                dtype="bf16", n_u=24, s_len=("uniform", 300, 1000),
                r_len=("uniform", 20, 100), k_len=("uniform", 32, 256)),
    3: Workload("stack8_bf16_b256_d1024", "stack", B=256, d=1024, H=16, d_ff=4096, L=8,
                dtype="bf16", n_u=32, s_len=("loguniform", 256, 3000),
                r_len=("uniform", 32, 128), k_len=("uniform", 64, 512)),
    4: Workload("sweep_b1_d512", "sweep", B=1, d=512, H=8, d_ff=2048, L=1, dtype="bf16",
                n_u=24, s_len=("fixed", 1000), r_len=("fixed", 64), k_len=("fixed", 64),
                sweep_k=(1, 8, 64, 512)),
}


def _draw_len(rng: np.random.Generator, spec: tuple, B: int) -> np.ndarray:
    kind = spec[0]
    if kind == "fixed":
        return np.full(B, spec[1], dtype=np.int64)
    if kind == "uniform":
        return rng.integers(spec[1], spec[2] + 1, size=B)
    if kind == "loguniform":
        u = rng.uniform(np.log(spec[1]), np.log(spec[2]), size=B)
        return np.floor(np.exp(u)).astype(np.int64)
    raise ValueError(f"unknown length spec {spec!r}")


def make_lengths(wl: Workload, rng: np.random.Generator, k_override: int | None = None,
                 B: int | None = None) -> np.ndarray:
    """Per-user token counts, int32 [B, 4] = (N_U, N_S, N_R, K)."""
    B = wl.B if B is None else B
    s = _draw_len(rng, wl.s_len, B)
    r = _draw_len(rng, wl.r_len, B)
    k = _draw_len(rng, wl.k_len, B) if k_override is None else np.full(B, k_override)
    u = np.full(B, wl.n_u, dtype=np.int64)
    return np.stack([u, s, r, k], axis=1).astype(np.int32)


def make_timestamps(lens: np.ndarray, rng: np.random.Generator) -> np.ndarray:
    """int64 [T] timestamps laid out user by user in the order U, S, R, C."""
    lens = np.asarray(lens, dtype=np.int64)
    n_u, n_s, n_r, n_k = lens[:, 0], lens[:, 1], lens[:, 2], lens[:, 3]
    ts_s = rng.integers(0, 1000, size=int(n_s.sum()))
    ts_r = rng.integers(1000, 2000, size=int(n_r.sum()))
    ts_c = rng.integers(1000, 2000, size=int(n_k.sum()))
    out = []
    ps = pr = pc = 0
    for b in range(lens.shape[0]):
        out.append(np.zeros(n_u[b], dtype=np.int64))
        out.append(ts_s[ps:ps + n_s[b]])
        out.append(np.sort(ts_r[pr:pr + n_r[b]]))
        out.append(ts_c[pc:pc + n_k[b]])
        ps += n_s[b]
        pr += n_r[b]
        pc += n_k[b]
    if not out:
        return np.zeros(0, dtype=np.int64)
    return np.concatenate(out).astype(np.int64)


def _token_groups(lens: np.ndarray) -> np.ndarray:
    """Group id per token (input layout only: which slice of D a row came from)."""
    reps = np.asarray(lens, dtype=np.int64).reshape(-1)
    kinds = np.tile(np.array([G_U, G_S, G_R, G_C], dtype=np.int8), len(reps) // 4)
    return np.repeat(kinds, reps)


def make_tokens(lens: np.ndarray, d: int, rng: np.random.Generator) -> np.ndarray:
    """float32 [T, d] token features, N(0,1) times the per-group scale."""
    T = int(np.asarray(lens).sum())
    x = rng.standard_normal((T, d), dtype=np.float32)
    scale = np.asarray(_SCALES, dtype=np.float32)[_token_groups(lens)]
    x *= scale[:, None]
    return x


def make_qkvu(lens: np.ndarray, d: int, rng: np.random.Generator) -> np.ndarray:
    """float32 [T, 4d] projected Q|K|V|U for the attention-only workload, N(0, var 1/8)."""
    T = int(np.asarray(lens).sum())
    return (rng.standard_normal((T, 4 * d), dtype=np.float32) * np.float32(1.0 / np.sqrt(8.0)))


def _xavier(rng: np.random.Generator, fan_out: int, fan_in: int) -> np.ndarray:
    bound = np.sqrt(6.0 / (fan_in + fan_out))
    return rng.uniform(-bound, bound, size=(fan_out, fan_in)).astype(np.float32)


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even), kept as float32.

    Works on the 32-bit patterns in place: add 0x7FFF plus the lowest kept bit,
    then clear the low 16 bits (exact for every finite input)."""
    a = np.array(a, dtype=np.float32, copy=True, order="C")
    u = a.view(np.uint32)
    lsb = u >> np.uint32(16)
    lsb &= np.uint32(1)
    u += np.uint32(0x7FFF)
    u += lsb
    u &= np.uint32(0xFFFF0000)
    return a


def make_block_params(d: int, d_ff: int, rng: np.random.Generator, dtype: str = "bf16") -> dict:
    """One HSTU block's parameters (float32 arrays; weights bf16-representable for bf16)."""
    sd = np.float32(np.sqrt(0.1))
    p = {}
    for name in ("gln1", "gln2"):
        p[name + "_gamma"] = (1.0 + sd * rng.standard_normal((4, d), dtype=np.float32)).astype(np.float32)
        p[name + "_beta"] = (sd * rng.standard_normal((4, d), dtype=np.float32)).astype(np.float32)
    p["w_qkvu"] = np.concatenate([_xavier(rng, d, d) for _ in range(4)], axis=0)
    p["w1"] = _xavier(rng, d_ff, d)
    p["w2"] = _xavier(rng, d, d_ff)
    if dtype == "bf16":
        for k in ("w_qkvu", "w1", "w2"):
            p[k] = bf16_round(p[k])
    return p


def make_rab_tables(H: int, rng: np.random.Generator, scale: float = 2.0, max_dist: int = 128,
                    time_buckets: int = 32) -> tuple:
    """Per-head relative attention bias tables, N(0, scale^2) float32:
    positions [H, 2 max_dist + 1] and time buckets [H, time_buckets]."""
    pos = (scale * rng.standard_normal((H, 2 * max_dist + 1))).astype(np.float32)
    tim = (scale * rng.standard_normal((H, time_buckets))).astype(np.float32)
    return pos, tim


def make_stack_params(L: int, d: int, d_ff: int, rng: np.random.Generator, dtype: str = "bf16") -> list:
    return [make_block_params(d, d_ff, rng, dtype) for _ in range(L)]


def make_workload(index: int, seed: int = 0, k_override: int | None = None,
                  B: int | None = None) -> dict:
    """Draw a whole workload. Returns host arrays:

    lens int32 [B,4]; ts int64 [T]; x float32 [T,d] (block/stack/sweep) or
    qkvu float32 [T,4d] (attention, bf16-representable); layers: list of
    parameter dicts; plus the shape fields of the workload.
    """
    wl = WORKLOADS[index]
    rng = np.random.default_rng(seed)
    if wl.kind == "sweep" and k_override is None:
        k_override = wl.k_len[1]
    lens = make_lengths(wl, rng, k_override=k_override, B=B)
    ts = make_timestamps(lens, rng)
    out = dict(name=wl.name, index=index, kind=wl.kind, seed=seed, d=wl.d, H=wl.H,
               d_ff=wl.d_ff, L=wl.L, dtype=wl.dtype, lens=lens, ts=ts, norm=None)
    if wl.kind == "attention":
        q = make_qkvu(lens, wl.d, rng)
        out["qkvu"] = bf16_round(q) if wl.dtype == "bf16" else q
        out["layers"] = []
    else:
        out["x"] = make_tokens(lens, wl.d, rng)
        out["layers"] = make_stack_params(wl.L, wl.d, wl.d_ff, rng, wl.dtype)
    return out


def assemble_workload(index: int, lens: np.ndarray, ts: np.ndarray, token_rng: np.random.Generator,
                      weight_rng: np.random.Generator) -> dict:
    """A workload of the shape of ``index`` over given lengths and timestamps:
    token features (or Q|K|V|U) from ``token_rng`` and the layers' weights
    from ``weight_rng``. Used for one rank's share of a global batch: every
    rank passes the same weight generator seed, so the weights are identical
    (replicated) across ranks."""
    wl = WORKLOADS[index]
    lens = np.ascontiguousarray(np.asarray(lens, dtype=np.int32).reshape(-1, 4))
    out = dict(name=wl.name, index=index, kind=wl.kind, seed=None, d=wl.d, H=wl.H,
               d_ff=wl.d_ff, L=wl.L, dtype=wl.dtype, lens=lens,
               ts=np.ascontiguousarray(ts, dtype=np.int64), norm=None)
    if wl.kind == "attention":
        q = make_qkvu(lens, wl.d, token_rng)
        out["qkvu"] = bf16_round(q) if wl.dtype == "bf16" else q
        out["layers"] = []
    else:
        out["x"] = make_tokens(lens, wl.d, token_rng)
        out["layers"] = make_stack_params(wl.L, wl.d, wl.d_ff, weight_rng, wl.dtype)
    return out


def sweep_expanded(wl: dict) -> dict:
    """The K single-candidate rows [U, S, R, c_i] of a one-user workload.

    Each expanded row repeats the user's U, S and R tokens (features and
    timestamps) and holds one candidate; every row keeps the aggregated user's
    normaliser N = N_U + N_S + N_R + K through the per-user override.
    """
    lens = np.asarray(wl["lens"])
    assert lens.shape[0] == 1
    n_u, n_s, n_r, K = (int(v) for v in lens[0])
    n_ctx = n_u + n_s + n_r
    x, ts = wl["x"], wl["ts"]
    xs, tss = [], []
    for i in range(K):
        xs.append(x[:n_ctx])
        xs.append(x[n_ctx + i:n_ctx + i + 1])
        tss.append(ts[:n_ctx])
        tss.append(ts[n_ctx + i:n_ctx + i + 1])
    out = dict(wl)
    out["lens"] = np.tile(np.array([[n_u, n_s, n_r, 1]], dtype=np.int32), (K, 1))
    out["x"] = np.concatenate(xs, axis=0) if xs else np.zeros((0, x.shape[1]), np.float32)
    out["ts"] = np.concatenate(tss) if tss else np.zeros(0, np.int64)
    out["norm"] = np.full(K, float(n_ctx + K), dtype=np.float32)
    out["kind"] = "sweep_expanded"
    return out


# Input widths of the token MLPs (S, R, candidate): an S or R item is four
# 64-wide field embeddings; a candidate is four item fields and four cross
# fields. The pages give no widths; these are the assumed sizes.
TOKEN_F = (256, 256, 512)
# Hidden width of each task head and the number of tasks (CTR, CTCVR).
HEAD_DH = 256
N_TASKS = 2


def make_token_inputs(lens: np.ndarray, d: int, rng: np.random.Generator,
                      f: tuple = TOKEN_F) -> list:
    """Per-domain inputs [E_U, E_S, E_R, E_C] (float32, bf16-representable):
    E_U [sum N_U, d] and E_g [sum N_g, F_g], N(0, 1), each domain's tokens user
    by user."""
    lens = np.asarray(lens, np.int64).reshape(-1, 4)
    widths = (d,) + tuple(f)
    return [bf16_round(rng.standard_normal((int(lens[:, g].sum()), widths[g]), dtype=np.float32))
            for g in range(4)]


def make_token_params(d: int, rng: np.random.Generator, f: tuple = TOKEN_F) -> dict:
    """Token MLP weights per domain s, r, c: W1 [d, F_g] and W2 [d, d]
    Xavier-uniform (bf16-representable), biases N(0, var 0.01)."""
    p = {}
    for g, fin in zip(("s", "r", "c"), f):
        p["w1_" + g] = bf16_round(_xavier(rng, d, fin))
        p["b1_" + g] = (0.1 * rng.standard_normal(d, dtype=np.float32)).astype(np.float32)
        p["w2_" + g] = bf16_round(_xavier(rng, d, d))
        p["b2_" + g] = (0.1 * rng.standard_normal(d, dtype=np.float32)).astype(np.float32)
    return p


def make_head_params(d: int, rng: np.random.Generator, d_h: int = HEAD_DH,
                     n_tasks: int = N_TASKS) -> dict:
    """Task heads: W1 [n_tasks, d_h, d] Xavier-uniform (bf16-representable),
    b1 N(0, var 0.01), w2 [n_tasks, d_h] Xavier-uniform (fan_out 1), b2
    N(0, var 0.01)."""
    w1 = np.stack([bf16_round(_xavier(rng, d_h, d)) for _ in range(n_tasks)])
    b1 = (0.1 * rng.standard_normal((n_tasks, d_h), dtype=np.float32)).astype(np.float32)
    w2 = np.stack([_xavier(rng, 1, d_h)[0] for _ in range(n_tasks)])
    b2 = (0.1 * rng.standard_normal(n_tasks, dtype=np.float32)).astype(np.float32)
    return dict(w1=w1, b1=b1, w2=w2, b2=b2)

