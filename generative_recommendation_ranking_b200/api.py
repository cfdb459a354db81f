"""User-facing API over libmtgr.so: device buffers (through PyTorch) plus calls
into the C ABI. Every step of the forward runs in the library's CUDA kernels;
this module only sizes and allocates buffers and marshals arguments.
"""

from __future__ import annotations

import numpy as np
import torch

from . import _lib
from ._lib import (MTGR_BF16, MTGR_F16, MTGR_F32, MtgrBatch, MtgrBlockParams, TILE_M, TILE_N)

EPS = 1e-5


def capacities(lens: np.ndarray) -> tuple:
    """Host-side buffer sizes of the mask metadata for per-user lengths [B,4]:
    q-tiles, largest per-user k-tile count, an upper bound on tile entries, and
    the rank-table entries (64-column groups holding R keys x (N_R + 1))."""
    lens = np.asarray(lens, dtype=np.int64).reshape(-1, 4)
    n = lens.sum(axis=1)
    nq = (n + TILE_M - 1) // TILE_M
    nk = (n + TILE_N - 1) // TILE_N
    q_cap = int(nq.sum())
    kt_cap = int(nk.max()) if nk.size else 0
    e_cap = int((nq * nk).sum())
    n_us = lens[:, 0] + lens[:, 1]
    c_lo = n_us + lens[:, 2]
    groups = np.where(lens[:, 2] > 0, (c_lo - 1) // 64 - n_us // 64 + 1, 0)
    rt_cap = int((groups * (lens[:, 2] + 1)).sum())
    return q_cap, kt_cap, e_cap, rt_cap


class PackedBatch:
    """A packed batch of users on one device with its mask metadata.

    ``lens`` int [B,4] (N_U, N_S, N_R, K per user; host) and ``ts`` int64 [T]
    (host array or device tensor). ``norm`` optionally overrides each user's
    normaliser N. Runs mtgr_pack_offsets and mtgr_build_mask_meta on
    ``stream``.
    """

    def __init__(self, lens, ts, device="cuda", norm=None, stream=None):
        lens = np.ascontiguousarray(np.asarray(lens, dtype=np.int32).reshape(-1, 4))
        self.lens = lens
        self.B = int(lens.shape[0])
        self.T = int(lens.sum())
        self.device = torch.device(device)
        dev = self.device
        self.q_cap, self.kt_cap, self.e_cap, self.rt_cap = capacities(lens)
        self.d_lens = torch.from_numpy(lens).to(dev, non_blocking=True)
        self.d_ts = (ts if isinstance(ts, torch.Tensor) else torch.from_numpy(
            np.ascontiguousarray(ts, dtype=np.int64))).to(dev, dtype=torch.int64, non_blocking=True)
        i32 = dict(dtype=torch.int32, device=dev)
        self.seg_off = torch.empty(4 * self.B + 1, **i32)
        self.user_off = torch.empty(self.B + 1, **i32)
        self.group_id = torch.empty(max(self.T, 1), dtype=torch.int8, device=dev)
        self.status = torch.zeros(1, **i32)
        self.qtile_desc = torch.empty(max(self.q_cap, 1), 2, **i32)
        self.row_ptr = torch.empty(self.q_cap + 1, **i32)
        self.entries = torch.empty(max(self.e_cap, 1), **i32)
        self.order = torch.empty(max(self.q_cap, 1), **i32)
        self.counts = torch.zeros(4, dtype=torch.int64, device=dev)
        self.rt_cnt = torch.empty(max(self.T, 1), **i32)
        self.rt_off = torch.empty(self.B + 1, dtype=torch.int64, device=dev)
        self.rt_mask = torch.empty(max(self.rt_cap, 1), dtype=torch.int64, device=dev)
        self.work = torch.empty(max(self.q_cap, 1) * _lib.WORK_ITEM_BYTES, dtype=torch.uint8,
                                device=dev)
        ws_bytes = _lib.mtgr_mask_meta_workspace_bytes(self.q_cap, self.kt_cap)
        self.meta_ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
        self.norm = None
        if norm is not None:
            self.norm = torch.as_tensor(np.asarray(norm, dtype=np.float32)).to(dev)
        _lib.mtgr_pack_offsets(self.B, self.d_lens, self.T, self.seg_off, self.user_off,
                               self.group_id, self.status, stream)
        self.build_meta(stream)
        self.c = MtgrBatch(
            B=self.B, T=self.T, q_capacity=self.q_cap, kt_capacity=self.kt_cap,
            seg_off=self.seg_off.data_ptr(), user_off=self.user_off.data_ptr(),
            group_id=self.group_id.data_ptr(), ts=self.d_ts.data_ptr(),
            qtile_desc=self.qtile_desc.data_ptr(), row_ptr=self.row_ptr.data_ptr(),
            entries=self.entries.data_ptr(), order=self.order.data_ptr(),
            counts=self.counts.data_ptr(), rt_cnt=self.rt_cnt.data_ptr(),
            rt_off=self.rt_off.data_ptr(), rt_mask=self.rt_mask.data_ptr(),
            work=self.work.data_ptr(), norm=None if self.norm is None else self.norm.data_ptr(),
            status=self.status.data_ptr())

    def pack(self, stream=None, d_lens=None) -> None:
        """(Re)run mtgr_pack_offsets into this batch's buffers."""
        _lib.mtgr_pack_offsets(self.B, self.d_lens if d_lens is None else d_lens, self.T,
                               self.seg_off, self.user_off, self.group_id, self.status, stream)

    def build_meta(self, stream=None, d_ts=None) -> None:
        """(Re)run mtgr_build_mask_meta into this batch's buffers."""
        _lib.mtgr_build_mask_meta(self.B, self.seg_off, self.d_ts if d_ts is None else d_ts,
                                  self.q_cap, self.kt_cap, self.e_cap, self.rt_cap,
                                  self.qtile_desc, self.row_ptr, self.entries, self.order,
                                  self.counts, self.rt_cnt, self.rt_off, self.rt_mask,
                                  self.work, self.meta_ws, self.status, stream)

    def check(self) -> None:
        """Synchronise and raise if a kernel recorded a device-side error."""
        torch.cuda.synchronize(self.device)
        st = int(self.status.item())
        if st != 0:
            raise _lib.MTGRError("device status", st)

    def meta(self) -> dict:
        """Mask metadata copied to the host (for inspection and tests)."""
        torch.cuda.synchronize(self.device)
        Q, E, V, P = (int(v) for v in self.counts.cpu())
        return dict(
            seg_off=self.seg_off.cpu().numpy(), user_off=self.user_off.cpu().numpy(),
            group_id=self.group_id[:self.T].cpu().numpy(),
            qtile_desc=self.qtile_desc[:Q].cpu().numpy(),
            row_ptr=self.row_ptr[:Q + 1].cpu().numpy(), entries=self.entries[:E].cpu().numpy(),
            order=self.order[:Q].cpu().numpy(), visible_pairs=V, Q=Q, E=E,
            rt_cnt=self.rt_cnt[:self.T].cpu().numpy(), rt_off=self.rt_off.cpu().numpy(),
            rt_mask=self.rt_mask[:self.rt_cap].cpu().numpy().view(np.uint64),
            work=self.work[:P * _lib.WORK_ITEM_BYTES].cpu().numpy().view(np.int32).reshape(P, 16),
            P=P)


class BlockWeights:
    """One HSTU block's parameters on the device (PyTorch Linear layouts).

    ``dtype`` "bf16" keeps W_qkvu, W1, W2 in bf16 (tensor-core path); "f32"
    keeps everything in fp32 (CUDA-core path). GroupLN parameters are fp32.
    ``variant``: 0, or MTGR_VARIANT_* flags (bf16 only): pooled GroupLN
    statistics, SiLU on the Q|K|V|U projections, the relative attention bias
    (tables ``rab_pos`` [H, 2 RAB_MAX_DIST + 1] and ``rab_time``
    [H, RAB_TIME_BUCKETS] in ``p``).
    """

    def __init__(self, p: dict, H: int, dtype: str = "bf16", device="cuda", eps: float = EPS,
                 variant: int = 0):
        dev = torch.device(device)
        wdt = torch.bfloat16 if dtype == "bf16" else torch.float32

        def f32(a):
            return None if a is None else torch.as_tensor(np.asarray(a, np.float32)).to(dev).contiguous()

        def w(a):
            return torch.as_tensor(np.asarray(a, np.float32)).to(dev).to(wdt).contiguous()

        self.t = dict(gln1_gamma=f32(p["gln1_gamma"]), gln1_beta=f32(p["gln1_beta"]),
                      gln2_gamma=f32(p["gln2_gamma"]), gln2_beta=f32(p["gln2_beta"]),
                      w_qkvu=w(p["w_qkvu"]), w1=w(p["w1"]), w2=w(p["w2"]),
                      b_qkvu=f32(p.get("b_qkvu")), b1=f32(p.get("b1")), b2=f32(p.get("b2")),
                      rab_pos=f32(p.get("rab_pos")), rab_time=f32(p.get("rab_time")))
        d = self.t["w_qkvu"].shape[1]
        d_ff = self.t["w1"].shape[0]
        ptr = {k: (None if v is None else v.data_ptr()) for k, v in self.t.items()}
        self.c = MtgrBlockParams(d=d, H=H, d_ff=d_ff,
                                 dtype=MTGR_BF16 if dtype == "bf16" else MTGR_F32, eps=eps,
                                 variant=variant, **ptr)
        self.d, self.H, self.d_ff, self.dtype = d, H, d_ff, dtype


def _ws(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def hstu_block_forward(w: BlockWeights, batch: PackedBatch, x: torch.Tensor, out=None, ws=None,
                       stream=None) -> torch.Tensor:
    """One HSTU block: x [T, d] float32 on the device -> new [T, d] float32."""
    if out is None:
        out = torch.empty_like(x)
    need = _lib.mtgr_block_workspace_bytes(batch.T, w.c)
    if ws is None or ws.numel() < need:
        ws = _ws(need, x.device)
    _lib.mtgr_hstu_block_fwd(w.c, batch.c, x, out, ws, stream)
    return out


GRAD_NAMES = ("gln1_gamma", "gln1_beta", "w_qkvu", "b_qkvu", "gln2_gamma", "gln2_beta", "w1", "b1",
              "w2", "b2")


def hstu_block_forward_train(w: BlockWeights, batch: PackedBatch, x: torch.Tensor, out=None,
                             saved=None, stream=None):
    """One HSTU block forward that keeps what its backward reads. Returns
    (x_out [T, d] float32, saved activations: a uint8 device buffer)."""
    if out is None:
        out = torch.empty_like(x)
    need = _lib.mtgr_block_saved_bytes(batch.T, w.c)
    if saved is None or saved.numel() < need:
        saved = _ws(need, x.device)
    _lib.mtgr_hstu_block_fwd_train(w.c, batch.c, x, out, saved, stream)
    return out, saved


def hstu_block_backward(w: BlockWeights, batch: PackedBatch, x: torch.Tensor, saved: torch.Tensor,
                        dy: torch.Tensor, bias_grads: bool = True, ws=None, stream=None):
    """Gradients of one HSTU block for the upstream gradient dy [T, d]
    (float32): returns (dx [T, d], {parameter name: fp32 gradient}). The
    bias gradients are computed when ``bias_grads`` (the block's biases may be
    absent; their gradients are defined all the same)."""
    dev = x.device
    d, dff = w.d, w.d_ff
    shapes = {"gln1_gamma": (4, d), "gln1_beta": (4, d), "w_qkvu": (4 * d, d), "b_qkvu": (4 * d,),
              "gln2_gamma": (4, d), "gln2_beta": (4, d), "w1": (dff, d), "b1": (dff,),
              "w2": (d, dff), "b2": (d,)}
    grads = {k: torch.empty(v, dtype=torch.float32, device=dev) for k, v in shapes.items()
             if bias_grads or not k.startswith("b")}
    c = _lib.MtgrBlockGrads(**{k: (grads[k].data_ptr() if k in grads else None) for k in GRAD_NAMES})
    dx = torch.empty_like(x)
    need = _lib.mtgr_block_bwd_workspace_bytes(batch.T, w.c, batch.c)
    if ws is None or ws.numel() < need:
        ws = _ws(need, dev)
    _lib.mtgr_hstu_block_bwd(w.c, batch.c, x, saved, dy, dx, c, ws, stream)
    return dx, grads


def stack_workspace(layers, batch: PackedBatch) -> torch.Tensor:
    return _ws(_lib.mtgr_stack_workspace_bytes(batch.T, [l.c for l in layers]), batch.device)


def hstu_stack_forward(layers, batch: PackedBatch, x: torch.Tensor, out=None, ws=None,
                       stream=None) -> torch.Tensor:
    """L stacked HSTU blocks sharing the batch's mask metadata."""
    if out is None:
        out = torch.empty_like(x)
    if ws is None:
        ws = stack_workspace(layers, batch)
    _lib.mtgr_stack_fwd([l.c for l in layers], batch.c, x, out, ws, stream)
    return out


def group_layernorm_pooled(batch: PackedBatch, x: torch.Tensor, gamma: torch.Tensor,
                           beta: torch.Tensor, eps: float = EPS, out_dtype=None, stream=None):
    """GroupLN with one mean and variance per (user, group) segment."""
    y = torch.empty(x.shape, dtype=out_dtype or x.dtype, device=x.device)
    _lib.mtgr_group_layernorm_pooled(batch.B, batch.seg_off, x.shape[1], x, gamma, beta, eps, y,
                                     stream)
    return y


def hstu_attention(batch: PackedBatch, qkvu: torch.Tensor, d: int, H: int,
                   out_dtype=torch.float32, stream=None) -> torch.Tensor:
    """G = (silu(Q K^T) (.) M / N) V (.) U for qkvu [T, 4d] (bf16, f16 or f32)."""
    g = torch.empty(batch.T, d, dtype=out_dtype, device=qkvu.device)
    _lib.mtgr_hstu_attention_fwd(batch.c, d, H, qkvu, g, stream)
    return g


def group_layernorm(x: torch.Tensor, group_id: torch.Tensor, gamma: torch.Tensor,
                    beta: torch.Tensor, eps: float = EPS, out_dtype=None, stream=None):
    T, d = x.shape
    y = torch.empty(T, d, dtype=out_dtype or x.dtype, device=x.device)
    _lib.mtgr_group_layernorm(T, d, x, group_id, gamma.shape[0], gamma, beta, eps, y, stream)
    return y


def gemm(a: torch.Tensor, b: torch.Tensor, bias=None, epi: int = 0, resid=None, q_cols: int = 0,
         out_dtype=torch.float32, status=None, stream=None) -> torch.Tensor:
    """out = epi(a b^T + bias); a [M, K], b [N, K]."""
    out = torch.empty(a.shape[0], b.shape[0], dtype=out_dtype, device=a.device)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=a.device)
    _lib.mtgr_gemm(a, b, bias, epi, resid, q_cols, out, status, stream)
    return out


def gemm_wgrad(a: torch.Tensor, b: torch.Tensor, out=None, status=None, stream=None) -> torch.Tensor:
    """out [M, N] fp32 (+)= a^T b; a [T, M] and b [T, N] bf16, token-major.
    With ``out`` given the sums are added to it, else a zeroed one is made."""
    acc = out is not None
    if out is None:
        out = torch.empty(a.shape[1], b.shape[1], dtype=torch.float32, device=a.device)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=a.device)
    _lib.mtgr_gemm_wgrad(a, b, out, acc, status, stream)
    return out


class ContextCache:
    """One user's context tokens (U, S, R) run once through a bf16 stack, with
    every layer's Q|K|V|U kept on the device, so that the user's candidates
    can then be scored chunk by chunk over the cached keys.

    The context never attends to a candidate and a candidate sees no other
    candidate (fun-rec 7.3.4, mask rules 1-3), so the context rows of every
    layer are the same whichever candidates follow; the MTGR practice
    article (5.2, inference latency) caches the rarely changing User/Seq
    tokens on that ground. ``k_total`` fixes the normaliser N = N_U + N_S +
    N_R + k_total that the aggregated pass over all candidates would use;
    ``max_chunk`` bounds the candidates of one ``score`` call.

    ``x_ctx`` float32 [N_U + N_S + N_R, d] and ``ts_ctx`` int64 (host or
    device) are the context features and timestamps (U tokens' stamps are
    not read). ``out`` holds the stack's output on the context rows.
    """

    def __init__(self, layers, n_u: int, n_s: int, n_r: int, ts_ctx, x_ctx: torch.Tensor,
                 k_total: int, max_chunk: int, stream=None):
        self.layers = list(layers)
        self.c_layers = [l.c for l in self.layers]
        self.n_u, self.n_s, self.n_r = int(n_u), int(n_s), int(n_r)
        self.n_ctx = self.n_u + self.n_s + self.n_r
        self.max_chunk = int(max_chunk)
        self.norm = float(self.n_ctx + int(k_total))
        dev = x_ctx.device
        d = self.layers[0].d
        self.cache_rows = self.n_ctx + self.max_chunk
        self.cache = torch.empty(len(self.layers), self.cache_rows, 4 * d, dtype=torch.float16,
                                 device=dev)
        self.ts_ctx = (ts_ctx if isinstance(ts_ctx, torch.Tensor) else torch.from_numpy(
            np.ascontiguousarray(ts_ctx, dtype=np.int64))).to(dev, dtype=torch.int64)
        self.q_first = torch.tensor([self.n_ctx], dtype=torch.int32, device=dev)
        batch = PackedBatch([[self.n_u, self.n_s, self.n_r, 0]], self.ts_ctx, device=dev,
                            norm=[self.norm], stream=stream)
        self.out = torch.empty_like(x_ctx)
        ws = _ws(_lib.mtgr_stack_rows_workspace_bytes(self.n_ctx, 0, self.c_layers), dev)
        _lib.mtgr_stack_fwd_rows(self.c_layers, batch.c, 0, self.cache, self.cache_rows, x_ctx,
                                 self.out, ws, stream)
        # the context pass's batch and workspace, kept so that the pass can be
        # run again in place (their buffers also stay alive for the stream)
        self.ctx_batch = batch
        self.ctx_ws = ws

    def candidate_batch(self, ts_cand, stream=None) -> PackedBatch:
        """The virtual batch of one chunk: the context followed by the
        chunk's candidates, with the work list cut to the candidate rows."""
        ts_c = (ts_cand if isinstance(ts_cand, torch.Tensor) else torch.from_numpy(
            np.ascontiguousarray(ts_cand, dtype=np.int64))).to(self.cache.device, dtype=torch.int64)
        k = int(ts_c.shape[0])
        if k < 1 or k > self.max_chunk:
            raise ValueError(f"chunk of {k} candidates, 1..{self.max_chunk} allowed")
        batch = PackedBatch([[self.n_u, self.n_s, self.n_r, k]], torch.cat([self.ts_ctx, ts_c]),
                            device=self.cache.device, norm=[self.norm], stream=stream)
        _lib.mtgr_restrict_work(batch.c, self.q_first, stream)
        return batch

    def workspace(self, k: int) -> torch.Tensor:
        return _ws(_lib.mtgr_stack_rows_workspace_bytes(self.n_ctx + k, self.n_ctx, self.c_layers),
                   self.cache.device)

    def score(self, ts_cand, x_cand: torch.Tensor, out=None, ws=None, batch=None,
              stream=None) -> torch.Tensor:
        """Stack output [k, d] float32 of k candidates (features ``x_cand``
        float32 [k, d], timestamps ``ts_cand``), equal to their rows of the
        aggregated pass over the context and all k_total candidates."""
        if batch is None:
            batch = self.candidate_batch(ts_cand, stream)
        k = batch.T - self.n_ctx
        if out is None:
            out = torch.empty(k, x_cand.shape[1], dtype=torch.float32, device=x_cand.device)
        if ws is None:
            ws = self.workspace(k)
        _lib.mtgr_stack_fwd_rows(self.c_layers, batch.c, self.n_ctx, self.cache, self.cache_rows,
                                 x_cand, out, ws, stream)
        return out


class BatchContextCache:
    """The contexts (U, S, R) of a whole batch of users run once through a
    bf16 stack, every layer's Q|K|V|U kept, so that each user's candidates
    can then be scored for the whole batch in one call that computes the
    candidate rows only.

    ``lens`` [B, 4] = (N_U, N_S, N_R, K_b): K_b candidate slots per user, the
    same in every later ``score``; ``ts`` and ``x`` [T, d] float32 are the
    packed timestamps and features of the batch. Their candidate rows may
    hold anything: no context token sees a candidate (fun-rec 7.3.4, mask
    rules 1-3). Each user's normaliser is its length N_U + N_S + N_R + K_b
    (or ``norm``), as in the aggregated pass over the batch. ``out`` holds
    the stack's output on all rows of this context pass.
    """

    def __init__(self, layers, lens, ts, x: torch.Tensor, norm=None, stream=None):
        self.layers = list(layers)
        self.c_layers = [l.c for l in self.layers]
        self.lens = np.ascontiguousarray(np.asarray(lens, dtype=np.int32).reshape(-1, 4))
        self.norm = norm
        dev = x.device
        self.batch = PackedBatch(self.lens, ts, device=dev, norm=norm, stream=stream)
        T, d = self.batch.T, self.layers[0].d
        self.T = T
        self.k_total = int(self.lens[:, 3].sum())
        self.cache = torch.empty(len(self.layers), max(T, 1), 4 * d, dtype=torch.float16, device=dev)
        self.out = torch.empty_like(x)
        ws = _ws(_lib.mtgr_stack_rows_workspace_bytes(T, 0, self.c_layers), dev)
        _lib.mtgr_stack_fwd_rows(self.c_layers, self.batch.c, 0, self.cache, T, x, self.out, ws,
                                 stream)
        self.ctx_ws = ws  # kept for re-running the context pass in place

    def candidate_batch(self, ts, stream=None) -> PackedBatch:
        """The batch of one candidate request: the same lens, with the packed
        timestamps ``ts`` holding the candidates' exposure times."""
        return PackedBatch(self.lens, ts, device=self.cache.device, norm=self.norm, stream=stream)

    def workspace(self) -> torch.Tensor:
        return _ws(_lib.mtgr_stack_candidates_workspace_bytes(self.batch.B, self.T, self.k_total,
                                                              self.c_layers), self.cache.device)

    def score(self, ts, x_cand: torch.Tensor, out=None, ws=None, batch=None,
              stream=None) -> torch.Tensor:
        """Stack output [K_total, d] float32 of the candidates (features
        ``x_cand`` [K_total, d] float32, user by user), equal to their rows
        of the aggregated pass over the batch."""
        if batch is None:
            batch = self.candidate_batch(ts, stream)
        if out is None:
            out = torch.empty(self.k_total, x_cand.shape[1], dtype=torch.float32, device=x_cand.device)
        if ws is None:
            ws = self.workspace()
        _lib.mtgr_stack_fwd_candidates(self.c_layers, batch.c, self.k_total, self.cache, self.T,
                                       x_cand, out, ws, stream)
        return out


class TokenMLPs:
    """The S, R and candidate token MLPs on the device: Linear(F_g, d) ->
    SiLU -> Linear(d, d) per domain, bf16 weights ([out, in]), fp32 biases.
    ``p`` holds ``w1_g``, ``b1_g``, ``w2_g``, ``b2_g`` for g in s, r, c
    (biases may be None)."""

    def __init__(self, p: dict, device="cuda"):
        dev = torch.device(device)
        self.t = {}
        mlps = []
        for g in ("s", "r", "c"):
            w1 = torch.as_tensor(np.asarray(p["w1_" + g], np.float32)).to(dev).to(torch.bfloat16).contiguous()
            w2 = torch.as_tensor(np.asarray(p["w2_" + g], np.float32)).to(dev).to(torch.bfloat16).contiguous()
            b1 = p.get("b1_" + g)
            b2 = p.get("b2_" + g)
            b1 = None if b1 is None else torch.as_tensor(np.asarray(b1, np.float32)).to(dev)
            b2 = None if b2 is None else torch.as_tensor(np.asarray(b2, np.float32)).to(dev)
            self.t[g] = (w1, b1, w2, b2)
            mlps.append(_lib.MtgrTokenMlp(f=w1.shape[1], reserved=0, w1=w1.data_ptr(),
                                          b1=None if b1 is None else b1.data_ptr(), w2=w2.data_ptr(),
                                          b2=None if b2 is None else b2.data_ptr()))
        self.c = mlps
        self.d = self.t["s"][2].shape[0]


def tokenize(mlps: TokenMLPs, batch: PackedBatch, e: list, out=None, ws=None,
             stream=None) -> torch.Tensor:
    """Block input X [T, d] float32 from the per-domain inputs ``e`` = [E_U,
    E_S, E_R, E_C] (bf16 device tensors, each domain's tokens user by user)."""
    d = mlps.d
    n_rows = [int(batch.lens[:, g].sum()) for g in range(4)]
    if out is None:
        out = torch.empty(batch.T, d, dtype=torch.float32, device=batch.device)
    need = _lib.mtgr_tokenize_workspace_bytes(batch.B, d, n_rows)
    if ws is None or ws.numel() < need:
        ws = _ws(need, batch.device)
    _lib.mtgr_tokenize(batch.c, d, n_rows, [t if t is not None and t.numel() else None for t in e],
                       mlps.c, out, ws, stream)
    return out


class CandidateHeads:
    """Task heads (CTR, CTCVR, ...) on the device: per task Linear(d, d_h) ->
    SiLU -> Linear(d_h, 1). ``p``: ``w1`` [n_tasks, d_h, d], ``b1``
    [n_tasks, d_h] or None, ``w2`` [n_tasks, d_h], ``b2`` [n_tasks] or None."""

    def __init__(self, p: dict, device="cuda"):
        dev = torch.device(device)
        w1 = np.asarray(p["w1"], np.float32)
        n_tasks, d_h, d = w1.shape
        self.w1 = torch.as_tensor(w1.reshape(n_tasks * d_h, d)).to(dev).to(torch.bfloat16).contiguous()
        self.b1 = (None if p.get("b1") is None else
                   torch.as_tensor(np.asarray(p["b1"], np.float32).reshape(-1)).to(dev))
        self.w2 = torch.as_tensor(np.asarray(p["w2"], np.float32).reshape(n_tasks, d_h)).to(dev).contiguous()
        self.b2 = (None if p.get("b2") is None else
                   torch.as_tensor(np.asarray(p["b2"], np.float32).reshape(-1)).to(dev))
        self.c = _lib.MtgrHeadParams(d=d, d_h=d_h, n_tasks=n_tasks, reserved=0,
                                     w1=self.w1.data_ptr(),
                                     b1=None if self.b1 is None else self.b1.data_ptr(),
                                     w2=self.w2.data_ptr(),
                                     b2=None if self.b2 is None else self.b2.data_ptr())
        self.n_tasks = n_tasks


def candidate_heads(heads: CandidateHeads, batch: PackedBatch, x: torch.Tensor, out=None, ws=None,
                    stream=None) -> torch.Tensor:
    """Logits [K_total, n_tasks] float32 of the batch's candidates (user by
    user) from the stack output x [T, d] float32."""
    k_total = int(batch.lens[:, 3].sum())
    if out is None:
        out = torch.empty(k_total, heads.n_tasks, dtype=torch.float32, device=x.device)
    need = _lib.mtgr_heads_workspace_bytes(batch.B, k_total, heads.c)
    if ws is None or ws.numel() < need:
        ws = _ws(need, x.device)
    _lib.mtgr_candidate_heads(heads.c, batch.c, k_total, x, out, ws, stream)
    return out
