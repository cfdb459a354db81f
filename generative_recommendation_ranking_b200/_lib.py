"""ctypes binding of libmtgr.so (argument marshalling only).

Every function here has the name of the C entry point it calls and takes
torch tensors (device tensors for the d_* arguments) plus an optional
torch.cuda.Stream. Non-zero host status raises MTGRError. Loading fails loudly
when the shared library is missing: there is no fallback implementation.
"""

from __future__ import annotations

import ctypes
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmtgr.so")

MTGR_OK = 0
MTGR_ERR_INVALID_ARG = 1
MTGR_ERR_CUDA = 2
MTGR_ERR_UNSUPPORTED = 3
MTGR_VARIANT_POOLED_GLN = 1
MTGR_VARIANT_SILU_QKVU = 2
MTGR_VARIANT_RAB = 4
RAB_MAX_DIST = 128
RAB_TIME_BUCKETS = 32
MTGR_ERR_CAPACITY = 4
MTGR_ERR_TIMEOUT = 5
MTGR_ERR_DEVICE_VALIDATION = 6
MTGR_ERR_RANGE = 7

MTGR_F32 = 0
MTGR_BF16 = 1
MTGR_F16 = 2

MTGR_EPI_NONE = 0
MTGR_EPI_SILU = 1
MTGR_EPI_RESID = 2

TILE_M = 128
TILE_N = 128

_TORCH_DTYPE = {MTGR_F32: torch.float32, MTGR_BF16: torch.bfloat16, MTGR_F16: torch.float16}
_MTGR_DTYPE = {v: k for k, v in _TORCH_DTYPE.items()}


class MTGRError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status_string(status)} (status {status})")
        self.status = status


c_i32, c_i64, c_size, c_vp, c_float = (ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t,
                                       ctypes.c_void_p, ctypes.c_float)


class MtgrBatch(ctypes.Structure):
    _fields_ = [("B", c_i32), ("T", c_i32), ("q_capacity", c_i32), ("kt_capacity", c_i32),
                ("seg_off", c_vp), ("user_off", c_vp), ("group_id", c_vp), ("ts", c_vp),
                ("qtile_desc", c_vp), ("row_ptr", c_vp), ("entries", c_vp), ("order", c_vp),
                ("counts", c_vp), ("rt_cnt", c_vp), ("rt_off", c_vp), ("rt_mask", c_vp),
                ("work", c_vp), ("norm", c_vp), ("status", c_vp)]

WORK_ITEM_BYTES = 64  # sizeof(mtgr_work_item)


class MtgrBlockParams(ctypes.Structure):
    _fields_ = [("d", c_i32), ("H", c_i32), ("d_ff", c_i32), ("dtype", c_i32), ("eps", c_float),
                ("variant", c_i32), ("gln1_gamma", c_vp), ("gln1_beta", c_vp),
                ("gln2_gamma", c_vp), ("gln2_beta", c_vp), ("w_qkvu", c_vp), ("w1", c_vp),
                ("w2", c_vp), ("b_qkvu", c_vp), ("b1", c_vp), ("b2", c_vp),
                ("rab_pos", c_vp), ("rab_time", c_vp)]


class MtgrBlockGrads(ctypes.Structure):
    _fields_ = [("gln1_gamma", c_vp), ("gln1_beta", c_vp), ("w_qkvu", c_vp), ("b_qkvu", c_vp),
                ("gln2_gamma", c_vp), ("gln2_beta", c_vp), ("w1", c_vp), ("b1", c_vp),
                ("w2", c_vp), ("b2", c_vp)]


class MtgrTokenMlp(ctypes.Structure):
    _fields_ = [("f", c_i32), ("reserved", c_i32), ("w1", c_vp), ("b1", c_vp), ("w2", c_vp),
                ("b2", c_vp)]


class MtgrHeadParams(ctypes.Structure):
    _fields_ = [("d", c_i32), ("d_h", c_i32), ("n_tasks", c_i32), ("reserved", c_i32),
                ("w1", c_vp), ("b1", c_vp), ("w2", c_vp), ("b2", c_vp)]


_SIGNATURES = {
    "mtgr_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "mtgr_version": (ctypes.c_int, []),
    "mtgr_pack_offsets": (ctypes.c_int, [c_i32, c_vp, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp]),
    "mtgr_mask_meta_workspace_bytes": (c_size, [c_i32, c_i32]),
    "mtgr_build_mask_meta": (ctypes.c_int, [c_i32, c_vp, c_vp, c_i32, c_i32, c_i32, c_i64, c_vp,
                                            c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                                            c_size, c_vp, c_vp]),
    "mtgr_build_mask_meta_static": (ctypes.c_int, [c_i32, c_vp, c_vp, c_i32, c_i32, c_i32, c_i64,
                                                   c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                                                   c_vp, c_vp, c_vp, c_vp]),
    "mtgr_group_layernorm": (ctypes.c_int, [c_i32, c_i32, c_i32, c_vp, c_vp, c_i32, c_vp, c_vp,
                                            c_float, c_i32, c_vp, c_vp]),
    "mtgr_group_layernorm_pooled": (ctypes.c_int, [c_i32, c_vp, c_i32, c_i32, c_vp, c_vp, c_vp,
                                                   c_float, c_i32, c_vp, c_vp]),
    "mtgr_hstu_attention_fwd": (ctypes.c_int, [ctypes.POINTER(MtgrBatch), c_i32, c_i32, c_i32,
                                               c_vp, c_i32, c_vp, c_vp]),
    "mtgr_block_workspace_bytes": (c_size, [c_i32, ctypes.POINTER(MtgrBlockParams)]),
    "mtgr_hstu_block_fwd": (ctypes.c_int, [ctypes.POINTER(MtgrBlockParams),
                                           ctypes.POINTER(MtgrBatch), c_vp, c_vp, c_vp, c_size,
                                           c_vp]),
    "mtgr_stack_workspace_bytes": (c_size, [c_i32, ctypes.POINTER(MtgrBlockParams), c_i32]),
    "mtgr_stack_fwd": (ctypes.c_int, [ctypes.POINTER(MtgrBlockParams), c_i32,
                                      ctypes.POINTER(MtgrBatch), c_vp, c_vp, c_vp, c_size, c_vp]),
    "mtgr_restrict_work": (ctypes.c_int, [ctypes.POINTER(MtgrBatch), c_vp, c_vp]),
    "mtgr_stack_rows_workspace_bytes": (c_size, [c_i32, c_i32, ctypes.POINTER(MtgrBlockParams),
                                                 c_i32]),
    "mtgr_stack_fwd_rows": (ctypes.c_int, [ctypes.POINTER(MtgrBlockParams), c_i32,
                                           ctypes.POINTER(MtgrBatch), c_i32, c_vp, c_i32, c_vp, c_vp,
                                           c_vp, c_size, c_vp]),
    "mtgr_stack_candidates_workspace_bytes": (c_size, [c_i32, c_i32, c_i32,
                                                       ctypes.POINTER(MtgrBlockParams), c_i32]),
    "mtgr_stack_fwd_candidates": (ctypes.c_int, [ctypes.POINTER(MtgrBlockParams), c_i32,
                                                 ctypes.POINTER(MtgrBatch), c_i32, c_vp, c_i32, c_vp,
                                                 c_vp, c_vp, c_size, c_vp]),
    "mtgr_tokenize_workspace_bytes": (c_size, [c_i32, c_i32, ctypes.POINTER(c_i32)]),
    "mtgr_tokenize": (ctypes.c_int, [ctypes.POINTER(MtgrBatch), c_i32, ctypes.POINTER(c_i32),
                                     ctypes.POINTER(c_vp), ctypes.POINTER(MtgrTokenMlp), c_vp, c_vp,
                                     c_size, c_vp]),
    "mtgr_heads_workspace_bytes": (c_size, [c_i32, c_i32, ctypes.POINTER(MtgrHeadParams)]),
    "mtgr_candidate_heads": (ctypes.c_int, [ctypes.POINTER(MtgrHeadParams), ctypes.POINTER(MtgrBatch),
                                            c_i32, c_vp, c_vp, c_vp, c_size, c_vp]),
    "mtgr_gemm": (ctypes.c_int, [c_i32, c_i32, c_i32, c_i32, c_vp, c_vp, c_vp, c_i32, c_vp, c_i32,
                                 c_i32, c_vp, c_vp, c_vp]),
    "mtgr_gemm_wgrad": (ctypes.c_int, [c_i32, c_i32, c_i64, c_vp, c_i64, c_vp, c_i64, c_vp, c_i32,
                                       c_vp, c_vp]),
    "mtgr_timer_create": (c_vp, []),
    "mtgr_timer_destroy": (None, [c_vp]),
    "mtgr_timer_attach": (ctypes.c_int, [c_vp]),
    "mtgr_timer_read": (ctypes.c_int, [c_vp, ctypes.POINTER(ctypes.c_double),
                                       ctypes.POINTER(ctypes.c_int64)]),
    "mtgr_selftest_bounded_wait": (ctypes.c_int, [ctypes.c_uint64, c_vp, c_vp]),
    "mtgr_stack_fwd_host_workspace_bytes": (c_size, [c_i32, c_vp, c_vp, c_i32]),
    "mtgr_stack_fwd_host": (ctypes.c_int, [c_vp, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                                           c_vp, c_size, c_vp]),
    "mtgr_block_saved_bytes": (c_size, [c_i32, ctypes.POINTER(MtgrBlockParams)]),
    "mtgr_hstu_block_fwd_train": (ctypes.c_int, [ctypes.POINTER(MtgrBlockParams),
                                                 ctypes.POINTER(MtgrBatch), c_vp, c_vp, c_vp,
                                                 c_size, c_vp]),
    "mtgr_block_bwd_workspace_bytes": (c_size, [c_i32, ctypes.POINTER(MtgrBlockParams),
                                                ctypes.POINTER(MtgrBatch)]),
    "mtgr_hstu_block_bwd": (ctypes.c_int, [ctypes.POINTER(MtgrBlockParams),
                                           ctypes.POINTER(MtgrBatch), c_vp, c_vp, c_vp, c_vp,
                                           ctypes.POINTER(MtgrBlockGrads), c_vp, c_size, c_vp]),
}

_lib = None


def load() -> ctypes.CDLL:
    """Load libmtgr.so (built in-tree). Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing; build it with "
            "`python -m generative_recommendation_ranking_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().mtgr_status_string(int(status)).decode()


def _ptr(t) -> int | None:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _check(fn: str, rc: int) -> None:
    if rc != MTGR_OK:
        raise MTGRError(fn, rc)


def dtype_code(t: torch.dtype) -> int:
    return _MTGR_DTYPE[t]


def mtgr_version() -> int:
    return load().mtgr_version()


def mtgr_pack_offsets(B, d_lens, T, d_seg_off, d_user_off, d_group_id, d_status, stream=None):
    _check("mtgr_pack_offsets", load().mtgr_pack_offsets(
        B, _ptr(d_lens), T, _ptr(d_seg_off), _ptr(d_user_off), _ptr(d_group_id), _ptr(d_status),
        _stream(stream)))


def mtgr_mask_meta_workspace_bytes(q_capacity: int, kt_capacity: int) -> int:
    return load().mtgr_mask_meta_workspace_bytes(q_capacity, kt_capacity)


def mtgr_build_mask_meta(B, d_seg_off, d_ts, q_capacity, kt_capacity, e_capacity, rt_capacity,
                         d_qtile_desc, d_row_ptr, d_entries, d_order, d_counts, d_rt_cnt, d_rt_off,
                         d_rt_mask, d_work, d_ws, d_status, stream=None):
    ws_bytes = 0 if d_ws is None else d_ws.numel() * d_ws.element_size()
    _check("mtgr_build_mask_meta", load().mtgr_build_mask_meta(
        B, _ptr(d_seg_off), _ptr(d_ts), q_capacity, kt_capacity, e_capacity, rt_capacity,
        _ptr(d_qtile_desc), _ptr(d_row_ptr), _ptr(d_entries), _ptr(d_order), _ptr(d_counts),
        _ptr(d_rt_cnt), _ptr(d_rt_off), _ptr(d_rt_mask), _ptr(d_work), _ptr(d_ws), ws_bytes,
        _ptr(d_status), _stream(stream)))


STATIC_META_SCRATCH_BYTES = 4 << 20


def mtgr_build_mask_meta_static(B, d_seg_off, d_ts, q_capacity, kt_capacity, e_capacity,
                                rt_capacity, d_qtile_desc, d_row_ptr, d_entries, d_order, d_counts,
                                d_rt_cnt, d_rt_off, d_rt_mask, d_work, d_status, stream=None):
    """mtgr_build_mask_meta with the library's fixed scratch instead of a workspace."""
    _check("mtgr_build_mask_meta_static", load().mtgr_build_mask_meta_static(
        B, _ptr(d_seg_off), _ptr(d_ts), q_capacity, kt_capacity, e_capacity, rt_capacity,
        _ptr(d_qtile_desc), _ptr(d_row_ptr), _ptr(d_entries), _ptr(d_order), _ptr(d_counts),
        _ptr(d_rt_cnt), _ptr(d_rt_off), _ptr(d_rt_mask), _ptr(d_work), _ptr(d_status),
        _stream(stream)))


def mtgr_group_layernorm(T, d, d_x, d_group_id, G, d_gamma, d_beta, eps, d_y, stream=None):
    _check("mtgr_group_layernorm", load().mtgr_group_layernorm(
        T, d, dtype_code(d_x.dtype), _ptr(d_x), _ptr(d_group_id), G, _ptr(d_gamma), _ptr(d_beta),
        float(eps), dtype_code(d_y.dtype), _ptr(d_y), _stream(stream)))


def mtgr_group_layernorm_pooled(B, d_seg_off, d, d_x, d_gamma, d_beta, eps, d_y, stream=None):
    _check("mtgr_group_layernorm_pooled", load().mtgr_group_layernorm_pooled(
        B, _ptr(d_seg_off), d, dtype_code(d_x.dtype), _ptr(d_x), _ptr(d_gamma), _ptr(d_beta), eps,
        dtype_code(d_y.dtype), _ptr(d_y), _stream(stream)))


def mtgr_hstu_attention_fwd(batch: MtgrBatch, d, H, d_qkvu, d_g, stream=None):
    _check("mtgr_hstu_attention_fwd", load().mtgr_hstu_attention_fwd(
        ctypes.byref(batch), d, H, dtype_code(d_qkvu.dtype), _ptr(d_qkvu),
        dtype_code(d_g.dtype), _ptr(d_g), _stream(stream)))


def mtgr_block_workspace_bytes(T: int, p: MtgrBlockParams) -> int:
    return load().mtgr_block_workspace_bytes(T, ctypes.byref(p))


def mtgr_hstu_block_fwd(p: MtgrBlockParams, batch: MtgrBatch, d_x_in, d_x_out, d_ws, stream=None):
    _check("mtgr_hstu_block_fwd", load().mtgr_hstu_block_fwd(
        ctypes.byref(p), ctypes.byref(batch), _ptr(d_x_in), _ptr(d_x_out), _ptr(d_ws),
        d_ws.numel() * d_ws.element_size(), _stream(stream)))


def mtgr_stack_workspace_bytes(T: int, layers) -> int:
    arr = (MtgrBlockParams * len(layers))(*layers)
    return load().mtgr_stack_workspace_bytes(T, arr, len(layers))


def mtgr_stack_fwd(layers, batch: MtgrBatch, d_x_in, d_x_out, d_ws, stream=None):
    arr = (MtgrBlockParams * len(layers))(*layers)
    _check("mtgr_stack_fwd", load().mtgr_stack_fwd(
        arr, len(layers), ctypes.byref(batch), _ptr(d_x_in), _ptr(d_x_out), _ptr(d_ws),
        d_ws.numel() * d_ws.element_size(), _stream(stream)))


def mtgr_restrict_work(batch: MtgrBatch, d_q_first, stream=None):
    _check("mtgr_restrict_work", load().mtgr_restrict_work(
        ctypes.byref(batch), _ptr(d_q_first), _stream(stream)))


def mtgr_stack_rows_workspace_bytes(T: int, row0: int, layers) -> int:
    arr = (MtgrBlockParams * len(layers))(*layers)
    return load().mtgr_stack_rows_workspace_bytes(T, row0, arr, len(layers))


def mtgr_stack_fwd_rows(layers, batch: MtgrBatch, row0: int, d_cache, cache_rows: int, d_x_in,
                        d_x_out, d_ws, stream=None):
    arr = (MtgrBlockParams * len(layers))(*layers)
    _check("mtgr_stack_fwd_rows", load().mtgr_stack_fwd_rows(
        arr, len(layers), ctypes.byref(batch), row0, _ptr(d_cache), cache_rows, _ptr(d_x_in),
        _ptr(d_x_out), _ptr(d_ws), d_ws.numel() * d_ws.element_size(), _stream(stream)))


def mtgr_stack_candidates_workspace_bytes(B: int, T: int, k_total: int, layers) -> int:
    arr = (MtgrBlockParams * len(layers))(*layers)
    return load().mtgr_stack_candidates_workspace_bytes(B, T, k_total, arr, len(layers))


def mtgr_stack_fwd_candidates(layers, batch: MtgrBatch, k_total: int, d_cache, cache_rows: int,
                              d_x_cand, d_x_out, d_ws, stream=None):
    arr = (MtgrBlockParams * len(layers))(*layers)
    _check("mtgr_stack_fwd_candidates", load().mtgr_stack_fwd_candidates(
        arr, len(layers), ctypes.byref(batch), k_total, _ptr(d_cache), cache_rows, _ptr(d_x_cand),
        _ptr(d_x_out), _ptr(d_ws), d_ws.numel() * d_ws.element_size(), _stream(stream)))


def mtgr_tokenize_workspace_bytes(B: int, d: int, n_rows) -> int:
    return load().mtgr_tokenize_workspace_bytes(B, d, (c_i32 * 4)(*n_rows))


def mtgr_tokenize(batch: MtgrBatch, d: int, n_rows, d_e, mlps, d_x, d_ws, stream=None):
    """d_e: four device tensors (U, S, R, C inputs; None where a domain has no
    rows); mlps: three MtgrTokenMlp (S, R, C)."""
    _check("mtgr_tokenize", load().mtgr_tokenize(
        ctypes.byref(batch), d, (c_i32 * 4)(*n_rows), (c_vp * 4)(*[_ptr(e) for e in d_e]),
        (MtgrTokenMlp * 3)(*mlps), _ptr(d_x), _ptr(d_ws), d_ws.numel() * d_ws.element_size(),
        _stream(stream)))


def mtgr_heads_workspace_bytes(B: int, k_total: int, p: MtgrHeadParams) -> int:
    return load().mtgr_heads_workspace_bytes(B, k_total, ctypes.byref(p))


def mtgr_candidate_heads(p: MtgrHeadParams, batch: MtgrBatch, k_total: int, d_x, d_out, d_ws,
                         stream=None):
    _check("mtgr_candidate_heads", load().mtgr_candidate_heads(
        ctypes.byref(p), ctypes.byref(batch), k_total, _ptr(d_x), _ptr(d_out), _ptr(d_ws),
        d_ws.numel() * d_ws.element_size(), _stream(stream)))


TIMER_CLASSES = ("pack", "mask_meta", "gln", "gemm_qkvu", "attention", "gemm_mlp1", "gemm_mlp2",
                 "token_mlp", "head_mlp", "rows", "bwd_gemm", "bwd_wgrad", "bwd_attention",
                 "bwd_gln", "bwd_rows")


class Timer:
    """Per-kernel-class CUDA-event timer (mtgr_timer_*). While attached to the
    calling thread, every library launch is bracketed by events and counted."""

    def __init__(self):
        self.h = load().mtgr_timer_create()
        if not self.h:
            raise MemoryError("mtgr_timer_create failed")

    def attach(self):
        load().mtgr_timer_attach(self.h)

    def detach(self):
        load().mtgr_timer_attach(None)

    def read(self) -> dict:
        n = len(TIMER_CLASSES)
        ms = (ctypes.c_double * n)()
        cnt = (ctypes.c_int64 * n)()
        _check("mtgr_timer_read", load().mtgr_timer_read(self.h, ms, cnt))
        return {c: (ms[i], cnt[i]) for i, c in enumerate(TIMER_CLASSES)}

    def __del__(self):
        h, self.h = getattr(self, "h", None), None
        if h and _lib is not None:
            _lib.mtgr_timer_destroy(h)


def mtgr_gemm(d_a, d_b, d_bias, epi, d_resid, q_cols, d_out, d_status, stream=None):
    M, K = d_a.shape
    N = d_b.shape[0]
    _check("mtgr_gemm", load().mtgr_gemm(
        M, N, K, dtype_code(d_a.dtype), _ptr(d_a), _ptr(d_b), _ptr(d_bias), epi, _ptr(d_resid),
        q_cols, dtype_code(d_out.dtype), _ptr(d_out), _ptr(d_status), _stream(stream)))


def mtgr_gemm_wgrad(d_a, d_b, d_out, accumulate, d_status, stream=None):
    T, M = d_a.shape
    N = d_b.shape[1]
    _check("mtgr_gemm_wgrad", load().mtgr_gemm_wgrad(
        M, N, T, _ptr(d_a), d_a.stride(0), _ptr(d_b), d_b.stride(0), _ptr(d_out),
        1 if accumulate else 0, _ptr(d_status), _stream(stream)))


def mtgr_selftest_bounded_wait(limit_ns: int, d_status, stream=None) -> None:
    _check("mtgr_selftest_bounded_wait",
           load().mtgr_selftest_bounded_wait(int(limit_ns), _ptr(d_status), _stream(stream)))


def mtgr_block_saved_bytes(T: int, p: MtgrBlockParams) -> int:
    return load().mtgr_block_saved_bytes(T, ctypes.byref(p))


def mtgr_hstu_block_fwd_train(p: MtgrBlockParams, batch: MtgrBatch, d_x_in, d_x_out, d_saved,
                              stream=None) -> None:
    _check("mtgr_hstu_block_fwd_train", load().mtgr_hstu_block_fwd_train(
        ctypes.byref(p), ctypes.byref(batch), _ptr(d_x_in), _ptr(d_x_out), _ptr(d_saved),
        d_saved.numel() * d_saved.element_size(), _stream(stream)))


def mtgr_block_bwd_workspace_bytes(T: int, p: MtgrBlockParams, batch: MtgrBatch) -> int:
    return load().mtgr_block_bwd_workspace_bytes(T, ctypes.byref(p), ctypes.byref(batch))


def mtgr_hstu_block_bwd(p: MtgrBlockParams, batch: MtgrBatch, d_x_in, d_saved, d_dy, d_dx,
                        grads: MtgrBlockGrads, d_ws, stream=None) -> None:
    _check("mtgr_hstu_block_bwd", load().mtgr_hstu_block_bwd(
        ctypes.byref(p), ctypes.byref(batch), _ptr(d_x_in), _ptr(d_saved), _ptr(d_dy), _ptr(d_dx),
        ctypes.byref(grads), _ptr(d_ws), d_ws.numel() * d_ws.element_size(), _stream(stream)))


def _layer_array(layers):
    arr = (MtgrBlockParams * len(layers))(*layers)
    return arr


def mtgr_stack_fwd_host_workspace_bytes(h_lens, layers) -> int:
    """h_lens: host int32 tensor [B, 4]; layers: MtgrBlockParams list."""
    arr = _layer_array(layers)
    return load().mtgr_stack_fwd_host_workspace_bytes(int(h_lens.shape[0]), _ptr(h_lens), arr,
                                                      len(layers))


def mtgr_stack_fwd_host(layers, h_lens, h_ts, h_norm, h_x_in, h_x_out, h_status, d_ws,
                        stream=None) -> None:
    """Host tensors (pinned) h_lens [B,4] int32, h_ts [T] int64, h_norm [B] float32 or None,
    h_x_in / h_x_out [T, d] float32, h_status [1] int32; d_ws a device workspace."""
    arr = _layer_array(layers)
    _check("mtgr_stack_fwd_host", load().mtgr_stack_fwd_host(
        arr, len(layers), int(h_lens.shape[0]), _ptr(h_lens), _ptr(h_ts), _ptr(h_norm),
        _ptr(h_x_in), _ptr(h_x_out), _ptr(h_status), _ptr(d_ws),
        d_ws.numel() * d_ws.element_size(), _stream(stream)))
