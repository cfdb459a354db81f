"""The C ABI library on the CPU: it loads, exports every entry point the header
declares, and rejects bad arguments on the host before touching a device."""

import ctypes
import os
import re

import numpy as np
import pytest

from generative_recommendation_ranking_b200 import _lib, api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "mtgr.h")).read()
    return sorted(set(re.findall(r"MTGR_API\s+[\w\s\*]+?\b(mtgr_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_lib.LIB_PATH):
        from generative_recommendation_ranking_b200 import build
        build.build()
    return _lib.load()


def test_struct_layouts_match_header(tmp_path):
    # the ctypes mirrors must match the C layouts field for field: compile the
    # header with the host C compiler and compare every offset and size
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "mtgr.h"', 'int main(void) {']
    structs = (("mtgr_batch", _lib.MtgrBatch), ("mtgr_block_params", _lib.MtgrBlockParams),
               ("mtgr_token_mlp", _lib.MtgrTokenMlp), ("mtgr_head_params", _lib.MtgrHeadParams),
               ("mtgr_block_grads", _lib.MtgrBlockGrads))
    for cname, cls in structs:
        lines.append(f'printf("{cname} %zu\\n", sizeof({cname}));')
        for f, _ in cls._fields_:
            lines.append(f'printf("{cname}.{f} %zu\\n", offsetof({cname}, {f}));')
    lines.append('printf("mtgr_work_item %zu\\n", sizeof(mtgr_work_item));')
    lines.append('printf("mtgr_work_item.rt_base %zu\\n", offsetof(mtgr_work_item, rt_base));')
    lines.append("return 0; }")
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = dict(l.split() for l in subprocess.run([str(exe)], capture_output=True, text=True,
                                                  check=True).stdout.splitlines())
    for cname, cls in structs:
        assert int(got[cname]) == ctypes.sizeof(cls), cname
        for f, _ in cls._fields_:
            assert int(got[f"{cname}.{f}"]) == getattr(cls, f).offset, f"{cname}.{f}"
    assert int(got["mtgr_work_item"]) == _lib.WORK_ITEM_BYTES
    assert int(got["mtgr_work_item.rt_base"]) == 56


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
        assert n in _lib._SIGNATURES, f"binding lacks {n}"


def test_status_strings(lib):
    for code in range(8):
        assert _lib.status_string(code) != "unknown status"
    assert _lib.status_string(99) == "unknown status"
    assert lib.mtgr_version() >= 100


def test_host_validation_without_device(lib):
    E = _lib.MTGR_ERR_INVALID_ARG
    assert lib.mtgr_pack_offsets(-1, None, 0, None, None, None, None, None) == E
    assert lib.mtgr_pack_offsets(2, None, 10, None, None, None, None, None) == E
    assert lib.mtgr_build_mask_meta(1, None, None, 1, 1, 1, 1, None, None, None, None, None, None,
                                    None, None, None, None, 0, None, None) == E
    assert lib.mtgr_group_layernorm(4, 12, 0, None, None, 4, None, None, 1e-5, 0, None, None) == E
    assert lib.mtgr_hstu_attention_fwd(None, 64, 2, 0, None, 0, None, None) == E
    assert lib.mtgr_stack_fwd(None, 0, None, None, None, None, 0, None) == E
    assert lib.mtgr_gemm(-1, 2, 64, 1, None, None, None, 0, None, 0, 0, None, None, None) == E
    assert lib.mtgr_restrict_work(None, None, None) == E
    assert lib.mtgr_group_layernorm_pooled(2, None, 64, 0, None, None, None, 1e-5, 0, None, None) == E
    assert lib.mtgr_tokenize(None, 512, None, None, None, None, None, 0, None) == E
    assert lib.mtgr_stack_fwd_candidates(None, 0, None, 0, None, 0, None, None, None, 0, None) == E
    assert lib.mtgr_candidate_heads(None, None, 0, None, None, None, 0, None) == E
    assert lib.mtgr_stack_fwd_rows(None, 0, None, 0, None, 0, None, None, None, 0, None) == E
    # weight-gradient GEMM: sizes, strides, alignment and the status word are
    # checked before any device work (the stand-in addresses are never read)
    f = 0x100000
    wg = lib.mtgr_gemm_wgrad
    assert wg(-1, 32, 64, f, 8, f, 32, f, 0, f, None) == E            # negative M
    assert wg(64, 32, 64, f, 32, f, 32, f, 0, f, None) == E           # lda < M
    assert wg(60, 32, 64, f, 60, f, 32, f, 0, f, None) == E           # lda not a multiple of 8
    assert wg(64, 30, 64, f, 64, f, 32, f, 0, f, None) == E           # N not a multiple of 4
    assert wg(64, 32, 64, f + 2, 64, f, 32, f, 0, f, None) == E       # unaligned a
    assert wg(64, 32, 64, f, 64, f, 32, None, 0, f, None) == E        # no output
    assert wg(64, 32, 64, f, 64, f, 32, f, 0, None, None) == E        # no status word
    assert wg(0, 32, 64, None, 8, None, 32, None, 0, f, None) == _lib.MTGR_OK  # empty output


def _params(d=512, H=8, d_ff=2048, dtype=_lib.MTGR_BF16):
    fake = 0x100000  # 16-byte aligned stand-in addresses; never dereferenced
    return _lib.MtgrBlockParams(d=d, H=H, d_ff=d_ff, dtype=dtype, eps=1e-5, variant=0,
                                gln1_gamma=fake, gln1_beta=fake, gln2_gamma=fake, gln2_beta=fake,
                                w_qkvu=fake, w1=fake, w2=fake, b_qkvu=None, b1=None, b2=None)


def test_workspace_sizes(lib):
    T = 1000
    p = _params()
    want = sum(-(-T * n * 2 // 256) * 256 for n in (512, 2048, 512, 2048))
    assert _lib.mtgr_block_workspace_bytes(T, p) == want
    assert _lib.mtgr_block_workspace_bytes(T, _params(H=4)) == 0        # dh = 128 unsupported
    assert _lib.mtgr_block_workspace_bytes(T, _params(d=100, H=2)) == 0  # d % 64 != 0
    v = _params()
    v.variant = _lib.MTGR_VARIANT_POOLED_GLN | _lib.MTGR_VARIANT_SILU_QKVU
    assert _lib.mtgr_block_workspace_bytes(T, v) == want
    v.variant = 4  # no such flag
    assert _lib.mtgr_block_workspace_bytes(T, v) == 0
    fv = _params(d=64, H=2, d_ff=256, dtype=_lib.MTGR_F32)
    fv.variant = _lib.MTGR_VARIANT_SILU_QKVU  # variants are bf16 only
    assert _lib.mtgr_block_workspace_bytes(T, fv) == 0
    f = _params(d=64, H=2, d_ff=256, dtype=_lib.MTGR_F32)
    assert _lib.mtgr_block_workspace_bytes(T, f) > 0
    two = _lib.mtgr_stack_workspace_bytes(T, [p, p])
    assert two == want + -(-T * 512 * 4 // 256) * 256
    assert _lib.mtgr_stack_workspace_bytes(T, [p]) == want
    assert _lib.mtgr_mask_meta_workspace_bytes(100, 8) == 1024


def test_rows_workspace_sizes(lib):
    # rows [row0, T) of a bf16 stack: GroupLN output and MLP hidden over the
    # k = T - row0 rows, attention output over all T rows, Q|K|V|U in the
    # caller's cache; a spare x buffer of k rows when L > 1
    T, row0 = 1000, 900
    p = _params()
    k = T - row0
    up = lambda n: -(-n // 256) * 256  # noqa: E731
    one = up(k * 512 * 2) + up(T * 512 * 2) + up(k * 2048 * 2)
    assert _lib.mtgr_stack_rows_workspace_bytes(T, row0, [p]) == one
    assert _lib.mtgr_stack_rows_workspace_bytes(T, row0, [p, p, p]) == one + up(k * 512 * 4)
    assert _lib.mtgr_stack_rows_workspace_bytes(T, 0, [p]) == up(T * 512 * 2) * 2 + up(T * 2048 * 2)
    assert _lib.mtgr_stack_rows_workspace_bytes(T, T + 1, [p]) == 0
    assert _lib.mtgr_stack_rows_workspace_bytes(T, -1, [p]) == 0
    f = _params(d=64, H=2, d_ff=256, dtype=_lib.MTGR_F32)
    assert _lib.mtgr_stack_rows_workspace_bytes(T, row0, [f]) == 0  # bf16 only


def test_capacities_host_logic():
    lens = np.array([[4, 32, 8, 8], [16, 300, 50, 100], [0, 0, 0, 0], [0, 60, 10, 0]])
    q, kt, e, rt = api.capacities(lens)
    assert (q, kt, e) == (1 + 4 + 0 + 1, 4, 1 + 16 + 1)
    # R groups: user 0 cols [36, 44) -> 1 group; user 1 [316, 366) -> groups 4, 5;
    # user 3 [60, 70) -> groups 0, 1
    assert rt == 1 * 9 + 2 * 51 + 0 + 2 * 11


def test_token_and_head_workspace_sizes(lib):
    # tokenize: per-domain user offsets 4 (B + 1) int32, the row map T int32,
    # the hidden rows of the largest of S, R, C (d bf16 each)
    up = lambda n: -(-n // 256) * 256  # noqa: E731
    n_rows = [48, 1000, 130, 300]
    B, d = 2, 512
    want = up(4 * (B + 1) * 4) + up(sum(n_rows) * 4) + up(1000 * d * 2)
    assert _lib.mtgr_tokenize_workspace_bytes(B, d, n_rows) == want
    assert _lib.mtgr_tokenize_workspace_bytes(B, 100, n_rows) == 0          # d % 64
    assert _lib.mtgr_tokenize_workspace_bytes(B, d, [1, -1, 0, 0]) == 0    # negative rows
    # heads: offsets, the candidate map, gathered rows (d bf16), hidden rows
    fake = 0x100000
    p = _lib.MtgrHeadParams(d=512, d_h=256, n_tasks=2, reserved=0, w1=fake, b1=None, w2=fake, b2=None)
    want = up(4 * (B + 1) * 4) + up(300 * 4) + up(300 * 512 * 2) + up(300 * 512 * 2)
    assert _lib.mtgr_heads_workspace_bytes(B, 300, p) == want
    p.d_h = 100  # % 32
    assert _lib.mtgr_heads_workspace_bytes(B, 300, p) == 0


def test_candidate_pass_workspace_sizes(lib):
    # offsets 4 (B + 1) int32, candidate map K int32, group ids K int8,
    # GroupLN output K x d bf16, attention output T x d bf16, gathered rows
    # K x d bf16, MLP hidden K x d_ff bf16, spare x K x d fp32 when L > 1
    up = lambda n: -(-n // 256) * 256  # noqa: E731
    B, T, K = 3, 2000, 300
    p = _params()
    one = (up(4 * (B + 1) * 4) + up(K * 4) + up(K) + up(K * 512 * 2) + up(T * 512 * 2)
           + up(K * 512 * 2) + up(K * 2048 * 2))
    assert _lib.mtgr_stack_candidates_workspace_bytes(B, T, K, [p]) == one
    assert _lib.mtgr_stack_candidates_workspace_bytes(B, T, K, [p, p]) == one + up(K * 512 * 4)
    assert _lib.mtgr_stack_candidates_workspace_bytes(B, T, T + 1, [p]) == 0


def test_training_workspace_sizes(lib):
    # saved activations: X~, Q|K|V|U, O/N, G, G~ [T][d..4d] and Z1, H [T][d_ff],
    # each region 256-byte aligned; 2 bytes per element on the bf16 path
    p = _lib.MtgrBlockParams(d=512, H=8, d_ff=2048, dtype=_lib.MTGR_BF16, eps=1e-5, variant=0,
                             gln1_gamma=16, gln1_beta=16, gln2_gamma=16, gln2_beta=16,
                             w_qkvu=16, w1=16, w2=16)
    T = 1000
    al = lambda v: (v + 255) // 256 * 256  # noqa: E731
    want = sum(al(T * c * 2) for c in (512, 4 * 512, 512, 512, 512, 2048, 2048))
    assert _lib.mtgr_block_saved_bytes(T, p) == want
    b = _lib.MtgrBatch(B=2, T=T, q_capacity=9, kt_capacity=5)
    ws = _lib.mtgr_block_bwd_workspace_bytes(T, p, b)
    assert ws >= al(T * 512 * 2) + al(T * 2048 * 2) + al(T * 4 * 512 * 2) + al(10 * 4) + al(45 * 4)
    p.variant = 1
    assert _lib.mtgr_block_saved_bytes(T, p) > 0  # sizes are shape-only; the call itself refuses


def test_training_entry_points_validate_on_the_host(lib):
    p = _lib.MtgrBlockParams(d=512, H=8, d_ff=2048, dtype=_lib.MTGR_BF16, eps=1e-5, variant=2,
                             gln1_gamma=16, gln1_beta=16, gln2_gamma=16, gln2_beta=16,
                             w_qkvu=16, w1=16, w2=16)
    b = _lib.MtgrBatch(B=0, T=0, seg_off=16, user_off=16, ts=16, counts=16, status=16)
    g = _lib.MtgrBlockGrads()
    # a variant block has no backward
    assert lib.mtgr_hstu_block_fwd_train(ctypes.byref(p), ctypes.byref(b), None, None, None, 0,
                                         None) == _lib.MTGR_ERR_UNSUPPORTED
    p.variant = 0
    # missing gradient outputs
    assert lib.mtgr_hstu_block_bwd(ctypes.byref(p), ctypes.byref(b), None, None, None, None,
                                   ctypes.byref(g), None, 0, None) == _lib.MTGR_ERR_INVALID_ARG


def test_host_entry_workspace_and_validation(lib):
    # the host-buffer forward sizes its workspace from the host lengths: the
    # staged inputs, the batch and metadata at api.capacities, the stack's
    # workspace; bad arguments are refused before any device work
    import torch
    p = _lib.MtgrBlockParams(d=512, H=8, d_ff=2048, dtype=_lib.MTGR_BF16, eps=1e-5, variant=0,
                             gln1_gamma=16, gln1_beta=16, gln2_gamma=16, gln2_beta=16,
                             w_qkvu=16, w1=16, w2=16)
    lens = torch.tensor([[24, 300, 20, 32], [24, 1000, 100, 256], [0, 0, 0, 0]], dtype=torch.int32)
    T = int(lens.sum())
    q_cap, kt_cap, e_cap, rt_cap = api.capacities(lens.numpy())
    need = _lib.mtgr_stack_fwd_host_workspace_bytes(lens, [p])
    stack = _lib.mtgr_stack_workspace_bytes(T, [p])
    at_least = T * 512 * 4 * 2 + T * 8 + e_cap * 4 + rt_cap * 8 + q_cap * 64 + stack
    assert at_least <= need <= at_least + 64 * 256 + 8 * T + 4 * T + 64 * q_cap
    bad = torch.tensor([[1, -2, 0, 0]], dtype=torch.int32)
    assert _lib.mtgr_stack_fwd_host_workspace_bytes(bad, [p]) == 0
    st = torch.zeros(1, dtype=torch.int32)
    arr = _lib._layer_array([p])
    assert lib.mtgr_stack_fwd_host(arr, 1, 3, lens.data_ptr(), None, None, None, None,
                                   st.data_ptr(), None, 0, None) == _lib.MTGR_ERR_INVALID_ARG
