"""The C ABI from plain C: a C99 program that includes include/mtgr.h, links
against libmtgr.so and calls its host-side paths (version, status strings,
workspace sizes, argument checks) with no Python and no GPU involved."""

import os
import shutil
import subprocess

import pytest

from generative_recommendation_ranking_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "mtgr.h"

static size_t up(size_t n) { return (n + 255) / 256 * 256; }

int main(void) {
  int fails = 0;
  const void* fake = (const void*)0x100000; /* 16-byte aligned; never dereferenced */
  mtgr_block_params p;
  memset(&p, 0, sizeof p);
  p.d = 512; p.H = 8; p.d_ff = 2048; p.dtype = MTGR_BF16; p.eps = 1e-5f; p.variant = 0;
  p.gln1_gamma = fake; p.gln1_beta = fake; p.gln2_gamma = fake; p.gln2_beta = fake;
  p.w_qkvu = fake; p.w1 = fake; p.w2 = fake;
  if (mtgr_version() < 100) { puts("version"); fails++; }
  if (mtgr_status_string(MTGR_ERR_INVALID_ARG) == NULL ||
      strcmp(mtgr_status_string(MTGR_ERR_INVALID_ARG), mtgr_status_string(MTGR_OK)) == 0) {
    puts("status strings"); fails++;
  }
  /* X~, Q|K|V|U, G, MLP hidden: 2 bytes each, 256-byte aligned regions */
  size_t want = up(1000u * 512 * 2) + up(1000u * 2048 * 2) + up(1000u * 512 * 2) + up(1000u * 2048 * 2);
  if (mtgr_block_workspace_bytes(1000, &p) != want) { puts("block workspace"); fails++; }
  p.variant = 4;
  if (mtgr_block_workspace_bytes(1000, &p) != 0) { puts("unknown variant"); fails++; }
  p.variant = MTGR_VARIANT_SILU_QKVU;
  if (mtgr_block_workspace_bytes(1000, &p) != want) { puts("variant workspace"); fails++; }
  if (mtgr_pack_offsets(-1, NULL, 0, NULL, NULL, NULL, NULL, NULL) != MTGR_ERR_INVALID_ARG) {
    puts("pack args"); fails++;
  }
  if (mtgr_gemm(-1, 2, 64, MTGR_BF16, NULL, NULL, NULL, MTGR_EPI_NONE, NULL, 0, MTGR_F32, NULL,
                NULL, NULL) != MTGR_ERR_INVALID_ARG) {
    puts("gemm args"); fails++;
  }
  const int32_t n_rows[4] = {48, 1000, 130, 300};
  if (mtgr_tokenize_workspace_bytes(2, 512, n_rows) !=
      up(4 * 3 * 4) + up(1478 * 4) + up(1000u * 512 * 2)) {
    puts("tokenize workspace"); fails++;
  }
  if (mtgr_stack_fwd_candidates(NULL, 0, NULL, 0, NULL, 0, NULL, NULL, NULL, 0, NULL) !=
      MTGR_ERR_INVALID_ARG) {
    puts("candidate pass args"); fails++;
  }
  printf("fails %d\n", fails);
  return fails;
}
"""


def test_c_program_links_and_calls_the_library(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    if not os.path.exists(_lib.LIB_PATH):
        from generative_recommendation_ranking_b200 import build
        build.build()
    libdir = os.path.dirname(_lib.LIB_PATH)
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi"
    subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                    "-L", libdir, "-l:libmtgr.so", f"-Wl,-rpath,{libdir}", "-o", str(exe)],
                   check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip().endswith("fails 0")
