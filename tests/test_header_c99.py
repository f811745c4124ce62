"""include/ckv.h is a C ABI: it compiles as strict C99 and C++17 on its own, and a plain C program
can link against libckv.so and call a host-only entry point (no GPU needed)."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
LIBDIR = os.path.join(ROOT, "compressed_kv_sparse_compress_b200")

C_SRC = r"""
#include "ckv.h"
#include <stdio.h>
int main(void) {
  ckv_pool* pool = 0;
  int32_t ids[3];
  ckv_layer_cfg cfg = {64, 512, 64, 4, 128, CKV_BF16, CKV_FP8_E4M3, 0.0f, 0.0f};
  ckv_index_cfg icfg = {64, 128};
  size_t comp = 0, cs = 0, win = 0, ws = 0;
  if (kv_block_pool_create(8, &pool) != CKV_OK) return 1;
  if (kv_block_alloc(pool, 3, ids) != CKV_OK || ids[0] != 0 || ids[2] != 2) return 2;
  if (kv_block_free(pool, ids, 3) != CKV_OK || kv_block_pool_num_free(pool) != 8) return 3;
  kv_block_pool_destroy(pool);
  if (ckv_cache_row_bytes(&cfg, &comp, &cs, &win, &ws) != CKV_OK || comp != 1024 || win != 512) return 4;
  if (ckv_mh_indexer_workspace_bytes(&cfg, &icfg, 8, 32768, 512) == 0) return 5;
  printf("%s\n", ckv_status_str(CKV_ERR_WORKSPACE));
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_header_is_c99_and_a_c_program_links_and_runs(tmp_path):
    src = tmp_path / "use_ckv.c"
    src.write_text(C_SRC)
    exe = tmp_path / "use_ckv"
    lib = os.path.join(LIBDIR, "libckv.so")
    assert os.path.exists(lib), "build libckv.so first"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", INCLUDE, str(src),
                    "-L", LIBDIR, "-lckv", f"-Wl,-rpath,{LIBDIR}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.returncode
    assert out.stdout.strip() == "workspace too small"


@pytest.mark.skipif(shutil.which("g++") is None, reason="g++ not installed")
def test_header_compiles_as_cpp(tmp_path):
    src = tmp_path / "use_ckv.cpp"
    src.write_text('#include "ckv.h"\nint f() { return CKV_OK; }\n')
    subprocess.run(["g++", "-std=c++17", "-Wall", "-Werror", "-c", "-I", INCLUDE, str(src), "-o",
                    str(tmp_path / "use_ckv.o")], check=True)
