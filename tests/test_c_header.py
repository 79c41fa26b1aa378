"""The C ABI from plain C: include/pa.h compiles as strict C99 and a C
program linked against libpa.so drives the host calls (status strings,
workspace size, the block pool with copy-on-write) without Python or a GPU.

The scenario is the shared-prefix copy-on-write of "GPU 学习日报 Day 28"
§六 item 4: sequence 1 holds 20 tokens (one full block and one with 4
tokens), sequence 2 is forked from it, and sequence 2's next token finds
the partly filled last block shared, so that block is copied first.
"""
import os
import shutil
import subprocess

import pytest

from paged_kv_cache_429_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "pa.h"

#define CHECK(c)                                                     \
  do {                                                               \
    if (!(c)) {                                                      \
      fprintf(stderr, "failed: %s (line %d)\n", #c, __LINE__);      \
      return 1;                                                      \
    }                                                                \
  } while (0)

int main(void) {
  int64_t slots[20], pairs[2], ids[2] = {1, 2};
  int32_t tables[2 * 4], ctx[2];
  int ncow = -1;
  pa_pool *pool;

  CHECK(strlen(pa_status_string(PA_OK)) > 0);
  CHECK(strlen(pa_status_string((pa_status)99)) > 0);
  /* 64 x 32 heads x ceil(2048 / 512) partitions x (128 + 2) floats,
     plus 512 bytes of sub-array alignment */
  CHECK(pa_decode_workspace_size(64, 32, 128, 2048, 512) == 4259840u + 512u);
  /* 2 partitions x 130 floats = 1040 bytes + 512, rounded up to 256 */
  CHECK(pa_decode_workspace_size(1, 1, 128, 513, 512) == 1792u);
  CHECK(pa_decode_workspace_size(64, 32, 128, 2048, 0) == 0u);

  CHECK(pa_pool_create(8, 8) == NULL); /* block size must be 16 */
  pool = pa_pool_create(8, 16);
  CHECK(pool != NULL);
  CHECK(pa_pool_add_seq(pool, 1) == PA_OK);
  CHECK(pa_pool_add_seq(pool, 1) == PA_ERR_INVALID_ARG);
  CHECK(pa_pool_append(pool, 1, 20, slots, pairs, &ncow) == PA_OK && ncow == 0);
  CHECK(slots[0] == 0 && slots[15] == 15 && slots[16] == 16 && slots[19] == 19);
  CHECK(pa_pool_fork(pool, 1, 2) == PA_OK);
  CHECK(pa_pool_refcount(pool, 0) == 2 && pa_pool_refcount(pool, 1) == 2);

  /* sequence 2's token 20 goes to the shared, partly filled block 1:
     copy it to a fresh block (2) first, then write slot 4 of the copy */
  CHECK(pa_pool_append(pool, 2, 1, slots, pairs, &ncow) == PA_OK && ncow == 1);
  CHECK(pairs[0] == 1 && pairs[1] == 2);
  CHECK(slots[0] == 2 * 16 + 4);
  CHECK(pa_pool_refcount(pool, 1) == 1 && pa_pool_refcount(pool, 2) == 1);
  CHECK(pa_pool_refcount(pool, 0) == 2);

  CHECK(pa_pool_block_tables(pool, ids, 2, tables, 4, ctx) == PA_OK);
  CHECK(ctx[0] == 20 && ctx[1] == 21);
  CHECK(tables[0] == 0 && tables[1] == 1 && tables[2] == -1 && tables[3] == -1);
  CHECK(tables[4] == 0 && tables[5] == 2 && tables[6] == -1 && tables[7] == -1);
  CHECK(pa_pool_block_tables(pool, ids, 2, tables, 1, ctx) == PA_ERR_INVALID_ARG);
  CHECK(pa_pool_num_free(pool) == 5);

  /* the first sequence leaves: its private block returns, the shared one stays */
  CHECK(pa_pool_free_seq(pool, 1) == PA_OK);
  CHECK(pa_pool_refcount(pool, 0) == 1 && pa_pool_refcount(pool, 1) == 0);
  CHECK(pa_pool_num_free(pool) == 6);
  CHECK(pa_pool_seq_len(pool, 1) == -1 && pa_pool_seq_len(pool, 2) == 21);
  CHECK(pa_pool_seq_num_blocks(pool, 2) == 2);
  pa_pool_destroy(pool);
  printf("c abi ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_uses_the_header_and_library(tmp_path):
    _lib.lib()  # the library is built and loads
    libdir = os.path.dirname(_lib.LIB_PATH)
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
           "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
           "-L", libdir, "-lpa", f"-Wl,-rpath,{libdir}"]
    build = subprocess.run(cmd, capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stderr
    assert run.stdout.strip() == "c abi ok"
