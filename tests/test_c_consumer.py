"""The C ABI from plain C (no Python, no torch): include/qsa.h compiles as C11
with -Wall -Wextra -Werror, a C program links against libqsa.so, and the
host-side paths answer as the header documents (version, status strings,
workspace sizes, host-checked errors before anything is enqueued, empty
batches as no-ops).  Runs on the CPU: none of these calls touch the device.
"""
import os
import subprocess
import tempfile

import pytest

import block_sparse_attention_22_b200 as qsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "qsa.h"

#define CHECK(cond) do { if (!(cond)) { printf("FAIL line %d: %s\n", __LINE__, #cond); return 1; } } while (0)

int main(void) {
  qsa_config_t cfg;
  memset(&cfg, 0, sizeof cfg);
  cfg.r = 4; cfg.budget_tokens = 2048; cfg.n_q_heads = 24; cfg.n_kv_groups = 2;
  cfg.head_dim = 256; cfg.idx_heads = 4; cfg.idx_dim = 128; cfg.rope_fraction = 0.25f;
  cfg.rope_base = 1e7; cfg.dtype = QSA_DTYPE_BF16;
  CHECK(qsa_version() >= 100);
  CHECK(strlen(qsa_status_string(QSA_ERR_WORKSPACE)) > 0);

  qsa_segment_t seg = {0, 131072, 0, 0};
  size_t fwd = qsa_workspace_size(&cfg, &seg, 1, 131072, QSA_OP_FORWARD);
  size_t low = qsa_workspace_size(&cfg, &seg, 1, 131072, QSA_OP_FORWARD_LOWMEM);
  size_t uni = qsa_workspace_size(&cfg, &seg, 1, 131072, QSA_OP_ATTN_UNION);
  CHECK(fwd != (size_t)-1 && low != (size_t)-1 && uni != (size_t)-1);
  CHECK(fwd >= (size_t)131072 * 32767 * 4);       /* the score rows */
  CHECK(low < fwd);
  CHECK(uni >= (size_t)13108 * 2 * 10 * 512 * 4);   /* 10-query tiles: blocks + masks */

  /* host-checked errors return before anything is enqueued (fake aligned pointers) */
  void* p = (void*)(uintptr_t)256;
  qsa_cache_t cache = {p, p, p, p, 1, 1024};
  qsa_segment_t small = {0, 16, 100, 0};
  qsa_config_t bad = cfg;
  bad.head_dim = 128;
  CHECK(qsa_forward(&bad, &cache, &small, 1, 16, p, p, p, p, NULL, NULL, NULL, p, (size_t)1 << 40, NULL)
        == QSA_ERR_UNSUPPORTED);
  bad = cfg;
  bad.budget_tokens = 2047;
  CHECK(qsa_forward(&bad, &cache, &small, 1, 16, p, p, p, p, NULL, NULL, NULL, p, (size_t)1 << 40, NULL)
        == QSA_ERR_INVALID_ARG);
  CHECK(qsa_forward(&cfg, &cache, &small, 1, 16, p, p, p, p, NULL, NULL, NULL, p, 10, NULL)
        == QSA_ERR_WORKSPACE);
  CHECK(qsa_sparse_attn_fwd_union(&cfg, &cache, &small, 1, 16, p, p, p, p, NULL, p, 10, NULL)
        == QSA_ERR_WORKSPACE);
  qsa_segment_t empty = {0, 0, 100, 0};
  CHECK(qsa_forward(&cfg, &cache, &empty, 1, 0, p, p, p, p, NULL, NULL, NULL, NULL, 0, NULL) == QSA_OK);
  printf("ok\n");
  return 0;
}
"""


def test_c_program_links_and_gets_host_answers():
    lib_dir = os.path.dirname(qsa.LIB_PATH)
    if not os.path.exists(qsa.LIB_PATH):
        pytest.fail("libqsa.so is not built")
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "consumer.c")
        exe = os.path.join(d, "consumer")
        with open(src, "w") as f:
            f.write(PROGRAM)
        subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), src,
                        "-L", lib_dir, "-lqsa", "-Wl,-rpath," + lib_dir, "-o", exe], check=True,
                       capture_output=True, text=True)
        r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
        assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
