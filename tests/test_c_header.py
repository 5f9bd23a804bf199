"""The C boundary from C: a C99 program includes include/gqa_rope_attn.h
(compiled with -Wall -Wextra -Werror -pedantic), links libgqa_rope_attn.so and
calls the entry points that do no CUDA work: workspace sizes, status strings,
the ABI version, and argument rejections of every compute entry point (each
returns its error before any CUDA call). CPU only."""
import os
import shutil
import subprocess

import pytest

from transformer_attention_gqa_b200.build import LIB, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "gqa_rope_attn.h"

#define CHECK(c) do { if (!(c)) { printf("FAILED %s (line %d)\n", #c, __LINE__); return 1; } } while (0)

int main(void) {
  void* a = (void*)(size_t)4096; /* aligned fake address, never dereferenced */
  CHECK(gqa_rope_attn_abi_version() == GQA_ROPE_ATTN_ABI_VERSION);
  CHECK(strcmp(gqa_rope_attn_strerror(GQA_OK), "ok") == 0);
  CHECK(strlen(gqa_rope_attn_strerror(GQA_ERR_TIMEOUT)) > 0);
  CHECK(gqa_rope_attn_workspace_size(1, 8192, 32, 8, 128, GQA_DTYPE_BF16) > 0);
  CHECK(gqa_rope_attn_workspace_size(1, 8192, 32, 8, 96, GQA_DTYPE_BF16) == 0);
  CHECK(gqa_rope_attn_decode_workspace_size(32, 4097, 32, 8, 128) > 0);
  CHECK(gqa_rope_attn_bwd_workspace_size(1, 8192, 32, 8, 128) > 0);
  CHECK(gqa_rope_attn_qkv_proj_workspace_size(8192, 128) > 0);
  /* forward: workspace missing */
  CHECK(gqa_rope_attn_fwd(a, a, a, NULL, 1e4, (const int32_t*)a, 1, 128, 4, 2, 64, 1, GQA_DTYPE_BF16, a, NULL,
                          NULL, 0, NULL) == GQA_ERR_WORKSPACE);
  /* forward: head_dim unsupported */
  CHECK(gqa_rope_attn_fwd(a, a, a, NULL, 1e4, (const int32_t*)a, 1, 128, 4, 2, 80, 1, GQA_DTYPE_BF16, a, NULL,
                          NULL, 0, NULL) == GQA_ERR_UNSUPPORTED);
  /* forward on rotated inputs: workspace missing; group of 256 heads unsupported */
  CHECK(gqa_rope_attn_fwd_rotated(a, a, a, (const int32_t*)a, 1, 128, 4, 2, 64, 1, a, NULL, NULL, 0, NULL) ==
        GQA_ERR_WORKSPACE);
  CHECK(gqa_rope_attn_fwd_rotated(a, a, a, (const int32_t*)a, 1, 128, 256, 1, 64, 1, a, NULL, NULL, 0, NULL) ==
        GQA_ERR_UNSUPPORTED);
  CHECK(gqa_rope_attn_fwd_noalloc(a, a, a, NULL, 1e4, (const int32_t*)a, 1, 1 << 22, 32, 8, 128, 1,
                                  GQA_DTYPE_BF16, a, NULL, NULL) == GQA_ERR_NOALLOC_LIMIT);
  /* decoding step: group of 32 query heads per KV head is unsupported */
  CHECK(gqa_rope_attn_decode(a, a, a, a, a, (const int32_t*)a, 1e4, 4, 100, 64, 2, 64, a, NULL, a, 1 << 20,
                             NULL) == GQA_ERR_UNSUPPORTED);
  /* backward: lse is required */
  CHECK(gqa_rope_attn_bwd(a, a, a, a, NULL, a, NULL, 1e4, (const int32_t*)a, 1, 128, 4, 2, 64, 1, a, a, a, NULL,
                          0, NULL) == GQA_ERR_INVALID_ARG);
  /* projection: hidden not a multiple of 8 */
  CHECK(gqa_rope_attn_qkv_proj(a, a, NULL, 1e4, (const int32_t*)a, 1, 128, 100, 4, 2, 64, a, a, a, NULL, 0,
                               NULL) == GQA_ERR_UNSUPPORTED);
  /* masked forward: mask row stride not a multiple of 8 */
  CHECK(gqa_rope_attn_fwd_masked(a, a, a, NULL, 1e4, (const int32_t*)a, 1, 128, 4, 2, 64, 1, a, 128, 132, a, NULL,
                                 NULL, 0, NULL) == GQA_ERR_INVALID_ARG);
  CHECK(gqa_rope_attn_last_launch_count() == 0);
  gqa_rope_attn_set_profile_events(NULL, NULL, NULL);
  printf("ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_compiles_as_c99_and_links(tmp_path):
    build()
    src = tmp_path / "use_abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "use_abi"
    libdir = os.path.dirname(LIB)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           str(src), "-o", str(exe), "-L", libdir, "-lgqa_rope_attn", "-Wl,-rpath," + libdir]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr
