"""The boundary from plain C: a C99 program that includes only include/*.h,
links libentmax_attn.so and calls entry points that need no GPU (sizes, error
strings, argument validation).  This checks that the headers are valid C and
that every call a C caller makes links.
"""

import os
import shutil
import subprocess

import pytest

from differentiable_sparse_attention_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "differentiable_sparse_attention_b200")

C_SOURCE = r"""
#include <stdint.h>
#include <stdio.h>
#include "entmax_attn.h"
#include "dash_route.h"

int main(void) {
  void* fake = (void*)(uintptr_t)(1u << 20);   /* aligned, never dereferenced */
  int failures = 0;
#define CHECK(cond) do { if (!(cond)) { printf("FAIL %s\n", #cond); ++failures; } } while (0)
  CHECK(entmax_attn_mask_words(4096, 128) == 1);
  CHECK(entmax_attn_mask_words(131072, 128) == 32);
  CHECK(entmax_attn_workspace_size(1, 1, 256, 64, 128, 1) > 0);
  CHECK(entmax_attn_workspace_size(1, 1, 0, 64, 128, 1) == 0);
  CHECK(dash_route_workspace_size(1, 4, 2, 256, 64, 16) > 0);
  CHECK(entmax_attn_fwd(NULL, fake, fake, 1, 1, 256, 64, ENTMAX_DTYPE_BF16, 1.5f, 1, 128, 2,
                        fake, (float*)fake, (uint32_t*)fake, NULL, fake, 1u << 30, NULL)
        == ENTMAX_E_NULL);
  CHECK(entmax_attn_fwd(fake, fake, fake, 1, 1, 256, 96, ENTMAX_DTYPE_BF16, 1.5f, 1, 128, 2,
                        fake, (float*)fake, (uint32_t*)fake, NULL, fake, 1u << 30, NULL)
        == ENTMAX_E_UNSUPPORTED);
  CHECK(entmax_attn_bwd(fake, fake, fake, fake, (const float*)fake, (const uint32_t*)fake,
                        1, 1, 256, 64, ENTMAX_DTYPE_BF16, 2.5f, 1, 128, fake, fake, fake,
                        fake, 1u << 30, NULL) == ENTMAX_E_ALPHA);
  CHECK(entmax_attn_fwd_noalloc(fake, fake, fake, 1, 1, 262144, 64, ENTMAX_DTYPE_BF16, 1.5f, 1,
                                128, 2, fake, (float*)fake, (uint32_t*)fake, NULL)
        == ENTMAX_E_SCRATCH);
  CHECK(entmax_attn_noalloc_status(NULL, NULL) == ENTMAX_E_NULL);
  CHECK(dash_route_fwd(fake, fake, 1, 3, 2, 256, 64, 16, 4.0f, 1.5f, 4, (float*)fake,
                       (uint32_t*)fake, (uint32_t*)fake, fake, 1u << 30, NULL) == ENTMAX_E_SHAPE);
  printf("%s\n", entmax_attn_error_string(ENTMAX_E_SCRATCH));
  printf("failures %d\n", failures);
  return failures == 0 ? 0 : 1;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c_program_includes_the_headers_and_links(tmp_path):
    lib = build_mod.build()
    src = tmp_path / "client.c"
    src.write_text(C_SOURCE)
    exe = tmp_path / "client"
    cc = subprocess.run(
        ["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
         str(src), "-o", str(exe), "-L", os.path.dirname(lib), "-lentmax_attn",
         "-Wl,-rpath," + os.path.dirname(lib)],
        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "failures 0" in run.stdout
    assert "8 MiB" in run.stdout
