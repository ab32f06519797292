"""The C ABI from plain C: include/fa2.h compiles as C99 (with warnings as
errors), a C program links against libfa2_b200.so, and the calls that need no
GPU behave as documented (sizes, status strings, argument errors returned
before any launch). Every call here fails its argument checks or is a pure
host function, so nothing reaches a device on any machine."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "exact_tiled_attention_30_b200")

C_SOURCE = r"""
#include <stdio.h>
#include <string.h>
#include "fa2.h"

#define CHECK(cond) do { if (!(cond)) { printf("FAILED %s (line %d)\n", #cond, __LINE__); return 1; } } while (0)

int main(void) {
  void* a = (void*)(size_t)0x10000;  /* aligned, never dereferenced: every call below fails
                                        its argument checks before any device work */
  CHECK(strcmp(fa2_status_string(FA2_OK), "FA2_OK") == 0);
  CHECK(strcmp(fa2_status_string(FA2_ERR_TIMEOUT), "FA2_ERR_TIMEOUT") == 0);
  CHECK(fa2_backward_workspace_size(1, 1, 128, 64) == (size_t)(128 * 64 * 4 + 2 * 128 * 4 + 16));
  CHECK(fa2_backward_workspace_size(1, 1, 128, 96) == 0);
  CHECK(fa2_forward(NULL, a, a, a, (float*)a, 1, 1, 128, 64, 0, 0.125f, NULL) == FA2_ERR_INVALID_ARG);
  CHECK(fa2_forward(a, a, a, a, (float*)a, 1, 1, 128, 80, 0, 0.125f, NULL) == FA2_ERR_UNSUPPORTED);
  CHECK(fa2_forward(a, a, a, a, (float*)a, 0, 1, 128, 64, 0, 0.125f, NULL) == FA2_ERR_INVALID_ARG);
  CHECK(fa2_forward_qk(a, a, a, a, (float*)a, 1, 1, 300, 200, 64, 1, 0.125f, NULL) == FA2_ERR_UNSUPPORTED);
  CHECK(fa2_backward(a, a, a, a, (float*)a, a, a, a, a, 1, 1, 128, 64, 0, 0.125f, a, 16, NULL)
        == FA2_ERR_INVALID_ARG);  /* workspace too small */
  CHECK(fa2_backward_ex(a, a, a, a, (float*)a, a, a, a, a, 1, 1, 128, 64, 0, 0.125f, a,
                        fa2_backward_workspace_size(1, 1, 128, 64), 7, NULL) == FA2_ERR_INVALID_ARG);
  CHECK(fa2_backward_dq_strategy(8, 16, 2048, 128, 1) == FA2_DQ_REDUCE);
  CHECK(fa2_forward_backward_host(a, a, a, a, a, (float*)a, a, a, a, 1, 1, 128, 64, 0, 0.125f, 0,
                                  NULL, 0, NULL) == FA2_ERR_INVALID_ARG);
  printf("ok\n");
  return 0;
}
"""


@pytest.fixture(scope="module")
def library():
    from exact_tiled_attention_30_b200 import build

    return build.build()


def test_header_is_valid_c_and_the_library_links_from_c(library, tmp_path):
    src = tmp_path / "caller.c"
    src.write_text(C_SOURCE)
    exe = tmp_path / "caller"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    f"-I{os.path.join(ROOT, 'include')}", str(src), f"-L{PKG}", "-lfa2_b200",
                    f"-Wl,-rpath,{PKG}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout + out.stderr
