"""The boundary from plain C (CPU only): a C99 program includes include/rz.h, links librz.so
and calls host-only paths (status names, workspace queries, argument checks that return
before any CUDA call).  Shows the header is valid C, with no C++ or torch types, and that the
exported names link as declared."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "rz.h"

#define CHECK(cond) do { if (!(cond)) { printf("FAIL line %d: %s\n", __LINE__, #cond); return 1; } } while (0)

int main(void) {
  CHECK(strcmp(rz_status_string(RZ_OK), "RZ_OK") == 0);
  CHECK(strcmp(rz_status_string(RZ_ERR_WORKSPACE_TOO_SMALL), "RZ_ERR_WORKSPACE_TOO_SMALL") == 0);
  CHECK(rz_workspace_bytes_logprobs(1000, 256, 4096) > 0);
  CHECK(rz_workspace_bytes_logprobs(10, 100, 4096) == 0);
  CHECK(rz_workspace_bytes_loss(1000, 8, 2, 256, 4096) > rz_workspace_bytes_logprobs(1000, 256, 4096));
  CHECK(rz_workspace_bytes_segment_loss(1000, 8, 2) > 0);
  CHECK(rz_workspace_bytes_ratio_stats(1000, 8) > 0);
  CHECK(rz_workspace_bytes_grad_norms() > 0);
  CHECK(rz_num_launches_loss(16385) == 13);

  /* argument errors return before anything is enqueued; no pointer is dereferenced */
  const rz_bf16* H = (const rz_bf16*)(size_t)256;
  const rz_bf16* W = (const rz_bf16*)(size_t)512;
  const int32_t* ids = (const int32_t*)(size_t)1024;
  float* lp = (float*)(size_t)2048;
  void* ws = (void*)(size_t)(1 << 20);
  CHECK(rz_token_logprobs(H, W, ids, 100, 100, 4096, lp, NULL, ws, (size_t)1 << 40, NULL)
        == RZ_ERR_UNSUPPORTED_SHAPE);
  CHECK(rz_token_logprobs(NULL, W, ids, 100, 256, 4096, lp, NULL, ws, (size_t)1 << 40, NULL) == RZ_ERR_INVALID_ARG);
  CHECK(rz_token_logprobs(H, W, ids, 100, 256, 4096, lp, NULL, ws, 1024, NULL) == RZ_ERR_WORKSPACE_TOO_SMALL);
  CHECK(rz_token_logprobs(NULL, NULL, NULL, 0, 256, 4096, NULL, NULL, NULL, 0, NULL) == RZ_OK);

  rz_loss_options o;
  memset(&o, 0, sizeof o);
  o.flags = RZ_LOSS_CLIP_IS;
  o.clip_max = 0.0f; /* must be > 0 */
  CHECK(rz_segment_loss_ex((const float*)(size_t)256, (const float*)(size_t)512, (const float*)(size_t)768,
                           (const int64_t*)(size_t)1024, (const int32_t*)(size_t)1280, 10, 2, 1, &o,
                           (float*)(size_t)1536, (float*)(size_t)1792, NULL, ws, (size_t)1 << 40, NULL)
        == RZ_ERR_INVALID_ARG);
  CHECK(rz_read_device_status(NULL, NULL, NULL) == RZ_ERR_INVALID_ARG);
  CHECK(RZ_NOALLOC_SCRATCH_BYTES == (32u << 20));
  printf("ok\n");
  return 0;
}
"""


@pytest.fixture(scope="module")
def lib_path():
    from invariant_logprobs_reinforce_b200 import build
    return build.build()


def test_header_compiles_as_c99_and_links(tmp_path, lib_path):
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi"
    libdir = os.path.dirname(lib_path)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), lib_path, f"-Wl,-rpath,{libdir}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
