"""include/hq.h is plain C: a C99 program compiles against it with gcc (-std=c99 -pedantic, all
warnings as errors), links libhq.so and runs the host-side argument checks, which return their
documented status before anything touches a device (so no GPU is needed)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "bit_tensor_activation_b200")

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "hq.h"

static int fails = 0;
static void expect(hq_status got, hq_status want, const char* what) {
  if (got != want) {
    printf("FAIL %s: %s, want %s\n", what, hq_status_string(got), hq_status_string(want));
    ++fails;
  }
}

int main(void) {
  /* only the addresses are used: every call below fails its checks first.  The unions with a
     long double give every buffer the 16-byte alignment the checks ask for (C99 has no alignas). */
  static union { uint16_t v[64]; long double a; } ux;
  static union { float v[64]; long double a; } uf;
  static union { int32_t v[16]; long double a; } ui;
  static union { uint8_t v[64]; long double a; } uz;
  static union { uint32_t v[16]; long double a; } uc;
  static union { uint16_t v[16]; long double a; } us;
  uint16_t* x = ux.v;
  float* f = uf.v;
  int32_t* idx = ui.v;
  uint8_t* z = uz.v;
  uint32_t* codes = uc.v;
  uint16_t* side = us.v;
  const uint16_t* odd = (const uint16_t*)((const char*)x + 2);

  expect(hq_calibrate(NULL, 1, 1, 8, 0.9f, 1, f, f, NULL), HQ_ERR_INVALID_ARG, "calibrate x NULL");
  expect(hq_calibrate(x, 0, 1, 8, 0.9f, 1, f, f, NULL), HQ_ERR_INVALID_ARG, "calibrate P = 0");
  expect(hq_calibrate(x, 1, 1, 12, 0.9f, 1, f, f, NULL), HQ_ERR_INVALID_ARG, "calibrate H % 8");
  expect(hq_calibrate(x, 1, 1, 8, 1.0f, 0, f, f, NULL), HQ_ERR_INVALID_ARG, "calibrate beta = 1");
  expect(hq_calibrate(odd, 1, 1, 8, 0.9f, 1, f, f, NULL), HQ_ERR_MISALIGNED, "calibrate x misaligned");
  expect(hq_select_topk(f, f, 65, 8, 0, idx, idx, f, f, z, NULL), HQ_ERR_INVALID_ARG, "select P = 65");
  expect(hq_select_topk(f, f, 1, 8, 4, idx, idx, f, f, z, NULL), HQ_ERR_INVALID_ARG, "select k % 8");
  expect(hq_quantize_pack(x, 1, 1, 8, 16, idx, idx, f, z, codes, side, NULL), HQ_ERR_INVALID_ARG,
         "quantize k > H");
  expect(hq_dequant_reduce(codes, side, 1, 1, 16, 8, idx, idx, f, z, x, (hq_out_dtype)7, NULL),
         HQ_ERR_INVALID_ARG, "dequant bad out dtype");
  expect(hq_dequant_reduce_bf16_shards(codes, side, 1, -1, 16, 8, idx, idx, f, z, x, HQ_OUT_BF16, NULL),
         HQ_ERR_INVALID_ARG, "bf16 shards T < 0");
  expect(hq_compress_reduce(x, 1, 1, 16, 8, idx, idx, f, f, z, (void*)odd, HQ_OUT_BF16, NULL, NULL, NULL),
         HQ_ERR_MISALIGNED, "fused out misaligned");
  expect(hq_selftest_bounded_wait(-1, NULL), HQ_ERR_INVALID_ARG, "self-test negative limit");
  expect(hq_selftest_set_pipeline_stall(1, 0), HQ_ERR_INVALID_ARG, "stall with one bound");
  expect(hq_selftest_set_pipeline_stall(0, 0), HQ_OK, "stall cleared");
  expect(hq_two_step_reduce(x, 2, 3, 16, 8, idx, idx, f, f, z, 8, idx, idx, f, f, z, x, 1 << 20, x, HQ_OUT_BF16, NULL),
         HQ_ERR_INVALID_ARG, "two-step T % P");
  expect(hq_two_step_reduce(x, 2, 4, 16, 8, idx, idx, f, f, z, 8, idx, idx, f, f, z, x, 1, x, HQ_OUT_BF16, NULL),
         HQ_ERR_INVALID_ARG, "two-step workspace too small");
  if (hq_two_step_workspace_bytes(2, 4, 16, 8, 8) == 0 || hq_two_step_workspace_bytes(2, 4, 12, 8, 8) != 0) {
    puts("FAIL two-step workspace bytes");
    ++fails;
  }
  if (hq_wire_bytes_per_row(8192, 256) != (8192 - 256) / 2 + 2 * 256) { puts("FAIL wire bytes"); ++fails; }
  if (hq_wire_bytes_per_row(8, 16) != -1) { puts("FAIL wire bytes k > H"); ++fails; }
  if (strcmp(hq_status_string(HQ_ERR_BAD_INDEX), "HQ_ERR_BAD_INDEX") != 0) { puts("FAIL string"); ++fails; }
  printf("%d failures\n", fails);
  return fails != 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c99_program_against_the_header(tmp_path):
    if not os.path.exists(os.path.join(PKG, "libhq.so")):
        pytest.skip("libhq.so is not built")
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi"
    subprocess.run(["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror",
                    "-I", os.path.join(ROOT, "include"), str(src), "-L", PKG, "-lhq",
                    f"-Wl,-rpath,{PKG}", "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "0 failures" in r.stdout
