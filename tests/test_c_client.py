"""The boundary from a plain C client: include/kda.h compiled as C11 (-Wall -Werror -pedantic),
linked against libkda.so with no Python or PyTorch in the process.

The client builds the plan for a ragged packed batch, sizes its workspace, checks the status
strings, and drives the host-side argument checks of kda_forward, kda_state_chain and
kda_decode with placeholder device addresses that are never dereferenced (every check named
here runs before any CUDA call).  It runs on a host without a GPU.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "chunked_kda_prefill_b200")
LIB = os.path.join(PKG, "libkda.so")

PROGRAM = r"""
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
#include "kda.h"

#define EXPECT(cond) do { if (!(cond)) { printf("failed: %s (line %d)\n", #cond, __LINE__); \
                                         return 1; } } while (0)

int main(void) {
  /* three packed sequences of 100, 1 and 130 tokens, 2 q/k heads, 4 value heads, D = 128 */
  const int32_t cu[4] = {0, 100, 101, 231};
  kda_shape_t sh;
  memset(&sh, 0, sizeof sh);
  sh.layout = KDA_LAYOUT_TND; sh.B = 3; sh.Nqk = 2; sh.Nv = 4; sh.S = 231; sh.D = 128;

  size_t n = 0;
  EXPECT(kda_plan_size(&sh, &n) == KDA_OK && n > 0);
  int32_t* plan = (int32_t*)calloc(n, sizeof(int32_t));
  EXPECT(kda_plan(&sh, cu, 148, plan, n) == KDA_OK);
  size_t ws = 0;
  EXPECT(kda_workspace_size(plan, n, &ws) == KDA_OK && ws >= 256);

  /* constraints of the problem statement, as status codes */
  const int32_t bad_cu[4] = {0, 100, 100, 231};
  EXPECT(kda_plan(&sh, bad_cu, 148, plan, n) == KDA_ERR_SEQLENS);
  EXPECT(kda_plan(&sh, NULL, 148, plan, n) == KDA_ERR_SEQLENS);
  kda_shape_t heads = sh; heads.Nv = 3;
  EXPECT(kda_plan_size(&heads, &n) == KDA_ERR_HEADS);
  kda_shape_t dim = sh; dim.D = 96;
  EXPECT(kda_plan_size(&dim, &n) == KDA_ERR_DIM);
  EXPECT(kda_plan(&sh, cu, 148, plan, 3) == KDA_ERR_PLAN);
  EXPECT(kda_plan_size(&sh, &n) == KDA_OK);
  EXPECT(kda_plan(&sh, cu, 148, plan, n) == KDA_OK);

  const char* s = kda_status_string(KDA_ERR_LOWER_BOUND);
  EXPECT(s != NULL && strlen(s) > 0);

  /* kda_forward's host checks (placeholder device addresses, 256-byte aligned) */
  const char* base = (const char*)0x10000000;
  const void* q = base; const void* k = base + 0x1000000; const void* v = base + 0x2000000;
  const void* g = base + 0x3000000; const void* beta = base + 0x4000000;
  const float* A_log = (const float*)(base + 0x5000000);
  const float* dt_bias = (const float*)(base + 0x5100000);
  void* work = (void*)(base + 0x6000000);
  void* out = (void*)(base + 0x7000000);
  float* fs = (float*)(base + 0x8000000);
  const int32_t* plan_dev = (const int32_t*)(base + 0x9000000);
  EXPECT(kda_forward(&sh, plan, plan_dev, n, q, k, v, g, beta, 0.088f, NULL, A_log, dt_bias,
                     0.5f, work, ws, out, fs, NULL) == KDA_ERR_LOWER_BOUND);
  EXPECT(kda_forward(&sh, plan, plan_dev, n, NULL, k, v, g, beta, 0.088f, NULL, A_log, dt_bias,
                     -5.0f, work, ws, out, fs, NULL) == KDA_ERR_NULL);
  EXPECT(kda_forward(&sh, plan, plan_dev, n, q, k, v, g, beta, 0.088f, NULL, A_log, dt_bias,
                     -5.0f, work, ws - 1, out, fs, NULL) == KDA_ERR_WORKSPACE);
  EXPECT(kda_forward(&sh, plan, plan_dev, n, (const char*)q + 8, k, v, g, beta, 0.088f, NULL,
                     A_log, dt_bias, -5.0f, work, ws, out, fs, NULL) == KDA_ERR_ALIGN);
  kda_shape_t other = sh; other.S = 232;
  EXPECT(kda_forward(&other, plan, plan_dev, n, q, k, v, g, beta, 0.088f, NULL, A_log, dt_bias,
                     -5.0f, work, ws, out, fs, NULL) != KDA_OK);

  /* kda_state_chain and kda_decode host checks */
  float* S = (float*)(base + 0xA000000);
  EXPECT(kda_state_chain(4, 96, 1, NULL, S, S + 65536, 0, fs, NULL) == KDA_ERR_DIM);
  EXPECT(kda_state_chain(4, 128, 2, NULL, NULL, NULL, 0, fs, NULL) == KDA_ERR_NULL);
  EXPECT(kda_decode(2, 3, 4, 128, q, k, v, g, beta, 0.088f, NULL, A_log, dt_bias, -5.0f, out,
                    fs, NULL) == KDA_ERR_HEADS);
  EXPECT(kda_decode(2, 2, 4, 128, q, k, v, g, beta, 0.088f, NULL, A_log, dt_bias, 1.0f, out,
                    fs, NULL) == KDA_ERR_LOWER_BOUND);
  free(plan);
  printf("ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_client(tmp_path):
    if not os.path.exists(LIB):
        pytest.fail("libkda.so is not built (python -m chunked_kda_prefill_b200.build)")
    src = tmp_path / "client.c"
    exe = tmp_path / "client"
    src.write_text(PROGRAM)
    r = subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic",
                        "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                        "-L", PKG, "-lkda", f"-Wl,-rpath,{PKG}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0 and run.stdout.strip() == "ok", (run.stdout, run.stderr)
