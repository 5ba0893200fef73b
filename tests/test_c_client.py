"""The boundary from C: a plain C program compiled against include/attn.h and linked to
libattn_b200.so calls the entry points that need no GPU -- status strings, workspace
sizes, the checking-build flag, and argument validation that rejects a call before any
launch -- and prints what it gets (no CUDA header, no torch, no Python in the client).
On a GPU a second client allocates device memory with the CUDA runtime and runs the
causal forward, checked against a plain double-precision restatement in the client."""
import os
import subprocess

import pytest

import __graft_entry__

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "io_aware_exact_26_b200")

CLIENT = r"""
#include <stdio.h>
#include "attn.h"

int main(void) {
  /* statuses and their texts */
  printf("ok=%s\n", attn_status_string(ATTN_OK));
  printf("conflict=%d\n", ATTN_ERR_SCHED_CONFLICT);
  printf("checks=%d\n", attn_checks_enabled());
  /* 8 bytes per query row, rows padded to whole 128-row tiles, 256-byte aligned parts */
  printf("ws=%zu\n", attn_bwd_workspace_size(2, 4, 2, 1000, 128, 1));
  printf("ws_bad=%zu\n", attn_bwd_workspace_size(2, 4, 3, 1000, 128, 1));
  /* rejected before any launch: NULL pointers, unsupported head size, bad GQA split */
  printf("null=%d\n", attn_fwd(NULL, NULL, NULL, NULL, NULL, 1, 2, 1, 128, 128, 0.088f, 1, NULL));
  printf("d96=%d\n", attn_fwd(NULL, NULL, NULL, NULL, NULL, 1, 2, 1, 128, 96, 0.088f, 1, NULL));
  printf("gqa=%d\n", attn_fwd(NULL, NULL, NULL, NULL, NULL, 1, 3, 2, 128, 128, 0.088f, 1, NULL));
  return 0;
}
"""


def test_c_program_links_the_library_and_calls_the_boundary(tmp_path):
    __graft_entry__.build()
    src = tmp_path / "client.c"
    src.write_text(CLIENT)
    exe = tmp_path / "client"
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                           "-L", LIBDIR, "-lattn_b200", f"-Wl,-rpath,{LIBDIR}", "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    got = dict(line.split("=", 1) for line in out.stdout.strip().splitlines())
    assert got["ok"] == "ok"
    assert int(got["conflict"]) == -9
    assert got["checks"] == "0"
    rows = 2 * 4 * 1024                                   # B * Hq * N padded to 1024
    assert int(got["ws"]) == 2 * rows * 4                 # -lse2 and -D, fp32, 256-byte aligned parts
    assert int(got["ws_bad"]) == 0
    assert int(got["null"]) == -1                         # ATTN_ERR_INVALID_ARG
    assert int(got["d96"]) == -2                          # ATTN_ERR_UNSUPPORTED
    assert int(got["gqa"]) == -1


GPU_CLIENT = r"""
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
#include <cuda_runtime_api.h>
#include "attn.h"

enum { B = 1, HQ = 2, HKV = 1, N = 130, D = 64 };

static uint16_t to_bf16(float f) {                 /* round to nearest even */
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}
static float from_bf16(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

int main(void) {
  const size_t nq = (size_t)B * HQ * N * D, nk = (size_t)B * HKV * N * D;
  uint16_t *q = malloc(nq * 2), *k = malloc(nk * 2), *v = malloc(nk * 2), *o = malloc(nq * 2);
  float* lse = malloc(sizeof(float) * B * HQ * N);
  uint32_t s = 12345u;
  for (size_t i = 0; i < nq; ++i) { s = s * 1664525u + 1013904223u; q[i] = to_bf16((float)(s >> 8) / 8388608.f - 1.f); }
  for (size_t i = 0; i < nk; ++i) { s = s * 1664525u + 1013904223u; k[i] = to_bf16((float)(s >> 8) / 8388608.f - 1.f); }
  for (size_t i = 0; i < nk; ++i) { s = s * 1664525u + 1013904223u; v[i] = to_bf16((float)(s >> 8) / 8388608.f - 1.f); }
  void *dq, *dk, *dv, *dout, *dlse;
  if (cudaMalloc(&dq, nq * 2) || cudaMalloc(&dk, nk * 2) || cudaMalloc(&dv, nk * 2) || cudaMalloc(&dout, nq * 2) ||
      cudaMalloc(&dlse, sizeof(float) * B * HQ * N)) { printf("malloc failed\n"); return 1; }
  cudaMemcpy(dq, q, nq * 2, cudaMemcpyHostToDevice);
  cudaMemcpy(dk, k, nk * 2, cudaMemcpyHostToDevice);
  cudaMemcpy(dv, v, nk * 2, cudaMemcpyHostToDevice);
  const float scale = 0.125f;
  int st = attn_fwd(dq, dk, dv, dout, (float*)dlse, B, HQ, HKV, N, D, scale, 1, NULL);
  if (st != ATTN_OK) { printf("attn_fwd: %s\n", attn_status_string(st)); return 1; }
  st = attn_get_device_status(NULL);
  if (st != ATTN_OK) { printf("device: %s\n", attn_status_string(st)); return 1; }
  cudaMemcpy(o, dout, nq * 2, cudaMemcpyDeviceToHost);
  cudaMemcpy(lse, dlse, sizeof(float) * B * HQ * N, cudaMemcpyDeviceToHost);
  /* plain causal attention in double on the same bf16 inputs */
  double err_o = 0, err_l = 0;
  for (int h = 0; h < HQ; ++h)
    for (int i = 0; i < N; ++i) {
      double sc[N], m = -INFINITY, l = 0;
      for (int j = 0; j <= i; ++j) {
        double acc = 0;
        for (int c = 0; c < D; ++c)
          acc += (double)from_bf16(q[((size_t)h * N + i) * D + c]) * from_bf16(k[(size_t)j * D + c]);
        sc[j] = acc * scale;
        if (sc[j] > m) m = sc[j];
      }
      for (int j = 0; j <= i; ++j) l += exp(sc[j] - m);
      for (int c = 0; c < D; ++c) {
        double acc = 0;
        for (int j = 0; j <= i; ++j) acc += exp(sc[j] - m) / l * from_bf16(v[(size_t)j * D + c]);
        double e = fabs(acc - from_bf16(o[((size_t)h * N + i) * D + c]));
        if (e > err_o) err_o = e;
      }
      double e = fabs(m + log(l) - lse[h * N + i]);
      if (e > err_l) err_l = e;
    }
  printf("err_o=%.3g\nerr_lse=%.3g\n", err_o, err_l);
  return 0;
}
"""


@pytest.mark.gpu
def test_c_program_runs_the_forward_on_the_gpu(tmp_path):
    """The same boundary from C on device memory (cudaMalloc'd by the client): the causal
    forward matches a plain double-precision restatement in the client."""
    __graft_entry__.build()
    src = tmp_path / "gpu_client.c"
    src.write_text(GPU_CLIENT)
    exe = tmp_path / "gpu_client"
    cuda = "/usr/local/cuda"
    subprocess.check_call(["gcc", "-std=c99", "-O2", "-Wall", "-I", os.path.join(ROOT, "include"),
                           "-I", os.path.join(cuda, "include"), str(src), "-L", LIBDIR, "-lattn_b200",
                           "-L", os.path.join(cuda, "lib64"), "-lcudart", "-lm",
                           f"-Wl,-rpath,{LIBDIR}", f"-Wl,-rpath,{os.path.join(cuda, 'lib64')}", "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stdout + out.stderr
    got = dict(line.split("=", 1) for line in out.stdout.strip().splitlines())
    assert float(got["err_o"]) < 2e-2          # bf16 O: 1e-2 plus half an ulp of values below 1
    assert float(got["err_lse"]) < 1e-3
