/*
 * abi_consumer.c -- a plain C consumer of libconv3d's C ABI (include/conv3d.h).
 *
 *   abi_consumer cpu   argument validation, shapes, workspace sizes and status
 *                      strings (no GPU needed: validation precedes any CUDA call)
 *   abi_consumer gpu   a centre-delta 3x3x3 convolution on the current device:
 *                      w[co][it][ih][iw][ci] = (it,ih,iw) == (kt-1,1,1) && co == ci,
 *                      causal replicate padding, so y = round(x + bias) exactly
 *                      (one nonzero product per output); checked element by
 *                      element against that value computed here.
 * Exit status 0 on success; prints the first failure otherwise.
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "conv3d.h"

#ifdef ABI_CONSUMER_GPU
#include <cuda_runtime.h>
#endif

static int failures = 0;
#define CHECK(cond)                                                      \
  do {                                                                   \
    if (!(cond)) {                                                       \
      fprintf(stderr, "%s:%d: check failed: %s\n", __FILE__, __LINE__, #cond); \
      ++failures;                                                        \
    }                                                                    \
  } while (0)

static int cpu_checks(void) {
  const int k3[3] = {3, 3, 3}, s1[3] = {1, 1, 1}, s2[3] = {1, 2, 2}, st2[3] = {2, 2, 2};
  const int p_causal[3] = {0, 1, 1}, p_zero[3] = {1, 1, 1};
  int out[3];
  CHECK(conv3d_output_shape(9, 128, 128, k3, s1, p_causal, CONV3D_TPAD_CAUSAL_REPLICATE, out) ==
        CONV3D_OK);
  CHECK(out[0] == 9 && out[1] == 128 && out[2] == 128);
  CHECK(conv3d_output_shape(9, 128, 128, k3, s2, p_causal, CONV3D_TPAD_CAUSAL_ZERO, out) ==
        CONV3D_OK);
  CHECK(out[0] == 9 && out[1] == 64 && out[2] == 64);
  CHECK(conv3d_output_shape(5, 32, 32, k3, s1, p_zero, CONV3D_TPAD_ZERO, out) == CONV3D_OK);
  CHECK(out[0] == 5);
  CHECK(conv3d_workspace_bytes(256, 256, k3, 1, CONV3D_TPAD_CAUSAL_REPLICATE) ==
        (size_t)2 * 256 * 9 * 256 * 2);
  CHECK(conv3d_workspace_bytes(256, 256, k3, 9, CONV3D_TPAD_CAUSAL_REPLICATE) == 0);
  CHECK(strcmp(conv3d_status_string(CONV3D_OK), "ok") == 0);
  /* fake, never dereferenced device addresses */
  const void* x = (const void*)0x100000000ull;
  const void* w = (const void*)0x200000000ull;
  void* y = (void*)0x300000000ull;
  CHECK(conv3d_fwd(NULL, w, NULL, NULL, y, 1, 64, 4, 8, 8, 64, k3, s1, p_causal,
                   CONV3D_TPAD_CAUSAL_REPLICATE, CONV3D_BF16, NULL) == CONV3D_ERR_INVALID_ARG);
  CHECK(conv3d_fwd(x, w, NULL, NULL, y, 1, 12, 4, 8, 8, 64, k3, s1, p_causal,
                   CONV3D_TPAD_CAUSAL_REPLICATE, CONV3D_BF16, NULL) == CONV3D_ERR_UNSUPPORTED);
  CHECK(conv3d_fwd((const char*)x + 2, w, NULL, NULL, y, 1, 64, 4, 8, 8, 64, k3, s1, p_causal,
                   CONV3D_TPAD_CAUSAL_REPLICATE, CONV3D_BF16, NULL) == CONV3D_ERR_ALIGNMENT);
  CHECK(conv3d_fwd_cached(x, NULL, w, NULL, NULL, y, 1, 64, 4, 8, 8, 64, k3, s1, p_causal,
                          CONV3D_BF16, NULL) == CONV3D_ERR_INVALID_ARG);
  CHECK(strlen(conv3d_last_error()) > 0);
  CHECK(conv3d_kernel_launches() == 0);   /* rejected calls launch nothing */

  /* backward entry points: workspace sizes and argument errors */
  void* ws = (void*)0x400000000ull;
  void* dx = (void*)0x500000000ull;
  CHECK(conv3d_bwd_weight_workspace_bytes(64, 64, k3) >=
        (size_t)64 * 27 * 64 * 4 + (size_t)64 * 4);
  CHECK(conv3d_bwd_data_workspace_bytes(1, 64, 4, 8, 8, 64, k3, p_zero, CONV3D_TPAD_ZERO) ==
        (size_t)64 * 27 * 64 * 2 + (size_t)160 * (128 * 256 * 4 + 64));
  CHECK(conv3d_bwd_data(y, w, dx, 1, 64, 4, 8, 8, 64, k3, st2, p_causal,
                        CONV3D_TPAD_CAUSAL_REPLICATE, CONV3D_BF16, ws, (size_t)1 << 30,
                        NULL) == CONV3D_ERR_UNSUPPORTED);          /* stride 2 */
  CHECK(conv3d_bwd_data(y, w, dx, 1, 64, 4, 8, 8, 64, k3, s1, p_causal,
                        CONV3D_TPAD_CAUSAL_REPLICATE, CONV3D_BF16, NULL, 0, NULL) ==
        CONV3D_ERR_WORKSPACE);
  CHECK(conv3d_bwd_weight(x, y, NULL, NULL, 1, 64, 4, 8, 8, 64, k3, s1, p_causal,
                          CONV3D_TPAD_CAUSAL_REPLICATE, CONV3D_BF16, ws, (size_t)1 << 30,
                          NULL) == CONV3D_ERR_INVALID_ARG);        /* dw missing */
  CHECK(conv3d_bwd_weight(x, y, dx, NULL, 1, 64, 4, 8, 8, 64, k3, s1, p_causal,
                          CONV3D_TPAD_CAUSAL_CACHED, CONV3D_BF16, ws, (size_t)1 << 30,
                          NULL) == CONV3D_ERR_UNSUPPORTED);

  /* GroupNorm entry points: argument errors */
  double* stats = (double*)0x600000000ull;
  CHECK(conv3d_groupnorm_stats(x, 1, 2, 4, 4, 64, 7, 0, 1e-6f, CONV3D_BF16, stats, NULL) ==
        CONV3D_ERR_INVALID_ARG);                                   /* C % groups */
  CHECK(conv3d_groupnorm_silu(x, stats, NULL, NULL, (char*)y + 2, 1, 2, 4, 4, 64, 8, 0, 1,
                              CONV3D_BF16, NULL) == CONV3D_ERR_ALIGNMENT);
  return failures;
}

#ifdef ABI_CONSUMER_GPU
static uint16_t f32_to_bf16(float f) { /* round to nearest even (finite inputs) */
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}
static float bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

static int gpu_checks(void) {
  const int N = 1, C = 64, D = 3, H = 10, W = 12;
  const int k3[3] = {3, 3, 3}, s1[3] = {1, 1, 1}, pad[3] = {0, 1, 1};
  const size_t nx = (size_t)N * D * H * W * C, nw = (size_t)C * 27 * C;
  uint16_t* hx = malloc(nx * 2);
  uint16_t* hw = calloc(nw, 2);
  uint16_t* hb = malloc(C * 2);
  uint16_t* hy = malloc(nx * 2);
  uint32_t s = 12345u;
  for (size_t i = 0; i < nx; ++i) {
    s = s * 1664525u + 1013904223u;
    hx[i] = f32_to_bf16(((int)(s >> 9) % 2001 - 1000) / 256.0f);
  }
  for (int c = 0; c < C; ++c) hb[c] = f32_to_bf16((c % 7 - 3) / 8.0f);
  for (int c = 0; c < C; ++c) /* tap (kt-1, 1, 1) reads frame `to` at the same pixel */
    hw[(((size_t)c * 3 + 2) * 3 * 3 + 1 * 3 + 1) * C + c] = f32_to_bf16(1.0f);
  void *dx, *dw, *db, *dy;
  CHECK(cudaMalloc(&dx, nx * 2) == cudaSuccess && cudaMalloc(&dw, nw * 2) == cudaSuccess &&
        cudaMalloc(&db, C * 2) == cudaSuccess && cudaMalloc(&dy, nx * 2) == cudaSuccess);
  if (failures) return failures;
  cudaMemcpy(dx, hx, nx * 2, cudaMemcpyHostToDevice);
  cudaMemcpy(dw, hw, nw * 2, cudaMemcpyHostToDevice);
  cudaMemcpy(db, hb, C * 2, cudaMemcpyHostToDevice);
  CHECK(conv3d_fwd(dx, dw, db, NULL, dy, N, C, D, H, W, C, k3, s1, pad,
                   CONV3D_TPAD_CAUSAL_REPLICATE, CONV3D_BF16, NULL) == CONV3D_OK);
  CHECK(conv3d_poll_status(NULL) == CONV3D_OK);
  cudaMemcpy(hy, dy, nx * 2, cudaMemcpyDeviceToHost);
  size_t bad = 0;
  for (size_t i = 0; i < nx; ++i) {
    const uint16_t expect = f32_to_bf16(bf16_to_f32(hx[i]) + bf16_to_f32(hb[i % C]));
    if (hy[i] != expect && bad++ < 5)
      fprintf(stderr, "y[%zu] = 0x%04x, expected 0x%04x\n", i, hy[i], expect);
  }
  CHECK(bad == 0);
  cudaFree(dx); cudaFree(dw); cudaFree(db); cudaFree(dy);
  free(hx); free(hw); free(hb); free(hy);
  conv3d_release();
  return failures;
}
#endif

int main(int argc, char** argv) {
  const char* mode = argc > 1 ? argv[1] : "cpu";
  int rc = 0;
  if (strcmp(mode, "cpu") == 0) rc = cpu_checks();
#ifdef ABI_CONSUMER_GPU
  else if (strcmp(mode, "gpu") == 0) rc = cpu_checks() + gpu_checks();
#endif
  else {
    fprintf(stderr, "unknown mode %s\n", mode);
    return 2;
  }
  if (rc == 0) printf("abi_consumer %s: ok\n", mode);
  return rc == 0 ? 0 : 1;
}
