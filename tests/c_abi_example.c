/* A plain C host of the streaming LM-head loss: no Python and no torch, only the C ABI of
 * libslm.so (include/slm.h) and the CUDA runtime for memory.
 *
 * With W = 0 every logit is 0, so for hard-label cross entropy ("Streaming Cross
 * Entropy"): every valid row's loss is log V; dH = dZ W = 0; and
 *   dW[v] = sum_n g_n (1/V - [v = y_n]) H[n],   g_n = 1 / n_valid,
 * with every valid row. The program checks these closed forms and exits 0 on success.
 * Usage: c_abi_example (no arguments). */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "slm.h"

#define CHECK_CUDA(x)                                                   \
  do {                                                                  \
    cudaError_t e_ = (x);                                               \
    if (e_ != cudaSuccess) {                                            \
      fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_));          \
      return 2;                                                         \
    }                                                                   \
  } while (0)
#define CHECK_SLM(x)                                                    \
  do {                                                                  \
    int s_ = (x);                                                       \
    if (s_ != SLM_OK) {                                                 \
      fprintf(stderr, "%s: %s\n", #x, slm_status_string(s_));           \
      return 3;                                                         \
    }                                                                   \
  } while (0)

static uint16_t bf16_of(float f) { /* round to nearest even */
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}
static float float_of(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

int main(void) {
  const int64_t N = 300, d = 64, V = 1000;
  const int32_t ignore = -100;
  uint16_t* hH = malloc(N * d * 2);
  int32_t* hy = malloc(N * 4);
  uint32_t seed = 12345u;
  int64_t n_valid_ref = 0;
  for (int64_t i = 0; i < N * d; ++i) {
    seed = seed * 1664525u + 1013904223u;
    hH[i] = bf16_of(((float)(seed >> 8) / 16777216.0f) * 2.0f - 1.0f);
  }
  for (int64_t n = 0; n < N; ++n) {
    seed = seed * 1664525u + 1013904223u;
    hy[n] = (n % 10 == 3) ? ignore : (int32_t)((seed >> 8) % (uint32_t)V);
    n_valid_ref += hy[n] != ignore;
  }
  void *H, *W, *dH, *ws;
  int32_t* y;
  float *loss_tok, *stats, *dW, *loss_mean;
  double* loss_sum;
  int64_t* n_valid;
  const size_t ws_bytes = slm_workspace_bytes(SLM_CE, N, d, V, 0);
  CHECK_CUDA(cudaMalloc(&H, N * d * 2));
  CHECK_CUDA(cudaMalloc(&W, V * d * 2));
  CHECK_CUDA(cudaMalloc(&dH, N * d * 2));
  CHECK_CUDA(cudaMalloc((void**)&dW, V * d * 4));
  CHECK_CUDA(cudaMalloc((void**)&y, N * 4));
  CHECK_CUDA(cudaMalloc((void**)&loss_tok, N * 4));
  CHECK_CUDA(cudaMalloc((void**)&stats, slm_stats_floats(SLM_CE) * N * 4));
  CHECK_CUDA(cudaMalloc((void**)&loss_sum, 8));
  CHECK_CUDA(cudaMalloc((void**)&n_valid, 8));
  CHECK_CUDA(cudaMalloc((void**)&loss_mean, 4));
  CHECK_CUDA(cudaMalloc(&ws, ws_bytes));
  CHECK_CUDA(cudaMemcpy(H, hH, N * d * 2, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(y, hy, N * 4, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemset(W, 0, V * d * 2));

  CHECK_SLM(slm_loss_fwd(SLM_CE, H, NULL, W, y, ignore, N, d, V, loss_tok, NULL, loss_sum,
                         n_valid, loss_mean, stats, ws, ws_bytes, NULL));
  CHECK_SLM(slm_loss_bwd(SLM_CE, H, NULL, W, y, ignore, N, d, V, NULL, NULL, n_valid, stats,
                         dH, dW, 0, 0, ws, ws_bytes, NULL));
  CHECK_SLM(slm_device_status(ws, NULL));

  float mean;
  int64_t nv;
  float* hdW = malloc(V * d * 4);
  uint16_t* hdH = malloc(N * d * 2);
  CHECK_CUDA(cudaMemcpy(&mean, loss_mean, 4, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(&nv, n_valid, 8, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(hdW, dW, V * d * 4, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(hdH, dH, N * d * 2, cudaMemcpyDeviceToHost));

  int bad = 0;
  if (nv != n_valid_ref) bad |= 1;
  if (fabs(mean - log((double)V)) > 2e-3 * log((double)V)) bad |= 2;
  for (int64_t i = 0; i < N * d; ++i)
    if (float_of(hdH[i]) != 0.0f) bad |= 4;
  /* dW against its closed form, every element, within the parity tolerance. */
  double* ref = calloc(V * d, 8);
  double refmax = 0.0, errmax = 0.0;
  for (int64_t n = 0; n < N; ++n) {
    if (hy[n] == ignore) continue;
    for (int64_t v = 0; v < V; ++v) {
      const double c = (1.0 / V - (v == hy[n] ? 1.0 : 0.0)) / (double)n_valid_ref;
      for (int64_t k = 0; k < d; ++k) ref[v * d + k] += c * float_of(hH[n * d + k]);
    }
  }
  for (int64_t i = 0; i < V * d; ++i) {
    if (fabs(ref[i]) > refmax) refmax = fabs(ref[i]);
    if (fabs(ref[i] - hdW[i]) > errmax) errmax = fabs(ref[i] - hdW[i]);
  }
  if (errmax > 1e-2 * refmax) bad |= 8;
  printf("n_valid %lld (want %lld)  mean %.6f (log V %.6f)  dW err/max %.3g  %s\n",
         (long long)nv, (long long)n_valid_ref, mean, log((double)V), errmax / refmax,
         bad ? "FAIL" : "ok");
  return bad ? 1 : 0;
}
