/* Calls bsa_forward through the C ABI from C (no Python): a tensor-core plan
 * (bf16, 128-token blocks, ragged grid, text tokens), Q and K from a fixed
 * pattern, V = 1 everywhere.  Every attention row is a convex combination of
 * value rows, so every output element must be 1 (up to bf16 rounding).  Also
 * checks that a too-small workspace is refused.  Exit status 0 = pass. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <cuda_runtime.h>
#include "bsa.h"

static uint16_t to_bf16(float f) {
  union { float f; uint32_t u; } x = {f};
  return (uint16_t)((x.u + 0x7fffu + ((x.u >> 16) & 1u)) >> 16);   /* round to nearest even */
}
static float from_bf16(uint16_t h) {
  union { uint32_t u; float f; } x = {(uint32_t)h << 16};
  return x.f;
}

int main(void) {
  const int B = 1, T = 3, H = 12, W = 20, heads = 2, D = 128, n_text = 40;
  bsa_plan_t plan;
  if (bsa_plan_create(&plan, B, T, H, W, 1, 8, 16, heads, D, n_text, BSA_BF16) != BSA_OK) {
    fprintf(stderr, "plan: %s\n", bsa_last_error_string());
    return 1;
  }
  bsa_plan_info_t info;
  bsa_plan_get_info(plan, &info);
  const size_t n = (size_t)B * info.n_tot * heads * D;
  uint16_t* hq = (uint16_t*)malloc(n * 2);
  uint16_t* hv = (uint16_t*)malloc(n * 2);
  uint16_t* ho = (uint16_t*)malloc(n * 2);
  for (size_t i = 0; i < n; ++i) {
    hq[i] = to_bf16(sinf(0.37f * (float)(i % 9973)) * 1.5f);
    hv[i] = to_bf16(1.0f);
  }
  void *q, *k, *v, *o, *ws;
  cudaMalloc(&q, n * 2); cudaMalloc(&k, n * 2); cudaMalloc(&v, n * 2); cudaMalloc(&o, n * 2);
  cudaMemcpy(q, hq, n * 2, cudaMemcpyHostToDevice);
  cudaMemcpy(k, hq, n * 2, cudaMemcpyHostToDevice);
  cudaMemcpy(v, hv, n * 2, cudaMemcpyHostToDevice);
  double density[2] = {0.3, 0.6};
  int kmax = 0;
  size_t select_ws = 0, forward_ws = 0;
  if (bsa_kmax_for(plan, BSA_TOPK, density, &kmax) != BSA_OK ||
      bsa_workspace_size(plan, kmax, &select_ws, &forward_ws) != BSA_OK) {
    fprintf(stderr, "sizes: %s\n", bsa_last_error_string());
    return 1;
  }
  cudaMalloc(&ws, forward_ws);
  cudaStream_t stream;
  cudaStreamCreate(&stream);
  if (bsa_forward(plan, q, k, v, BSA_TOPK, density, kmax, o, NULL, NULL, ws, forward_ws - 256, NULL,
                  stream) != BSA_ERR_WORKSPACE) {
    fprintf(stderr, "a too-small workspace was not refused\n");
    return 1;
  }
  bsa_status s = bsa_forward(plan, q, k, v, BSA_TOPK, density, kmax, o, NULL, NULL, ws, forward_ws,
                             NULL, stream);
  if (s == BSA_OK) s = bsa_check_status(plan, stream);
  if (s != BSA_OK) {
    fprintf(stderr, "forward: %s\n", bsa_last_error_string());
    return 1;
  }
  cudaMemcpy(ho, o, n * 2, cudaMemcpyDeviceToHost);
  double max_err = 0.0;
  for (size_t i = 0; i < n; ++i) {
    const double e = fabs((double)from_bf16(ho[i]) - 1.0);
    if (!(e <= max_err)) max_err = e;   /* NaN propagates */
  }
  printf("attn_path %d, kmax %d, %zu outputs, max |o - 1| = %.3e\n", info.attn_path, kmax, n, max_err);
  cudaFree(q); cudaFree(k); cudaFree(v); cudaFree(o); cudaFree(ws);
  cudaStreamDestroy(stream);
  bsa_plan_destroy(plan);
  free(hq); free(hv); free(ho);
  return (info.attn_path == 1 && max_err <= 1e-2) ? 0 : 1;
}
