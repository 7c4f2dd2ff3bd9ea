/* A plain C client that runs one layer on the GPU through the ABI: C99,
   device memory from the CUDA runtime's C API, bf16 values as raw 16-bit
   patterns.  Built and run by tests/test_abi_c.py on a GPU; prints "ok" when
   moe_forward returns MOE_OK, the device status word is clear, every output
   is finite and every token's gate weights sum to 1.  With a file name as
   its argument it also writes the layer output y (T*d bf16 bit patterns) and
   the expert ids (T*k int32) there, for the test to compare with the oracle
   on the same inputs (splitmix64 draws, regenerated on the Python side). */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "moe.h"

static uint16_t bf16_bits(float f) {  /* round to nearest even */
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

static float uniform(uint64_t* s) {  /* splitmix64 -> [-1, 1) */
  uint64_t z = (*s += 0x9E3779B97F4A7C15ull);
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  z ^= z >> 31;
  return (float)((double)(z >> 11) / 9007199254740992.0 * 2.0 - 1.0);
}

static void* upload(size_t n, float scale, uint64_t* seed) {
  uint16_t* h = (uint16_t*)malloc(n * 2);
  for (size_t i = 0; i < n; ++i) h[i] = bf16_bits(uniform(seed) * scale);
  void* d = NULL;
  if (cudaMalloc(&d, n * 2) != cudaSuccess || cudaMemcpy(d, h, n * 2, cudaMemcpyHostToDevice) != cudaSuccess) d = NULL;
  free(h);
  return d;
}

int main(int argc, char** argv) {
  moe_config c;
  memset(&c, 0, sizeof c);
  c.T = 300;
  c.d_model = 512;
  c.n_experts = 8;
  c.top_k = 2;
  c.d_ff = 640;
  c.dtype = MOE_BF16;
  c.gating = MOE_SOFTMAX_TOPK;
  const int64_t T = c.T, d = c.d_model, E = c.n_experts, k = c.top_k, f = c.d_ff;
  uint64_t seed = 7;
  void* x = upload((size_t)(T * d), 1.0f, &seed);
  void* wr = upload((size_t)(E * d), 0.05f, &seed);
  void* wgu = upload((size_t)(E * 2 * f * d), 0.05f, &seed);
  void* wd = upload((size_t)(E * d * f), 0.05f, &seed);
  void *y = NULL, *w = NULL, *ws = NULL, *ids = NULL;
  const size_t ws_bytes = moe_workspace_bytes(&c);
  if (!x || !wr || !wgu || !wd || cudaMalloc(&y, (size_t)(T * d * 2)) != cudaSuccess ||
      cudaMalloc(&w, (size_t)(T * k * 4)) != cudaSuccess || cudaMalloc(&ws, ws_bytes) != cudaSuccess ||
      cudaMalloc(&ids, (size_t)(T * k * 4)) != cudaSuccess) {
    fprintf(stderr, "device allocation failed\n");
    return 1;
  }
  moe_status st =
      moe_forward(&c, x, wr, NULL, wgu, wd, NULL, NULL, y, (int32_t*)ids, (float*)w, NULL, ws, ws_bytes, NULL);
  if (st != MOE_OK) {
    fprintf(stderr, "moe_forward: %s\n", moe_status_string(st));
    return 1;
  }
  st = moe_device_status(ws, ws_bytes, NULL);
  if (st != MOE_OK) {
    fprintf(stderr, "device status: %s\n", moe_status_string(st));
    return 1;
  }
  uint16_t* yh = (uint16_t*)malloc((size_t)(T * d * 2));
  float* wh = (float*)malloc((size_t)(T * k * 4));
  cudaMemcpy(yh, y, (size_t)(T * d * 2), cudaMemcpyDeviceToHost);
  cudaMemcpy(wh, w, (size_t)(T * k * 4), cudaMemcpyDeviceToHost);
  int bad = 0;
  if (argc > 1) {
    int32_t* ih = (int32_t*)malloc((size_t)(T * k * 4));
    cudaMemcpy(ih, ids, (size_t)(T * k * 4), cudaMemcpyDeviceToHost);
    FILE* fo = fopen(argv[1], "wb");
    if (!fo || fwrite(yh, 2, (size_t)(T * d), fo) != (size_t)(T * d) ||
        fwrite(ih, 4, (size_t)(T * k), fo) != (size_t)(T * k))
      bad += 1;
    if (fo) fclose(fo);
    free(ih);
  }
  for (int64_t i = 0; i < T * d; ++i) bad += (yh[i] & 0x7F80u) == 0x7F80u; /* Inf or NaN */
  for (int64_t t = 0; t < T; ++t) {
    double s = 0.0;
    for (int64_t j = 0; j < k; ++j) s += wh[t * k + j];
    bad += fabs(s - 1.0) > 1e-5;
  }
  free(yh);
  free(wh);
  cudaFree(x);
  cudaFree(wr);
  cudaFree(wgu);
  cudaFree(wd);
  cudaFree(y);
  cudaFree(w);
  cudaFree(ws);
  cudaFree(ids);
  if (bad) {
    fprintf(stderr, "%d bad values\n", bad);
    return 1;
  }
  printf("ok\n");
  return 0;
}
