// FP8 E4M3 row quantisation for the 8-bit expert path.
//
// The pages name 8-bit (and 4-bit) experts as the way serving systems shrink
// the expert weights ("Mixture of Experts: why a model with 671 billion
// parameters uses only 37", "How data centres handle it"; "Mixture of
// experts: how MoE works and what it costs", the memory arithmetic) without
// fixing a scheme.  This build uses the plainest one: every row (a weight
// output channel, or a token's activation vector) gets its own fp32 scale
//   s = max|x| / 448   (448 = the largest finite E4M3 value; s = 1 for a zero row)
// and its values are stored as q = E4M3(x / s), rounded to nearest even with
// saturation, so that x ~ q * s.  The division and the rounding are the
// IEEE-rounded fp32 division and the hardware fp32 -> e4m3 conversion.
//
// One warp per row: a pass for the absolute maximum, then a pass that
// converts eight values per lane and stores them as one 8-byte word.
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

__global__ void __launch_bounds__(kThreads)
    quantize_rows_e4m3_kernel(const __nv_bfloat16* __restrict__ src, int64_t rows, const int32_t* rows_dev,
                              int cols, uint8_t* __restrict__ q, float* __restrict__ scale) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t dr = rows_dev ? (int64_t)*rows_dev : rows;  // rows in use (device count), at most `rows`
  const int64_t n = dr < rows ? dr : rows;
  const int nv = cols / 8;  // 16-byte vectors of 8 bf16
  for (int64_t r = (int64_t)blockIdx.x * kWarps + warp; r < n; r += (int64_t)gridDim.x * kWarps) {
    const uint4* row = reinterpret_cast<const uint4*>(src + r * cols);
    float amax = 0.f;
    for (int v = lane; v < nv; v += 32) {
      const uint4 w = __ldg(row + v);
      const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&w);
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(__bfloat162float(e[i])));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const float s = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    if (lane == 0) scale[r] = s;
    uint2* out = reinterpret_cast<uint2*>(q + r * cols);
    for (int v = lane; v < nv; v += 32) {
      const uint4 w = __ldg(row + v);
      const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&w);
      uint32_t word[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t pk = 0;
#pragma unroll
        for (int i = 0; i < 4; i += 2) {
          const float2 f2 = make_float2(__fdiv_rn(__bfloat162float(e[4 * h + i]), s),
                                        __fdiv_rn(__bfloat162float(e[4 * h + i + 1]), s));
          const __nv_fp8x2_storage_t c = __nv_cvt_float2_to_fp8x2(f2, __NV_SATFINITE, __NV_E4M3);
          pk |= (uint32_t)c << (16 * (i / 2));
        }
        word[h] = pk;
      }
      out[v] = make_uint2(word[0], word[1]);
    }
  }
}

}  // namespace

cudaError_t launch_quantize_e4m3(const void* src, int64_t rows, const int32_t* rows_dev, int cols, uint8_t* q,
                                 float* scale, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  int64_t blocks = (rows + kWarps - 1) / kWarps;
  const int64_t cap = (int64_t)device_sm_count() * 16;
  if (blocks > cap) blocks = cap;
  quantize_rows_e4m3_kernel<<<(unsigned)blocks, kThreads, 0, stream>>>(static_cast<const __nv_bfloat16*>(src), rows,
                                                                        rows_dev, cols, q, scale);
  return cudaGetLastError();
}

}  // namespace moe
