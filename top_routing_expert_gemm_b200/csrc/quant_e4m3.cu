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
// One warp per row; eight values per lane leave as one 8-byte word.  The
// dispatch path quantises while it gathers: output row r is the token row
// perm[r] / k, so each dispatched copy is quantised straight from x (the same
// codes as quantising the gathered bf16 copy) and the bf16 copy is never
// written.
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

// eight bf16 values -> eight E4M3 codes of x / s (one 8-byte word)
__device__ __forceinline__ uint2 e4m3x8(const uint4& w, float s) {
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
  return make_uint2(word[0], word[1]);
}

__device__ __forceinline__ float amax8(const uint4& w, float amax) {
  const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&w);
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(__bfloat162float(e[i])));
  return amax;
}

__device__ __forceinline__ float row_scale(float amax) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  return amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
}

// Output row r reads source row perm[r] / k (a dispatched copy of a token's
// vector) when perm is given, else row r.  Rows past *rows_dev (when given)
// are left alone.

// A pass for the absolute maximum, then a pass that converts (it finds the
// row in L1).  Four independent 16-byte loads in flight per lane; 40
// registers, so that many warps per SM hide the latency of the loads and of
// the IEEE divisions (a variant holding the whole row in registers ran at
// one block per SM and measured slower).
__global__ void __launch_bounds__(kThreads)
    quantize_rows_e4m3_kernel(const __nv_bfloat16* __restrict__ src, const int32_t* __restrict__ perm, int k,
                              int64_t rows, const int32_t* rows_dev, int cols, uint8_t* __restrict__ q,
                              float* __restrict__ scale) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t dr = rows_dev ? (int64_t)*rows_dev : rows;
  const int64_t n = dr < rows ? dr : rows;
  const int nv = cols / 8;
  for (int64_t r = (int64_t)blockIdx.x * kWarps + warp; r < n; r += (int64_t)gridDim.x * kWarps) {
    const int64_t sr = perm ? (int64_t)(perm[r] / k) : r;
    const uint4* row = reinterpret_cast<const uint4*>(src + sr * cols);
    float amax = 0.f;
    int v = lane;
    for (; v + 96 < nv; v += 128) {  // four independent loads in flight per lane
      const uint4 a0 = __ldg(row + v), a1 = __ldg(row + v + 32), a2 = __ldg(row + v + 64), a3 = __ldg(row + v + 96);
      amax = amax8(a3, amax8(a2, amax8(a1, amax8(a0, amax))));
    }
    for (; v < nv; v += 32) amax = amax8(__ldg(row + v), amax);
    const float s = row_scale(amax);
    if (lane == 0) scale[r] = s;
    uint2* out = reinterpret_cast<uint2*>(q + r * cols);
    for (v = lane; v + 96 < nv; v += 128) {
      const uint4 a0 = __ldg(row + v), a1 = __ldg(row + v + 32), a2 = __ldg(row + v + 64), a3 = __ldg(row + v + 96);
      out[v] = e4m3x8(a0, s);
      out[v + 32] = e4m3x8(a1, s);
      out[v + 64] = e4m3x8(a2, s);
      out[v + 96] = e4m3x8(a3, s);
    }
    for (; v < nv; v += 32) out[v] = e4m3x8(__ldg(row + v), s);
  }
}

cudaError_t launch_rows(const void* src, const int32_t* perm, int k, int64_t rows, const int32_t* rows_dev, int cols,
                        uint8_t* q, float* scale, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  int64_t blocks = (rows + kWarps - 1) / kWarps;
  const int64_t cap = (int64_t)device_sm_count() * 16;
  if (blocks > cap) blocks = cap;
  const auto* x = static_cast<const __nv_bfloat16*>(src);
  quantize_rows_e4m3_kernel<<<(unsigned)blocks, kThreads, 0, stream>>>(x, perm, k, rows, rows_dev, cols, q, scale);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize_e4m3(const void* src, int64_t rows, const int32_t* rows_dev, int cols, uint8_t* q,
                                 float* scale, cudaStream_t stream) {
  return launch_rows(src, nullptr, 1, rows, rows_dev, cols, q, scale, stream);
}

cudaError_t launch_gather_quantize_e4m3(const void* x, const int32_t* perm, int k, int64_t rows,
                                        const int32_t* rows_dev, int cols, uint8_t* q, float* scale,
                                        cudaStream_t stream) {
  return launch_rows(x, perm, k, rows, rows_dev, cols, q, scale, stream);
}

}  // namespace moe
