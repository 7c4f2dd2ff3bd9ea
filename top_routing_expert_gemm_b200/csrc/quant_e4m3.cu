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
// dispatch path quantises while it gathers: each token's vector is quantised
// once, straight from x, and its codes are written to the token's rows (the
// same codes as quantising the gathered bf16 copies, which are never written).
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.cuh"
#include "pdl.cuh"

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

// Row r of src -> codes row r and scale[r]; rows past *rows_dev (when given)
// are left alone.  A pass for the absolute maximum (skipped when amax_bits
// holds it: the 8-bit GEMM-1 leaves it there for h), then a pass that converts
// (it finds the row in L1).  Eight independent 16-byte loads in flight per
// lane, with registers left for many warps per SM to hide the latency of the
// loads and of the IEEE divisions (a variant holding the whole row in
// registers ran at one block per SM and measured slower).
__global__ void __launch_bounds__(kThreads)
    quantize_rows_e4m3_kernel(const __nv_bfloat16* __restrict__ src, int64_t rows, const int32_t* rows_dev,
                              int cols, uint8_t* __restrict__ q, float* scale, const uint32_t* amax_bits) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t dr = rows_dev ? (int64_t)*rows_dev : rows;
  const int64_t n = dr < rows ? dr : rows;
  const int nv = cols / 8;
  for (int64_t r = (int64_t)blockIdx.x * kWarps + warp; r < n; r += (int64_t)gridDim.x * kWarps) {
    const uint4* row = reinterpret_cast<const uint4*>(src + r * cols);
    float s;
    int v = lane;
    if (amax_bits) {  // the row's maximum is known: read it before its scale overwrites it
      const float amax = __uint_as_float(amax_bits[r] << 16);
      s = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
      __syncwarp();
    } else {
      float amax = 0.f;
      for (; v + 7 * 32 < nv; v += 8 * 32) {  // eight independent loads in flight per lane
        uint4 a[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) a[i] = __ldg(row + v + 32 * i);
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = amax8(a[i], amax);
      }
      for (; v < nv; v += 32) amax = amax8(__ldg(row + v), amax);
      s = row_scale(amax);
    }
    if (lane == 0) scale[r] = s;
    uint2* out = reinterpret_cast<uint2*>(q + r * cols);
    for (v = lane; v + 7 * 32 < nv; v += 8 * 32) {
      uint4 a[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = __ldg(row + v + 32 * i);
#pragma unroll
      for (int i = 0; i < 8; ++i) out[v + 32 * i] = e4m3x8(a[i], s);
    }
    for (; v < nv; v += 32) out[v] = e4m3x8(__ldg(row + v), s);
  }
}

// The dispatch with 8-bit experts: token t of x is quantised once and its
// codes and scale go to every kept row row_of[t*k + s] (one warp per token,
// as in the bf16 gather), so x crosses HBM once and no bf16 copy is written.
__global__ void __launch_bounds__(kThreads)
    gather_quantize_e4m3_kernel(const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ row_of,
                                int64_t T, int k, int cols, uint8_t* __restrict__ q, float* __restrict__ scale) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nv = cols / 8;
  grid_dependency_wait();  // row_of of the dispatch (programmatic launch)
  if (threadIdx.x == 0) grid_launch_dependents();
  for (int64_t t = (int64_t)blockIdx.x * kWarps + warp; t < T; t += (int64_t)gridDim.x * kWarps) {
    const uint4* row = reinterpret_cast<const uint4*>(x + t * cols);
    const int my_row = lane < k ? row_of[t * k + lane] : -1;  // k <= kMaxTopK <= 32
    float amax = 0.f;
    int v = lane;
    for (; v + 7 * 32 < nv; v += 8 * 32) {  // eight independent loads in flight per lane
      uint4 a[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = __ldg(row + v + 32 * i);
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = amax8(a[i], amax);
    }
    for (; v < nv; v += 32) amax = amax8(__ldg(row + v), amax);
    const float s = row_scale(amax);
    if (my_row >= 0) scale[my_row] = s;
    for (int v0 = 0; v0 < nv; v0 += 128) {  // the same trip count on every lane (shuffles inside)
      v = v0 + lane;
      uint2 c[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (v + 32 * i < nv) c[i] = e4m3x8(__ldg(row + v + 32 * i), s);
      for (int j = 0; j < k; ++j) {
        const int r = __shfl_sync(0xffffffffu, my_row, j);
        if (r < 0) continue;  // dropped by the capacity
        uint2* out = reinterpret_cast<uint2*>(q + (int64_t)r * cols);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (v + 32 * i < nv) out[v + 32 * i] = c[i];
      }
    }
  }
}

int64_t grid_for(int64_t units) {
  int64_t blocks = (units + kWarps - 1) / kWarps;
  const int64_t cap = (int64_t)device_sm_count() * 16;
  return blocks > cap ? cap : blocks;
}

}  // namespace

cudaError_t launch_quantize_e4m3(const void* src, int64_t rows, const int32_t* rows_dev, int cols, uint8_t* q,
                                 float* scale, cudaStream_t stream, const uint32_t* amax_bits) {
  if (rows == 0) return cudaSuccess;
  quantize_rows_e4m3_kernel<<<(unsigned)grid_for(rows), kThreads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(src), rows, rows_dev, cols, q, scale, amax_bits);
  return cudaGetLastError();
}

cudaError_t launch_gather_quantize_e4m3(const void* x, const int32_t* row_of, int k, int64_t T, int cols,
                                        uint8_t* q, float* scale, bool chained, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  return launch_maybe_chained(gather_quantize_e4m3_kernel, dim3((unsigned)grid_for(T)), dim3(kThreads), 0, stream,
                              chained, static_cast<const __nv_bfloat16*>(x), row_of, T, k, cols, q, scale);
}

}  // namespace moe
