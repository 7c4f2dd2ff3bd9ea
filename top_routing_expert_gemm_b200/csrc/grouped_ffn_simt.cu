// fp32 grouped experts on CUDA cores (no TF32: the fp32 layer keeps a 24-bit
// mantissa end to end).  Same grouping contract as the tensor-core path: rows
// [offsets[g], offsets[g+1]) of A use weight group g.
//
//   GEMM-1 + SwiGLU : h = SiLU(A Wg^T) * (A Wu^T)     (gate rows 0..f-1, up rows f..2f-1)
//   GEMM-1 + GELU   : h = GELU(A Wu^T)                (two-matrix expert)
//   GEMM-2          : y = h Wd^T
//
// Expert FFN: "Mixture of Experts Explained: Routers, Active Parameters and
// VRAM" (a gated feed-forward block with three matrices; the runnable build's
// two-matrix expert with GELU between them).
// 64x64 output tiles, K in steps of 16 through shared memory, 4x4 outputs per
// thread.  The grid covers an upper bound of the (group, m-tile) pairs; each
// block finds its pair from the device offsets, so no host sync is needed.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {
namespace {

constexpr int BM = 64, BN = 64, BK = 16, kThreads = 256;

// m-tile index -> (group, first row, rows in group); false when past the end
__device__ bool find_group_tile(const int32_t* offsets, int G, int64_t rows, int64_t mt_index, int* g_out,
                                int64_t* row0, int64_t* n_rows) {
  if (offsets == nullptr) {
    if (mt_index * BM >= rows) return false;
    *g_out = 0;
    *row0 = mt_index * BM;
    *n_rows = rows - mt_index * BM;
    return true;
  }
  int64_t acc = 0;
  for (int g = 0; g < G; ++g) {
    const int64_t n = offsets[g + 1] - offsets[g];
    const int64_t mt = (n + BM - 1) / BM;
    if (mt_index < acc + mt) {
      const int64_t local = mt_index - acc;
      *g_out = g;
      *row0 = offsets[g] + local * BM;
      *n_rows = n - local * BM;
      return true;
    }
    acc += mt;
  }
  return false;
}

template <int EPI>
__global__ void __launch_bounds__(kThreads) grouped_gemm_f32_kernel(const float* __restrict__ A, int64_t rows,
                                                                    const int32_t* __restrict__ offsets, int G,
                                                                    const float* __restrict__ W,
                                                                    int64_t w_group_rows, int up_off, int K,
                                                                    int N, float* __restrict__ out) {
  constexpr bool SWIGLU = EPI == kEpiSwiGLU;
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[SWIGLU ? 2 : 1][BK][BN + 4];
  __shared__ int s_g;
  __shared__ long long s_row0, s_n;
  if (threadIdx.x == 0) {
    int g;
    int64_t r0, n;
    if (!find_group_tile(offsets, G, rows, blockIdx.x, &g, &r0, &n)) g = -1;
    s_g = g;
    s_row0 = r0;
    s_n = n;
  }
  __syncthreads();
  const int g = s_g;
  if (g < 0) return;
  const int64_t row0 = s_row0;
  const int m_valid = (int)min((long long)BM, s_n);
  const int n0 = blockIdx.y * BN;
  const float* Wg = W + (int64_t)g * w_group_rows * K;

  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc0[4][4], acc1[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc0[i][j] = acc1[i][j] = 0.f;

  // loader mapping: 64 rows x 16 k = 256 threads x 4 consecutive k
  const int lr = threadIdx.x / 4, lk = (threadIdx.x % 4) * 4;
  for (int k0 = 0; k0 < K; k0 += BK) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int kk = k0 + lk + j;
      As[lk + j][lr] = (lr < m_valid && kk < K) ? A[(row0 + lr) * K + kk] : 0.f;
      const int nrow = n0 + lr;
      Bs[0][lk + j][lr] = (nrow < N && kk < K) ? Wg[(int64_t)nrow * K + kk] : 0.f;
      if (SWIGLU) Bs[SWIGLU ? 1 : 0][lk + j][lr] = (nrow < N && kk < K) ? Wg[(int64_t)(up_off + nrow) * K + kk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b0[4], b1[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        b0[j] = Bs[0][kk][tx * 4 + j];
        b1[j] = SWIGLU ? Bs[SWIGLU ? 1 : 0][kk][tx * 4 + j] : 0.f;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc0[i][j] = fmaf(a[i], b0[j], acc0[i][j]);
          if (SWIGLU) acc1[i][j] = fmaf(a[i], b1[j], acc1[i][j]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty * 4 + i;
    if (r >= m_valid) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = n0 + tx * 4 + j;
      if (c >= N) continue;
      out[(row0 + r) * N + c] = EPI == kEpiSwiGLU ? silu_f(acc0[i][j]) * acc1[i][j]
                                : EPI == kEpiGELU  ? gelu_f(acc0[i][j])
                                                   : acc0[i][j];
    }
  }
}

}  // namespace

cudaError_t launch_grouped_ffn_f32_simt(const GroupedFfnArgs& a, cudaStream_t stream) {
  if (a.rows == 0) return cudaSuccess;
  const int64_t mt_bound = (a.rows + BM - 1) / BM + (a.offsets ? a.G : 0);
  const dim3 grid1((unsigned)mt_bound, (unsigned)((a.f + BN - 1) / BN));
  if (a.act == kEpiGELU)
    grouped_gemm_f32_kernel<kEpiGELU><<<grid1, kThreads, 0, stream>>>(
        static_cast<const float*>(a.a), a.rows, a.offsets, a.G, static_cast<const float*>(a.w_gate_up),
        (int64_t)a.f, 0, a.d, a.f, static_cast<float*>(a.h));
  else
    grouped_gemm_f32_kernel<kEpiSwiGLU><<<grid1, kThreads, 0, stream>>>(
        static_cast<const float*>(a.a), a.rows, a.offsets, a.G, static_cast<const float*>(a.w_gate_up),
        2 * (int64_t)a.f, a.f, a.d, a.f, static_cast<float*>(a.h));
  const dim3 grid2((unsigned)mt_bound, (unsigned)((a.d + BN - 1) / BN));
  grouped_gemm_f32_kernel<kEpiNone><<<grid2, kThreads, 0, stream>>>(
      static_cast<const float*>(a.h), a.rows, a.offsets, a.G, static_cast<const float*>(a.w_down), a.d, 0, a.f,
      a.d, static_cast<float*>(a.y));
  return cudaGetLastError();
}

}  // namespace moe
