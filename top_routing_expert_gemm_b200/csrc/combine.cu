// Weighted un-permute ("Run and combine"): y[t] = sum_s w[t,s] * y_perm[row_of[t*k+s]]
// (+ y_shared[t]).  "Mixture of Experts Explained: Routers, Active Parameters
// and VRAM" (step 5: multiply each expert output by its weight and add them
// up); "Mixture of Experts: why a model with 671 billion parameters uses only
// 37" ("Where MoE changes the Transformer": outputs summed, weighted by the
// router's scores).  One block per token, 16-byte vectors, fp32 accumulation.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {
namespace {

constexpr int kThreads = 128;

template <typename T>
__global__ void __launch_bounds__(kThreads) combine_kernel(const T* __restrict__ y_perm,
                                                           const int32_t* __restrict__ row_of,
                                                           const float* __restrict__ w,
                                                           const T* __restrict__ y_shared, T* __restrict__ y,
                                                           int64_t n_tok, int k, int d) {
  constexpr int V = Vec16<T>::N;
  const int nv = d / V;
  for (int64_t t = blockIdx.x; t < n_tok; t += gridDim.x) {
    for (int v = threadIdx.x; v < nv; v += kThreads) {
      float acc[V];
#pragma unroll
      for (int j = 0; j < V; ++j) acc[j] = 0.f;
      for (int s = 0; s < k; ++s) {
        const int row = row_of[t * k + s];
        if (row < 0) continue;
        const float ws = w[t * k + s];
        const Vec16<T> yv = ld16(y_perm + (int64_t)row * d + (int64_t)v * V);
#pragma unroll
        for (int j = 0; j < V; ++j) acc[j] = fmaf(ws, Elem<T>::to_f(yv.v[j]), acc[j]);
      }
      if (y_shared) {
        const Vec16<T> sv = ld16(y_shared + t * d + (int64_t)v * V);
#pragma unroll
        for (int j = 0; j < V; ++j) acc[j] += Elem<T>::to_f(sv.v[j]);
      }
      Vec16<T> o;
#pragma unroll
      for (int j = 0; j < V; ++j) o.v[j] = Elem<T>::from_f(acc[j]);
      st16(y + t * d + (int64_t)v * V, o);
    }
  }
}

}  // namespace

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t stream) {
  if (a.T == 0) return cudaSuccess;
  int64_t blocks = a.T;
  const int64_t cap = (int64_t)device_sm_count() * 64;
  if (blocks > cap) blocks = cap;
  if (a.bf16) {
    combine_kernel<__nv_bfloat16><<<(unsigned)blocks, kThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(a.y_perm), a.row_of, a.w,
        static_cast<const __nv_bfloat16*>(a.y_shared), static_cast<__nv_bfloat16*>(a.y), a.T, a.k, a.d);
  } else {
    combine_kernel<float><<<(unsigned)blocks, kThreads, 0, stream>>>(
        static_cast<const float*>(a.y_perm), a.row_of, a.w, static_cast<const float*>(a.y_shared),
        static_cast<float*>(a.y), a.T, a.k, a.d);
  }
  return cudaGetLastError();
}

}  // namespace moe
