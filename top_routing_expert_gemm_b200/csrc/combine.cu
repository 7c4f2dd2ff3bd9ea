// Weighted un-permute ("Run and combine"): y[t] = sum_s w[t,s] * y_perm[row_of[t*k+s]]
// (+ y_shared[t]).  "Mixture of Experts Explained: Routers, Active Parameters
// and VRAM" (step 5: multiply each expert output by its weight and add them
// up); "Mixture of Experts: why a model with 671 billion parameters uses only
// 37" ("Where MoE changes the Transformer": outputs summed, weighted by the
// router's scores).  One block per token, 16-byte vectors, fp32 accumulation
// in slot order.
#include "common.cuh"
#include "kernels.cuh"
#include "pdl.cuh"

namespace moe {
namespace {

constexpr int kThreads = 128;

// KMAX >= k: the k rows of a token are read with independent loads (the slot
// loop is unrolled), so each thread has k 16-byte loads in flight instead of
// one; the token's rows and weights are read once per thread.
template <typename T, int KMAX>
__global__ void __launch_bounds__(kThreads) combine_kernel(const T* __restrict__ y_perm,
                                                           const int32_t* __restrict__ row_of,
                                                           const float* __restrict__ w,
                                                           const T* __restrict__ y_shared, T* __restrict__ y,
                                                           int64_t n_tok, int k, int d) {
  constexpr int V = Vec16<T>::N;
  const int nv = d / V;
  grid_dependency_wait();  // the expert outputs (programmatic launch)
  for (int64_t t = blockIdx.x; t < n_tok; t += gridDim.x) {
    int rows[KMAX];
    float ws[KMAX];
#pragma unroll
    for (int s = 0; s < KMAX; ++s) {
      rows[s] = s < k ? row_of[t * k + s] : -1;
      ws[s] = s < k ? w[t * k + s] : 0.f;
    }
    for (int v = threadIdx.x; v < nv; v += kThreads) {
      Vec16<T> yv[KMAX];
#pragma unroll
      for (int s = 0; s < KMAX; ++s)
        if (rows[s] >= 0) yv[s] = ld16(y_perm + (int64_t)rows[s] * d + (int64_t)v * V);
      float acc[V];
#pragma unroll
      for (int j = 0; j < V; ++j) acc[j] = 0.f;
#pragma unroll
      for (int s = 0; s < KMAX; ++s) {  // slot order: the same sums as a plain loop over s
        if (rows[s] >= 0) {
#pragma unroll
          for (int j = 0; j < V; ++j) acc[j] = fmaf(ws[s], Elem<T>::to_f(yv[s].v[j]), acc[j]);
        }
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

template <typename T>
cudaError_t launch_t(const CombineArgs& a, unsigned blocks, cudaStream_t stream) {
  const T* yp = static_cast<const T*>(a.y_perm);
  const T* ys = static_cast<const T*>(a.y_shared);
  T* y = static_cast<T*>(a.y);
  auto run = [&](auto kernel) {
    return launch_maybe_chained(kernel, dim3(blocks), dim3(kThreads), 0, stream, a.chained, yp, a.row_of, a.w, ys, y,
                                a.T, a.k, a.d);
  };
  if (a.k <= 2) return run(combine_kernel<T, 2>);
  if (a.k <= 4) return run(combine_kernel<T, 4>);
  if (a.k <= 8) return run(combine_kernel<T, 8>);
  return run(combine_kernel<T, kMaxTopK>);
}

}  // namespace

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t stream) {
  if (a.T == 0) return cudaSuccess;
  int64_t blocks = a.T;
  const int64_t cap = (int64_t)device_sm_count() * 64;
  if (blocks > cap) blocks = cap;
  return a.bf16 ? launch_t<__nv_bfloat16>(a, (unsigned)blocks, stream) : launch_t<float>(a, (unsigned)blocks, stream);
}

}  // namespace moe
