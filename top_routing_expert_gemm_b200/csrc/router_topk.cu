// Fused router: logits = x W_r^T, selection key = logits + bias, top-k with a
// warp-shuffle merge, then the gate weights of the chosen experts.
//
// Follows the router steps of "Mixture of Experts Explained: Routers, Active
// Parameters and VRAM" (Score, Normalise, Keep the top k, Renormalise), the
// top-k-then-softmax router of "Mixture of Experts: why a model with 671
// billion parameters uses only 37" ("The router: how a token chooses
// experts") and its sigmoid gating ("How many experts to pick and how to
// score them"); softmax probabilities kept without renormalisation as in
// "Mixture of Experts (MoE): routing, expert parallelism, and memory" ("How
// does MoE routing work"), the raw router probability of top-1 routing.
//
// One warp owns one token at a time.  Lanes split d (16-byte vector loads),
// accumulate eight experts' dot products at once in fp32, and butterfly-reduce
// them into a per-warp logit row in shared memory.  When W_r fits in shared
// memory (small E: Mixtral-shaped and decode layers) every block stages it
// once; otherwise it streams from L2.  Top-k: each lane keeps the best KMAX of
// its strided experts, then k rounds of a warp arg-max (key desc, index asc)
// pop the winners.
#include "common.cuh"
#include "kernels.cuh"
#include "pdl.cuh"

namespace moe {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kGroup = 8;  // experts accumulated per pass over x

struct RouterParams {
  const void* x;
  const void* w;
  const float* bias;
  int32_t* ids;
  float* wts;
  int64_t T;
  int d, E, k, gating, bias_select_only;
  float* aux_part;  // AUX: [gridDim.x][E + 1] per-block penalty sums
};

// Top k of kappa = logit + bias over the E logits in shared memory, then the
// gate weights of the chosen experts; one warp, results for token t.
template <int KMAX>
__device__ __forceinline__ void select_and_weigh(const RouterParams& p, const float* logits, int64_t t, int lane) {
  const int E = p.E, k = p.k;
  // ---- Keep the top k of kappa = logit + bias
  TopK<KMAX> tk;
  tk.init();
  float mx = -INFINITY;
  for (int e = lane; e < E; e += 32) {
    const float kap = logits[e] + (p.bias ? p.bias[e] : 0.f);
    tk.push(kap, e);
    mx = fmaxf(mx, kap);
  }
  float sel_key[KMAX];
  int sel_idx[KMAX];
#pragma unroll
  for (int s = 0; s < KMAX; ++s) {
    if (s < k) {
      float bk = tk.key[0];
      int bi = tk.idx[0];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ok = __shfl_xor_sync(0xffffffffu, bk, off);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
        if (ranks_before(ok, oi, bk, bi)) { bk = ok; bi = oi; }
      }
      sel_key[s] = bk;
      sel_idx[s] = bi;
      if (tk.idx[0] == bi) {  // the owning lane pops its head
#pragma unroll
        for (int j = 0; j + 1 < KMAX; ++j) { tk.key[j] = tk.key[j + 1]; tk.idx[j] = tk.idx[j + 1]; }
        tk.key[KMAX - 1] = -INFINITY;
        tk.idx[KMAX - 1] = 0x7fffffff;
      }
    } else {
      sel_key[s] = -INFINITY;
      sel_idx[s] = 0;
    }
  }

  // ---- gate weights of the selected experts
  float wsel[KMAX];
  float denom = 0.f;
  if (p.gating == 0 || p.gating == 3) {
    // softmax over all E, keep the selected probabilities (rule 0 then
    // renormalises them, rule 3 keeps them as they are)
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float z = 0.f;
    for (int e = lane; e < E; e += 32) z += expf(logits[e] + (p.bias ? p.bias[e] : 0.f) - mx);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
#pragma unroll
    for (int s = 0; s < KMAX; ++s) {
      wsel[s] = (s < k) ? expf(sel_key[s] - mx) / z : 0.f;
      denom += wsel[s];
    }
  } else if (p.gating == 1) {
    // softmax over the k kept kappas
#pragma unroll
    for (int s = 0; s < KMAX; ++s) {
      wsel[s] = (s < k) ? expf(sel_key[s] - sel_key[0]) : 0.f;
      denom += wsel[s];
    }
  } else {
    // sigmoid score, normalised over the selected set
#pragma unroll
    for (int s = 0; s < KMAX; ++s) {
      if (s < k) {
        const float sc = p.bias_select_only ? logits[sel_idx[s]] : sel_key[s];
        wsel[s] = 1.0f / (1.0f + expf(-sc));
      } else {
        wsel[s] = 0.f;
      }
      denom += wsel[s];
    }
  }
#pragma unroll
  for (int s = 0; s < KMAX; ++s) {
    if (s < k && lane == s) {
      p.ids[t * k + s] = sel_idx[s];
      p.wts[t * k + s] = p.gating == 3 ? wsel[s] : wsel[s] / denom;
    }
  }
}

// Small batches: one block per token; its eight warps split the experts (one
// full dot product per warp at a time, lanes over d), so a handful of tokens
// still spreads over many SMs and nothing is staged; warp 0 then selects.
template <typename T, int KMAX>
__global__ void __launch_bounds__(kThreads) router_topk_token_block_kernel(RouterParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  float* logits = reinterpret_cast<float*>(smem);  // [E]
  constexpr int V = Vec16<T>::N;
  const int d = p.d, E = p.E;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const T* __restrict__ x = static_cast<const T*>(p.x);
  const T* __restrict__ w = static_cast<const T*>(p.w);
  if (threadIdx.x == 0) grid_launch_dependents();  // the dispatch may be scheduled (it waits for these ids)
  for (int64_t t = blockIdx.x; t < p.T; t += gridDim.x) {
    const T* xr = x + t * d;
    for (int e = warp; e < E; e += kWarps) {
      const T* wr = w + (int64_t)e * d;
      float acc = 0.f;
#pragma unroll 4
      for (int i0 = lane * V; i0 < d; i0 += 32 * V) {
        const Vec16<T> xv = ld16(xr + i0), wv = ld16(wr + i0);
#pragma unroll
        for (int v = 0; v < V; ++v) acc = fmaf(Elem<T>::to_f(xv.v[v]), Elem<T>::to_f(wv.v[v]), acc);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (lane == 0) logits[e] = acc;
    }
    __syncthreads();
    if (warp == 0) select_and_weigh<KMAX>(p, logits, t, lane);
    __syncthreads();
  }
}

// Shared memory: logit rows [kWarps][E], with AUX the per-warp penalty sums
// [kWarps][E] and [kWarps], then W_r [E][d] when staged.
__host__ __device__ inline size_t router_smem_head(int E, bool aux) {
  return sizeof(float) * kWarps * (size_t)E * (aux ? 2 : 1) + (aux ? sizeof(float) * kWarps : 0);
}

template <typename T, bool W_SMEM, int KMAX, bool AUX>
__global__ void __launch_bounds__(kThreads) router_topk_simt_kernel(RouterParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int V = Vec16<T>::N;
  const int d = p.d, E = p.E;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const T* __restrict__ x = static_cast<const T*>(p.x);
  const T* __restrict__ wg = static_cast<const T*>(p.w);

  float* logits = reinterpret_cast<float*>(smem) + warp * E;      // [kWarps][E]
  float* p_sum = reinterpret_cast<float*>(smem) + kWarps * E;     // AUX: [kWarps][E]
  float* z_sum = p_sum + kWarps * E;                              // AUX: [kWarps]
  T* sw = reinterpret_cast<T*>(smem + router_smem_head(E, AUX));  // [E][d] when staged
  if (AUX) {
    for (int i = threadIdx.x; i < kWarps * E; i += kThreads) p_sum[i] = 0.f;
    if (threadIdx.x < kWarps) z_sum[threadIdx.x] = 0.f;
    __syncthreads();
  }
  if (W_SMEM) {  // eight 16-byte loads in flight per thread: W_r crosses from L2 in few round trips
    const int64_t n16 = (int64_t)E * d / V;
    const uint4* src = reinterpret_cast<const uint4*>(wg);
    uint4* dst = reinterpret_cast<uint4*>(sw);
    int64_t i = threadIdx.x;
    for (; i + 7 * kThreads < n16; i += 8 * kThreads) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = __ldg(src + i + u * kThreads);
#pragma unroll
      for (int u = 0; u < 8; ++u) dst[i + u * kThreads] = v[u];
    }
    for (; i < n16; i += kThreads) dst[i] = __ldg(src + i);
    __syncthreads();
  }
  const T* wsrc = W_SMEM ? sw : wg;

  for (int64_t t = (int64_t)blockIdx.x * kWarps + warp; t < p.T; t += (int64_t)gridDim.x * kWarps) {
    const T* xr = x + t * d;
    // ---- Score: logits of all E experts, kGroup at a time
    for (int e0 = 0; e0 < E; e0 += kGroup) {
      float acc[kGroup];
#pragma unroll
      for (int j = 0; j < kGroup; ++j) acc[j] = 0.f;
      auto fma_chunk = [&](const Vec16<T>& xv, int i0) {
        float xf[V];
#pragma unroll
        for (int v = 0; v < V; ++v) xf[v] = Elem<T>::to_f(xv.v[v]);
#pragma unroll
        for (int j = 0; j < kGroup; ++j) {
          if (e0 + j < E) {
            Vec16<T> wv;
            const T* wp = wsrc + (int64_t)(e0 + j) * d + i0;
            if (W_SMEM) *reinterpret_cast<uint4*>(wv.v) = *reinterpret_cast<const uint4*>(wp);
            else wv = ld16(wp);
#pragma unroll
            for (int v = 0; v < V; ++v) acc[j] = fmaf(xf[v], Elem<T>::to_f(wv.v[v]), acc[j]);
          }
        }
      };
      // eight row chunks in flight per lane: the x row streams from HBM
      // (with a token or two per warp the row's latency is the cost)
      int i0 = lane * V;
      for (; i0 + 7 * 32 * V < d; i0 += 8 * 32 * V) {
        Vec16<T> xv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) xv[u] = ld16(xr + i0 + u * 32 * V);
#pragma unroll
        for (int u = 0; u < 8; ++u) fma_chunk(xv[u], i0 + u * 32 * V);
      }
      for (; i0 < d; i0 += 32 * V) fma_chunk(ld16(xr + i0), i0);
#pragma unroll
      for (int j = 0; j < kGroup; ++j)
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], off);
      float mine = acc[0];
#pragma unroll
      for (int j = 1; j < kGroup; ++j) mine = (lane == j) ? acc[j] : mine;
      if (lane < kGroup && e0 + lane < E) logits[e0 + lane] = mine;
    }
    __syncwarp();

    if (AUX) {
      // penalties on the bias-free logits: softmax probabilities per expert and
      // the squared log-sum-exp, summed over this warp's tokens in token order
      float m = -INFINITY;
      for (int e = lane; e < E; e += 32) m = fmaxf(m, logits[e]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      float se = 0.f;
      for (int e = lane; e < E; e += 32) se += expf(logits[e] - m);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) se += __shfl_xor_sync(0xffffffffu, se, off);
      const float inv = 1.0f / se;
      for (int e = lane; e < E; e += 32) p_sum[warp * E + e] += expf(logits[e] - m) * inv;
      if (lane == 0) {
        const float lse = m + logf(se);
        z_sum[warp] += lse * lse;
      }
    }

    select_and_weigh<KMAX>(p, logits, t, lane);
    __syncwarp();
  }
  if (AUX) {  // this block's sums, warps added in a fixed order
    __syncthreads();
    float* out = p.aux_part + (int64_t)blockIdx.x * (E + 1);
    for (int e = threadIdx.x; e < E; e += kThreads) {
      float v = 0.f;
      for (int w = 0; w < kWarps; ++w) v += p_sum[w * E + e];
      out[e] = v;
    }
    if (threadIdx.x == 0) {
      float v = 0.f;
      for (int w = 0; w < kWarps; ++w) v += z_sum[w];
      out[E] = v;
    }
  }
}

// out[0] = E * sum_e (counts[e] / sum counts) * (P_e / T), out[1] = Z / T, where
// P_e and Z sum the per-block partials in block order.  One block.
constexpr int kAuxThreads = 1024;
__global__ void __launch_bounds__(kAuxThreads) router_aux_finalize_kernel(const float* __restrict__ part, int blocks,
                                                                          int E, int64_t T,
                                                                          const int32_t* __restrict__ counts,
                                                                          float* out) {
  __shared__ float red[kAuxThreads / 32];
  float fp = 0.f;
  for (int e = threadIdx.x; e < E; e += kAuxThreads) {
    float pe = 0.f;
    for (int b = 0; b < blocks; ++b) pe += part[(int64_t)b * (E + 1) + e];
    fp += (float)counts[e] * pe;
  }
  // block sum of counts * P: fixed shuffle tree, then the warps in order
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) fp += __shfl_xor_sync(0xffffffffu, fp, off);
  if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = fp;
  __syncthreads();
  if (threadIdx.x == 0) {
    float fptot = 0.f;
    for (int w = 0; w < kAuxThreads / 32; ++w) fptot += red[w];
    int64_t ctot = 0;
    for (int e = 0; e < E; ++e) ctot += counts[e];
    float z = 0.f;
    for (int b = 0; b < blocks; ++b) z += part[(int64_t)b * (E + 1) + E];
    out[0] = ctot > 0 ? (float)((double)E * (double)fptot / ((double)ctot * (double)T)) : 0.f;
    out[1] = z / (float)T;
  }
}

template <typename T, bool W_SMEM, bool AUX>
cudaError_t launch_t(const RouterParams& p, int64_t max_blocks, int64_t* blocks_out, cudaStream_t stream) {
  const size_t smem = router_smem_head(p.E, AUX) + (W_SMEM ? (size_t)p.E * p.d * sizeof(T) : 0);
  const int sms = device_sm_count();
  int64_t blocks = (p.T + kWarps - 1) / kWarps;
  int64_t cap = (int64_t)sms * (W_SMEM ? 2 : 8);
  if (cap > max_blocks) cap = max_blocks;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  if (blocks_out) *blocks_out = blocks;
  auto run = [&](auto kernel) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kernel<<<(unsigned)blocks, kThreads, smem, stream>>>(p);
    return cudaGetLastError();
  };
  if (p.k <= 2) return run(router_topk_simt_kernel<T, W_SMEM, 2, AUX>);
  if (p.k <= 4) return run(router_topk_simt_kernel<T, W_SMEM, 4, AUX>);
  if (p.k <= 8) return run(router_topk_simt_kernel<T, W_SMEM, 8, AUX>);
  return run(router_topk_simt_kernel<T, W_SMEM, 16, AUX>);
}

// W_r is staged in shared memory when it fits next to the logit rows.
constexpr size_t kRouterSmemBudget = 160 * 1024;

// Batches up to this many tokens use one block per token.
constexpr int64_t kTokenBlockMaxT = 64;

template <typename T>
cudaError_t launch_token_block(const RouterParams& p, cudaStream_t stream) {
  const size_t smem = sizeof(float) * p.E;
  auto run = [&](auto kernel) -> cudaError_t {
    kernel<<<(unsigned)p.T, kThreads, smem, stream>>>(p);
    return cudaGetLastError();
  };
  if (p.k <= 2) return run(router_topk_token_block_kernel<T, 2>);
  if (p.k <= 4) return run(router_topk_token_block_kernel<T, 4>);
  if (p.k <= 8) return run(router_topk_token_block_kernel<T, 8>);
  return run(router_topk_token_block_kernel<T, 16>);
}

template <bool AUX>
cudaError_t launch_simt(const RouterArgs& a, int64_t max_blocks, int64_t* blocks, cudaStream_t stream) {
  RouterParams p{a.x, a.w_router, a.bias, a.ids, a.w, a.T, a.d, a.E, a.k, a.gating, a.bias_select_only, a.aux_part};
  if (!AUX && a.T <= kTokenBlockMaxT)
    return a.bf16 ? launch_token_block<__nv_bfloat16>(p, stream) : launch_token_block<float>(p, stream);
  const size_t eb = a.bf16 ? 2 : 4;
  const bool fits = router_smem_head(a.E, AUX) + (size_t)a.E * a.d * eb <= kRouterSmemBudget;
  if (a.bf16)
    return fits ? launch_t<__nv_bfloat16, true, AUX>(p, max_blocks, blocks, stream)
                : launch_t<__nv_bfloat16, false, AUX>(p, max_blocks, blocks, stream);
  return fits ? launch_t<float, true, AUX>(p, max_blocks, blocks, stream)
              : launch_t<float, false, AUX>(p, max_blocks, blocks, stream);
}

}  // namespace

cudaError_t launch_router_topk_simt(const RouterArgs& a, cudaStream_t stream) {
  return launch_simt<false>(a, INT64_MAX, nullptr, stream);
}

cudaError_t launch_router_aux_losses(const RouterArgs& a, const int32_t* counts, float* out, cudaStream_t stream) {
  if (a.aux_part == nullptr) return cudaErrorInvalidValue;
  int64_t blocks = 0;
  cudaError_t e = launch_simt<true>(a, kAuxMaxBlocks, &blocks, stream);
  if (e != cudaSuccess) return e;
  router_aux_finalize_kernel<<<1, kAuxThreads, 0, stream>>>(a.aux_part, (int)blocks, a.E, a.T, counts, out);
  return cudaGetLastError();
}

}  // namespace moe
