// Dispatch: a stable counting sort of the T*k (token, slot) assignments by
// expert, then the row gather x_perm[row] = x[perm[row] / k].
//
// "Mixture of Experts: why a model with 671 billion parameters uses only 37",
// "Capacity factor: when tokens don't fit" (dropless: each expert gets exactly
// the rows the router assigned; with a capacity, tokens beyond an expert's
// buffer skip it) and "How data centres handle it" (tokens are grouped by
// their assigned expert before the expert multiplies).  The capacity rule is
// that of "Mixture of Experts Explained: Routers, Active Parameters and VRAM"
// (expert capacity): an expert keeps its first C assignments in token order.
//
// Three small kernels keep the result deterministic and stable without any
// global atomics on positions:
//   count   : per chunk of kChunk assignments, a shared-memory histogram
//             -> chunk_counts[chunk][e] (chunk-major, so that the scan's
//             threads, one per expert, read each chunk's row coalesced)
//   scan    : one block turns the histograms into counts, exclusive offsets
//             of the kept rows (min(count, C) per expert) and per-(expert,
//             chunk) starting ranks
//   scatter : each warp walks its slice of the chunk in order; ranks among
//             equal experts come from __match_any_sync, so an expert's
//             assignments are ranked in ascending index t*k+s; rank r < C
//             lands on row offsets[e] + r, the rest are dropped (row -1)
// and a gather kernel that moves whole rows with 16-byte loads/stores.
#include "common.cuh"
#include "kernels.cuh"
#include "pdl.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kPerWarp = 256;                 // assignments per warp slice
constexpr int kChunk = kWarps * kPerWarp;     // assignments per block

__global__ void __launch_bounds__(kThreads) permute_count_kernel(const int32_t* __restrict__ ids, int64_t n,
                                                                 int E, int32_t* chunk_counts, int n_chunks,
                                                                 int* status) {
  extern __shared__ int hist[];
  for (int e = threadIdx.x; e < E; e += kThreads) hist[e] = 0;
  __syncthreads();
  const int64_t base = (int64_t)blockIdx.x * kChunk;
  const int64_t end = min(base + kChunk, n);
  for (int64_t i = base + threadIdx.x; i < end; i += kThreads) {
    const int e = ids[i];
    if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
    else set_status(status, kDevBadExpertId);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kThreads) chunk_counts[(int64_t)blockIdx.x * E + e] = hist[e];
}

// one block of kScanThreads >= E threads
constexpr int kScanThreads = 1024;
__global__ void __launch_bounds__(kScanThreads) permute_scan_kernel(int32_t* chunk_counts, int n_chunks, int E,
                                                                    int32_t* counts, int32_t* offsets,
                                                                    int64_t capacity) {
  __shared__ int warp_sums[kScanThreads / 32];
  const int e = threadIdx.x, lane = e % 32, warp = e / 32;
  int total = 0;
  if (e < E) {  // eight independent loads in flight per thread
    int b = 0;
    for (; b + 8 <= n_chunks; b += 8) {
      int c[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) c[i] = chunk_counts[(int64_t)(b + i) * E + e];
#pragma unroll
      for (int i = 0; i < 8; ++i) total += c[i];
    }
    for (; b < n_chunks; ++b) total += chunk_counts[(int64_t)b * E + e];
  }
  const int kept = (int)min((int64_t)total, capacity);
  // block-wide exclusive scan of the rows each expert keeps
  int incl = kept;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int s = warp_sums[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, s, off);
      if (lane >= off) s += v;
    }
    warp_sums[lane] = s;  // inclusive over warps
  }
  __syncthreads();
  const int excl = incl - kept + (warp > 0 ? warp_sums[warp - 1] : 0);
  if (e < E) {
    counts[e] = total;
    offsets[e] = excl;
    if (e == E - 1) offsets[E] = excl + kept;
    int run = 0;  // per-chunk starting ranks of expert e
    int b = 0;
    for (; b + 8 <= n_chunks; b += 8) {
      int c[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) c[i] = chunk_counts[(int64_t)(b + i) * E + e];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        chunk_counts[(int64_t)(b + i) * E + e] = run;
        run += c[i];
      }
    }
    for (; b < n_chunks; ++b) {
      const int c = chunk_counts[(int64_t)b * E + e];
      chunk_counts[(int64_t)b * E + e] = run;
      run += c;
    }
  }
}

__global__ void __launch_bounds__(kThreads) permute_scatter_kernel(const int32_t* __restrict__ ids, int64_t n,
                                                                   int E, const int32_t* __restrict__ chunk_base,
                                                                   int n_chunks, const int32_t* __restrict__ offsets,
                                                                   int64_t capacity, int32_t* perm, int32_t* row_of) {
  extern __shared__ int wc[];  // [kWarps][E]: per-warp counts, then per-warp next row
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int i = threadIdx.x; i < kWarps * E; i += kThreads) wc[i] = 0;
  __syncthreads();
  const int64_t slice = (int64_t)blockIdx.x * kChunk + (int64_t)warp * kPerWarp;
  int* mine = wc + warp * E;
  // pass 1: per-warp histogram, one update per distinct expert per round
  for (int r = 0; r < kPerWarp / 32; ++r) {
    const int64_t i = slice + r * 32 + lane;
    int e = (i < n) ? ids[i] : -1;
    if (e >= E) e = -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(peers) - 1) mine[e] += __popc(peers);
  }
  __syncthreads();
  // per expert: exclusive scan over the warps, starting at this chunk's base rank
  for (int e = threadIdx.x; e < E; e += kThreads) {
    int run = chunk_base[(int64_t)blockIdx.x * E + e];
    for (int w = 0; w < kWarps; ++w) {
      const int c = wc[w * E + e];
      wc[w * E + e] = run;
      run += c;
    }
  }
  __syncthreads();
  // pass 2: ranks inside each round follow lane order, rounds follow index order
  const unsigned lt = (1u << lane) - 1u;
  for (int r = 0; r < kPerWarp / 32; ++r) {
    const int64_t i = slice + r * 32 + lane;
    const bool in = i < n;
    int e = in ? ids[i] : -1;
    if (e >= E) e = -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    int row = -1;
    if (e >= 0) {
      const int rank = mine[e] + __popc(peers & lt);  // among expert e's assignments, in index order
      if (rank < capacity) row = offsets[e] + rank;
    }
    __syncwarp();
    if (e >= 0 && lane == __ffs(peers) - 1) mine[e] += __popc(peers);
    __syncwarp();
    if (in) {
      row_of[i] = row;  // -1 for an id outside [0, E) or a slot beyond the capacity
      if (row >= 0) perm[row] = (int32_t)i;
    }
  }
}

// Small dispatch (at most kSmallDispatch assignments, the decode regime): the
// histogram, the scan and the stable scatter in one block -- a shared-memory
// histogram, one block scan over the experts, then warp 0 walks the
// assignments in index order, 32 per round, ranking equal experts with
// __match_any_sync.  Same results as the three kernels above, two launches
// fewer.
constexpr int64_t kSmallDispatch = 1024;
constexpr int kSmallThreads = 1024;  // >= kMaxExperts: one expert per thread in the scan

__global__ void __launch_bounds__(kSmallThreads)
    permute_small_kernel(const int32_t* __restrict__ ids, int64_t n, int E, int64_t capacity, int32_t* counts,
                         int32_t* offsets, int32_t* perm, int32_t* row_of, int* status) {
  extern __shared__ int sm[];  // hist[E], base[E], run[E]
  __shared__ int warp_sums[kSmallThreads / 32];
  int* hist = sm;
  int* base = sm + E;
  int* run = sm + 2 * E;
  const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
  grid_dependency_wait();  // the router's ids (programmatic launch)
  if (tid == 0) grid_launch_dependents();
  for (int e = tid; e < E; e += kSmallThreads) {
    hist[e] = 0;
    run[e] = 0;
  }
  __syncthreads();
  for (int64_t i = tid; i < n; i += kSmallThreads) {
    const int e = ids[i];
    if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
    else set_status(status, kDevBadExpertId);
  }
  __syncthreads();
  // exclusive scan of the rows each expert keeps
  const int total = tid < E ? hist[tid] : 0;
  const int kept = (int)min((int64_t)total, capacity);
  int incl = kept;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int v = warp_sums[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += u;
    }
    warp_sums[lane] = v;
  }
  __syncthreads();
  const int excl = incl - kept + (warp > 0 ? warp_sums[warp - 1] : 0);
  if (tid < E) {
    counts[tid] = total;
    offsets[tid] = excl;
    base[tid] = excl;
    if (tid == E - 1) offsets[E] = excl + kept;
  }
  __syncthreads();
  if (warp == 0) {
    const unsigned lt = (1u << lane) - 1u;
    for (int64_t r0 = 0; r0 < n; r0 += 32) {
      const int64_t i = r0 + lane;
      const bool in = i < n;
      int e = in ? ids[i] : -1;
      if (e >= E || e < 0) e = -1;
      const unsigned peers = __match_any_sync(0xffffffffu, e);
      int row = -1;
      if (e >= 0) {
        const int rank = run[e] + __popc(peers & lt);
        if (rank < capacity) row = base[e] + rank;
      }
      __syncwarp();
      if (e >= 0 && lane == __ffs(peers) - 1) run[e] += __popc(peers);
      __syncwarp();
      if (in) {
        row_of[i] = row;
        if (row >= 0) perm[row] = (int32_t)i;
      }
    }
  }
}

// Mid-size dispatch (at most kMidDispatch assignments over at most
// kMidExperts experts, such as a 2048-token batch with k = 2): one block as
// well, with every warp ranking.  Warp w owns a contiguous segment of the
// assignments and counts it per expert (__match_any_sync: one add per
// distinct expert and round); a scan over the experts gives the offsets and
// one over the warps each warp's first rank per expert; then each warp walks
// its segment again in order and ranks from there.  An assignment's rank is
// the number of earlier assignments of its expert, so the scatter is stable
// and equal to the kernels above, in one launch instead of three.
constexpr int64_t kMidDispatch = 8192;
constexpr int kMidExperts = 64;
constexpr int kMidWarps = kSmallThreads / 32;

__global__ void __launch_bounds__(kSmallThreads)
    permute_mid_kernel(const int32_t* __restrict__ ids, int64_t n, int E, int64_t capacity, int32_t* counts,
                       int32_t* offsets, int32_t* perm, int32_t* row_of, int* status) {
  __shared__ int wrank[kMidWarps][kMidExperts];  // per warp and expert: its count, then its first rank
  __shared__ int base[kMidExperts];
  __shared__ int warp_sums[kMidWarps];
  const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
  grid_dependency_wait();  // the router's ids (programmatic launch)
  if (tid == 0) grid_launch_dependents();
  for (int e = lane; e < kMidExperts; e += 32) wrank[warp][e] = 0;
  __syncwarp();
  const int64_t seg = ((n + kMidWarps - 1) / kMidWarps + 31) / 32 * 32;  // a multiple of 32
  const int64_t lo = (int64_t)warp * seg, hi = min(n, lo + seg);
  const unsigned lt = (1u << lane) - 1u;
  for (int64_t r0 = lo; r0 < hi; r0 += 32) {
    const int64_t i = r0 + lane;
    int e = -1;
    if (i < hi) {
      e = ids[i];
      if (e < 0 || e >= E) {
        set_status(status, kDevBadExpertId);
        e = -1;
      }
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(peers) - 1) wrank[warp][e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // per expert (a thread each): the total, and each warp's first rank
  int total = 0;
  if (tid < E) {
    for (int w = 0; w < kMidWarps; ++w) {
      const int c = wrank[w][tid];
      wrank[w][tid] = total;
      total += c;
    }
  }
  // exclusive scan of the rows each expert keeps
  const int kept = (int)min((int64_t)total, capacity);
  int incl = kept;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int v = warp_sums[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += u;
    }
    warp_sums[lane] = v;
  }
  __syncthreads();
  const int excl = incl - kept + (warp > 0 ? warp_sums[warp - 1] : 0);
  if (tid < E) {
    counts[tid] = total;
    offsets[tid] = excl;
    base[tid] = excl;
    if (tid == E - 1) offsets[E] = excl + kept;
  }
  __syncthreads();
  for (int64_t r0 = lo; r0 < hi; r0 += 32) {
    const int64_t i = r0 + lane;
    const bool in = i < hi;
    int e = in ? ids[i] : -1;
    if (e < 0 || e >= E) e = -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    int row = -1;
    if (e >= 0) {
      const int rank = wrank[warp][e] + __popc(peers & lt);
      if (rank < capacity) row = base[e] + rank;
    }
    __syncwarp();
    if (e >= 0 && lane == __ffs(peers) - 1) wrank[warp][e] += __popc(peers);
    __syncwarp();
    if (in) {
      row_of[i] = row;
      if (row >= 0) perm[row] = (int32_t)i;
    }
  }
}

// x_perm[row_of[t*k + s]] = x[t] for every kept slot s of token t.  Token
// major: one warp per token reads the token's vector once (16-byte vectors,
// four in flight per lane) and writes it to each of its rows, so x crosses
// HBM once however many experts a token picked (walking the rows in dispatch
// order instead re-reads x from HBM once its k copies have pushed it out of L2).
__global__ void __launch_bounds__(kThreads) gather_rows_kernel(const uint8_t* __restrict__ x,
                                                               const int32_t* __restrict__ row_of, int64_t T,
                                                               int k, int64_t row_bytes, uint8_t* x_perm) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t n16 = row_bytes / 16;
  grid_dependency_wait();  // row_of of the dispatch (programmatic launch)
  if (threadIdx.x == 0) grid_launch_dependents();
  for (int64_t t = (int64_t)blockIdx.x * kWarps + warp; t < T; t += (int64_t)gridDim.x * kWarps) {
    const int my_row = lane < k ? row_of[t * k + lane] : -1;  // k <= kMaxTopK <= 32
    const uint4* src = reinterpret_cast<const uint4*>(x + t * row_bytes);
    for (int64_t j0 = 0; j0 < n16; j0 += 128) {  // the same trip count on every lane (shuffles inside)
      const int64_t j = j0 + lane;
      uint4 a[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (j + 32 * i < n16) a[i] = __ldg(src + j + 32 * i);
      for (int s = 0; s < k; ++s) {
        const int row = __shfl_sync(0xffffffffu, my_row, s);
        if (row < 0) continue;  // dropped by the capacity
        uint4* dst = reinterpret_cast<uint4*>(x_perm + (int64_t)row * row_bytes);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (j + 32 * i < n16) dst[j + 32 * i] = a[i];
      }
    }
  }
}

}  // namespace

int permute_n_chunks(int64_t n_assign) { return (int)((n_assign + kChunk - 1) / kChunk); }

cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t stream) {
  const int n_chunks = permute_n_chunks(a.n_assign);
  if (n_chunks == 0) {
    // no assignments: zero counts and offsets
    cudaError_t e = cudaMemsetAsync(a.counts, 0, sizeof(int32_t) * a.E, stream);
    if (e != cudaSuccess) return e;
    return cudaMemsetAsync(a.offsets, 0, sizeof(int32_t) * (a.E + 1), stream);
  }
  if (a.n_assign <= kSmallDispatch) {
    const cudaError_t e = launch_maybe_chained(permute_small_kernel, dim3(1), dim3(kSmallThreads),
                                               3 * sizeof(int) * a.E, stream, a.chained, a.ids, a.n_assign, a.E,
                                               a.capacity, a.counts, a.offsets, a.perm, a.row_of, a.status);
    if (e != cudaSuccess) return e;
  } else if (a.n_assign <= kMidDispatch && a.E <= kMidExperts) {
    const cudaError_t e = launch_maybe_chained(permute_mid_kernel, dim3(1), dim3(kSmallThreads), 0, stream,
                                               a.chained, a.ids, a.n_assign, a.E, a.capacity, a.counts, a.offsets,
                                               a.perm, a.row_of, a.status);
    if (e != cudaSuccess) return e;
  } else {
    permute_count_kernel<<<n_chunks, kThreads, sizeof(int) * a.E, stream>>>(a.ids, a.n_assign, a.E,
                                                                            a.chunk_counts, n_chunks, a.status);
    permute_scan_kernel<<<1, kScanThreads, 0, stream>>>(a.chunk_counts, n_chunks, a.E, a.counts, a.offsets,
                                                        a.capacity);
    permute_scatter_kernel<<<n_chunks, kThreads, sizeof(int) * kWarps * a.E, stream>>>(
        a.ids, a.n_assign, a.E, a.chunk_counts, n_chunks, a.offsets, a.capacity, a.perm, a.row_of);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || a.x == nullptr || a.x_perm == nullptr) return e;
  const int64_t T = a.n_assign / a.k;
  int64_t blocks = (T + kWarps - 1) / kWarps;
  const int64_t cap = (int64_t)device_sm_count() * 16;
  if (blocks > cap) blocks = cap;
  return launch_maybe_chained(gather_rows_kernel, dim3((unsigned)blocks), dim3(kThreads), 0, stream, a.chained,
                              static_cast<const uint8_t*>(a.x), a.row_of, T, a.k, (int64_t)a.d * a.elem_bytes,
                              static_cast<uint8_t*>(a.x_perm));
}

}  // namespace moe
