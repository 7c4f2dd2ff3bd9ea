// Grouped expert GEMMs on CTA pairs (tcgen05 cta_group::2 + TMEM + TMA).
//
// "Mixture of Experts: why a model with 671 billion parameters uses only 37",
// "How data centres handle it": tokens grouped by their assigned expert and
// all expert multiplies run in a single launch over a stacked weight matrix.
// Expert FFN: "Mixture of Experts Explained: Routers, Active Parameters and
// VRAM" (a gated feed-forward block with three matrices), read as SwiGLU.
//
// A cluster of two CTAs (a pair, on two SMs) owns one output tile at a time:
// 256 token rows (128 per CTA) x 256 accumulator columns, computed by
// M = 256 pair MMAs that the pair's first CTA (the leader) issues.  Each CTA
// loads only its own operands with plain (non-multicast) TMA: its 128 rows of
// A and its half of B (128 of the 256 B rows); the pair MMA reads both CTAs'
// shared memory, so every B byte crosses L2 -> SM once per pair instead of
// once per CTA, and the MMA runs at the full tensor rate of both SMs.
//
//   GEMM-1 (MODE_SWIGLU): h[rows, f] = SiLU(A Wg^T) * (A Wu^T).  A tile's 256
//     B rows are [gate 64 | up 64] in the leader and the next [gate 64 | up
//     64] in the peer, so every accumulator row holds each gate column next to
//     its up column (64 apart) and the SwiGLU runs in the epilogue straight
//     out of tensor memory: 128 h columns per tile.
//   GEMM-1 (MODE_GELU, the two-matrix expert): h = GELU(A Wu^T), 256 columns.
//   GEMM-2 (MODE_PLAIN):  y[rows, d] = h Wd^T, 256 columns.
//
// Padding: an expert's rows are cut into 256-row blocks; a last block of at
// most 128 rows runs as a half-height pair tile (M = 128 pair MMAs, 64 rows
// per CTA), so no expert pads more than 127 rows.  In a half tile each CTA's
// 64 x 256 accumulator is folded into tensor memory as 128 lanes x 128
// columns: lanes 0-63 hold accumulator columns 0-127 of the CTA's 64 rows,
// lanes 64-127 columns 128-255.
//
// Per CTA (both CTAs run the same roles; only the leader issues MMAs):
//   warp 0     TMA producer: 6-stage ring of (A 128x64, B-half 128x64) bf16
//              (128x128 with 8-bit operands), 128-byte swizzle; completion
//              counted on the leader's stage barrier
//   warp 1     TMEM allocator (both CTAs, cta_group::2); in the leader the
//              single-thread pair-MMA issuer
//   warps 2..  epilogue: tcgen05.ld of the CTA's own accumulator rows,
//              SwiGLU / GELU / scales, bf16 stores; four warps in bf16,
//              eight with 8-bit operands
// Two 256-column accumulators (all 512 TMEM columns) per CTA let a tile's
// epilogue overlap the next tile's main loop.
//
// Barriers: the leader's full[s] counts both CTAs' TMA bytes of stage s; the
// leader's MMA commit arrives on both CTAs' empty[s] (one commit signalling
// both) and, at the end of a tile, on both CTAs' tfull[acc]; the epilogue warps
// of both CTAs arrive on the leader's tempty[acc].  Every wait is bounded
// (Params::wait_limit_ns); on expiry a CTA raises the device status word,
// lets its own copies land, and both CTAs meet at a cluster barrier before
// they free their tensor memory and exit.
#include <cudaTypedefs.h>

#include "kernels.cuh"
#include "tc_primitives.cuh"

namespace moe {
namespace tc {
namespace pair {

constexpr int STAGES = 6;
constexpr int ROWS = 128;                  // A rows per CTA (a full tile has 256 per pair)
constexpr int A_BYTES = ROWS * 128;        // 16 KiB: 128 rows x one 128-byte K slice
constexpr int B_BYTES = 128 * 128;         // 16 KiB: this CTA's 128 B rows
constexpr int TMEM_COLS = 512;
constexpr int ACC_COLS = 256;
constexpr int MODE_SWIGLU = 0, MODE_PLAIN = 1, MODE_GELU = 3;
constexpr int kMBlock = 8;                 // 256-row blocks per walk block of a hot expert (2048 rows)

template <bool FP8>
constexpr int kThreads = FP8 ? 320 : 192;

struct Params {
  const int32_t* offsets;  // [G+1] device, or null: one group of `rows` rows
  int G;
  int64_t rows;            // rows of A and of the output
  int K;                   // reduction length
  int N;                   // output columns
  int nt;                  // n-tiles per group
  int64_t b_group_rows;    // rows of B per group (2f, f or d)
  int up_off;              // row offset of the up half inside a group (SwiGLU: f)
  void* out;
  int64_t ldo;
  int* status;
  uint64_t wait_limit_ns;
  const float* sa;         // 8-bit operands: per-row scales of A
  const float* sb;         //                 per-row scales of B (indexed like B's rows)
};

size_t smem_bytes(int G) {
  return 1024 + (size_t)STAGES * (A_BYTES + B_BYTES) + 256 + 2 * sizeof(int) * (size_t)(G + 1);
}

// m-blocks of 256 rows per group: cum[g] = m-blocks of groups before g
// tile t -> (group, m-block, n-tile): blocks of kMBlock m-blocks, then the
// n-tile, then the m-block (fastest), so the CTAs running together share a
// weight panel while one block of token rows stays in L2
__device__ __forceinline__ void decode_tile(int64_t t, int nt, const int* cum, int G, int& g, int& mb, int& ntile) {
  int lo = 0, hi = G;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if ((int64_t)cum[mid] * nt <= t) lo = mid;
    else hi = mid;
  }
  g = lo;
  const int mblocks = cum[lo + 1] - cum[lo];
  const int64_t local = t - (int64_t)cum[lo] * nt;
  const int blk = (int)(local / ((int64_t)kMBlock * nt));
  const int64_t rest = local - (int64_t)blk * kMBlock * nt;
  const int nb = min(kMBlock, mblocks - blk * kMBlock);
  ntile = (int)(rest / nb);
  mb = blk * kMBlock + (int)(rest % nb);
}

template <bool FP8>
__host__ __device__ constexpr uint32_t idesc_pair(int M, int N) {
  return idesc_f32acc<FP8>(M, N);
}

template <int MODE, bool FP8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads<FP8>, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA64,
                             const __grid_constant__ CUtensorMap tmB, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + STAGES * B_BYTES);
  uint64_t* full = bars;                   // leader: both CTAs' bytes of stage s
  uint64_t* empty = bars + STAGES;         // own: stage s free again
  uint64_t* tfull = bars + 2 * STAGES;     // own: accumulator a ready
  uint64_t* tempty = bars + 2 * STAGES + 2;  // leader: accumulator a drained by both CTAs
  uint64_t* drain = bars + 2 * STAGES + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* fill_par = reinterpret_cast<int*>(tmem_slot + 2);  // [STAGES]
  int* s_off = fill_par + STAGES;                          // [G+1]
  int* s_cum = s_off + (p.G + 1);                          // [G+1]

  constexpr int NT = kThreads<FP8>;
  constexpr int kEpiWarps = NT / 32 - 2;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int G = p.G;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair_id = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
      fill_par[s] = -1;
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&tfull[a]), 1);
      mbar_init(smem_u32(&tempty[a]), 2 * kEpiWarps);
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmA64);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (p.offsets) {
    for (int g = threadIdx.x; g <= G; g += NT) s_off[g] = p.offsets[g];
  } else if (threadIdx.x == 0) {
    s_off[0] = 0;
    s_off[1] = (int)p.rows;
  }
  __syncthreads();
  if (warp == 0) {  // cumulative 256-row m-block counts, 32 groups per step
    int carry = 0;
    if (lane == 0) s_cum[0] = 0;
    for (int base = 0; base < G; base += 32) {
      const int g = base + lane;
      int v = 0;
      if (g < G) v = max(0, (s_off[g + 1] - s_off[g] + 2 * ROWS - 1) / (2 * ROWS));
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += u;
      }
      if (g < G) s_cum[g + 1] = carry + v;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
  }
  // barrier initialisation and the tensor-memory allocation of both CTAs are
  // complete before either CTA touches the other's barriers or memory
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();

  const uint32_t tmem_base = *tmem_slot;
  const int64_t total = (int64_t)s_cum[G] * p.nt;
  constexpr int KB = FP8 ? 128 : 64;  // elements per 128-byte K slice
  const int kb_count = (p.K + KB - 1) / KB;
  const int bno = MODE == MODE_SWIGLU ? ACC_COLS / 2 : ACC_COLS;  // output columns per tile

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      for (int64_t t = pair_id; t < total; t += n_pairs) {
        int g, mb, ntile;
        decode_tile(t, p.nt, s_cum, G, g, mb, ntile);
        const int rows_t = min(2 * ROWS, s_off[g + 1] - s_off[g] - mb * 2 * ROWS);
        const bool half = rows_t <= ROWS;
        const int a_row = s_off[g] + mb * 2 * ROWS + (int)rank * (half ? ROWS / 2 : ROWS);
        const int64_t b_base = (int64_t)g * p.b_group_rows + (int64_t)ntile * bno;
        const uint32_t a_bytes = half ? A_BYTES / 2 : A_BYTES;
        bool ok = true;
        for (int kb = 0; kb < kb_count; ++kb) {
          if (!mbar_wait_bounded(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, p.wait_limit_ns, p.status)) {
            ok = false;
            break;
          }
          // the stage's bytes from both CTAs are counted on the leader's barrier
          if (leader) mbar_expect_tx(smem_u32(&full[stage]), 2 * (a_bytes + B_BYTES));
          const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
          fill_par[stage] = (int)phase;
          tma_load_2d_pair(smem_u32(sA + stage * A_BYTES), half ? &tmA64 : &tmA, fb, kb * KB, a_row);
          if (MODE == MODE_SWIGLU) {  // 64 gate rows, then the matching 64 up rows
            const int gr = (int)(b_base + 64 * rank);
            tma_load_2d_pair(smem_u32(sB + stage * B_BYTES), &tmB, fb, kb * KB, gr);
            tma_load_2d_pair(smem_u32(sB + stage * B_BYTES + 64 * 128), &tmB, fb, kb * KB, gr + p.up_off);
          } else {
            tma_load_2d_pair(smem_u32(sB + stage * B_BYTES), &tmB, fb, kb * KB, (int)(b_base + 128 * rank));
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------ pair-MMA issuer (leader)
      const uint32_t idesc_full = idesc_pair<FP8>(2 * ROWS, ACC_COLS);
      const uint32_t idesc_half = idesc_pair<FP8>(ROWS, ACC_COLS);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int64_t t = pair_id; t < total && ok; t += n_pairs) {
        int g, mb, ntile;
        decode_tile(t, p.nt, s_cum, G, g, mb, ntile);
        const int rows_t = min(2 * ROWS, s_off[g + 1] - s_off[g] - mb * 2 * ROWS);
        const uint32_t idesc = rows_t <= ROWS ? idesc_half : idesc_full;
        if (!mbar_wait_bounded(smem_u32(&tempty[acc]), acc_phase ^ 1u, abort_flag, p.wait_limit_ns, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * ACC_COLS);
        for (int kb = 0; kb < kb_count; ++kb) {
          if (!mbar_wait_bounded(smem_u32(&full[stage]), phase, abort_flag, p.wait_limit_ns, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          mma_kslice_pair<FP8>(d_tmem, smem_u32(sA + stage * A_BYTES), smem_u32(sB + stage * B_BYTES), idesc,
                               kb == 0);
          mma_commit_pair_both(smem_u32(&empty[stage]));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_pair_both(smem_u32(&tfull[acc]));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
    }
  } else {
    // -------------------------------------------------- epilogue (warps 2.., both CTAs)
    const int q = warp & 3;                        // TMEM lane quarter this warp may access
    constexpr int kPerQuarter = kEpiWarps / 4;     // epilogue warps per lane quarter
    const int part = (warp - 2) >> 2;              // which of them this warp is
    const int r = q * 32 + lane;                   // TMEM lane of this thread
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty[0]), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int64_t t = pair_id; t < total; t += n_pairs) {
      int g, mb, ntile;
      decode_tile(t, p.nt, s_cum, G, g, mb, ntile);
      if (!mbar_wait_bounded(smem_u32(&tfull[acc]), acc_phase, abort_flag, p.wait_limit_ns, p.status)) break;
      tc_fence_after();
      const int rows_g = s_off[g + 1] - s_off[g];
      const int rows_t = min(2 * ROWS, rows_g - mb * 2 * ROWS);
      const bool half = rows_t <= ROWS;
      // this thread's accumulator row and the accumulator-column half it holds
      //   full tile: lane r = row r of this CTA's 128, all 256 columns
      //   half tile: lane r = row (r mod 64) of this CTA's 64, columns 128*(r / 64) + [0, 128)
      const int lr = mb * 2 * ROWS + (half ? (int)rank * (ROWS / 2) + (r & 63) : (int)rank * ROWS + r);
      const int64_t grow = (int64_t)s_off[g] + lr;
      const bool ok = lr < rows_g && grow >= 0 && grow < p.rows;
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * ACC_COLS);
      const float s_row = FP8 && ok ? p.sa[grow] : 1.f;
      // accumulator-column halves this thread finishes: both (full tile) or one (half tile)
      const int h_lo = half ? (r >> 6) : 0, h_hi = half ? (r >> 6) : 1;
      for (int hh = h_lo; hh <= h_hi; ++hh) {
        const uint32_t tcol = half ? 0u : (uint32_t)(hh * 128);  // TMEM column of this half
        // output columns of this half: SwiGLU 64 h columns, else 128 columns
        const int ocols = MODE == MODE_SWIGLU ? 64 : 128;
        const int col_base = ntile * bno + hh * ocols;
        const int col_lim = min(p.N, col_base + ocols);
        __nv_bfloat16* orow = out + grow * p.ldo + col_base;
        const float* sg = FP8 ? p.sb + (int64_t)g * p.b_group_rows + col_base : nullptr;
#pragma unroll 1
        for (int c = 32 * part; c < ocols; c += 32 * kPerQuarter) {
          uint32_t v[32], u[32];
          tmem_ld32(tb + tcol + c, v);
          if (MODE == MODE_SWIGLU) tmem_ld32(tb + tcol + 64 + c, u);
          tmem_ld_wait();
          if (ok && col_base + c < col_lim) {
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              float h0 = __uint_as_float(v[2 * j]), h1 = __uint_as_float(v[2 * j + 1]);
              float u0 = MODE == MODE_SWIGLU ? __uint_as_float(u[2 * j]) : 0.f;
              float u1 = MODE == MODE_SWIGLU ? __uint_as_float(u[2 * j + 1]) : 0.f;
              if (FP8) {  // columns past N read no scale (their outputs are never stored)
                const int c0 = col_base + c + 2 * j;
                h0 *= s_row * (c0 < col_lim ? sg[c + 2 * j] : 0.f);
                h1 *= s_row * (c0 + 1 < col_lim ? sg[c + 2 * j + 1] : 0.f);
                if (MODE == MODE_SWIGLU) {
                  u0 *= s_row * (c0 < col_lim ? sg[p.up_off + c + 2 * j] : 0.f);
                  u1 *= s_row * (c0 + 1 < col_lim ? sg[p.up_off + c + 2 * j + 1] : 0.f);
                }
              }
              if (MODE == MODE_SWIGLU) {
                h0 = silu_f(h0) * u0;
                h1 = silu_f(h1) * u1;
              }
              if (MODE == MODE_GELU) {
                h0 = gelu_f(h0);
                h1 = gelu_f(h1);
              }
              pk[j] = pack_bf16x2(h0, h1);
            }
            if (col_base + c + 32 <= col_lim) {
              uint4* dst = reinterpret_cast<uint4*>(orow + c);
#pragma unroll
              for (int j = 0; j < 4; ++j) dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const int cc = col_base + c + 2 * j;
                if (cc < col_lim) orow[c + 2 * j] = __ushort_as_bfloat16((unsigned short)(pk[j] & 0xFFFFu));
                if (cc + 1 < col_lim) orow[c + 2 * j + 1] = __ushort_as_bfloat16((unsigned short)(pk[j] >> 16));
              }
            }
          }
        }
      }
      // this warp is done with accumulator `acc`: one arrival on the leader's barrier
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(tempty_leader0 + (uint32_t)(acc * sizeof(uint64_t)));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  if (warp == 0 && lane == 0 && !*abort_flag) {
    // every stage this CTA filled has been released by the leader's MMAs (their
    // completion arrivals target this CTA's barriers, which must outlive them)
    for (int s = 0; s < STAGES; ++s)
      if (fill_par[s] >= 0) drain_wait(smem_u32(&empty[s]), (uint32_t)fill_par[s]);
  }
  __syncthreads();
  if (*abort_flag) {
    // let this CTA's own copies land (they are counted on the leader's
    // barrier, so wait out the drain bound) and the leader's MMAs finish
    if (warp == 0 && lane == 0) {
      const uint64_t t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 2000000ull) {
      }
    }
    if (warp == 1 && lane == 0 && leader) {
      mma_commit_pair(smem_u32(drain));
      drain_wait(smem_u32(drain), 0);
    }
  }
  tc_fence_before();
  __syncthreads();
  // neither CTA frees its tensor memory or exits (its shared memory is read by
  // the pair MMAs and its barriers receive the other CTA's arrivals) before
  // both are done
  cluster_sync_all();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// Pairs that can be resident at once.  A pair needs two SMs of one GPC, and a
// GPC with an odd number of usable SMs leaves one idle, so this can be below
// half the SM count; a persistent grid larger than this would run its last
// pairs' whole share of tiles after the others finish.
template <int MODE, bool FP8>
int resident_pairs(size_t smem, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)device_sm_count());
  cfg.blockDim = dim3(kThreads<FP8>);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, grouped_gemm_pair_kernel<MODE, FP8>, &cfg) != cudaSuccess || n < 1) {
    cudaGetLastError();
    n = device_sm_count() / 2;
  }
  return n;
}

template <int MODE, bool FP8>
cudaError_t launch(const CUtensorMap& ta, const CUtensorMap& ta64, const CUtensorMap& tb, const Params& p,
                   int64_t tiles_bound, cudaStream_t stream) {
  const size_t smem = smem_bytes(p.G);
  cudaError_t e = cudaFuncSetAttribute(grouped_gemm_pair_kernel<MODE, FP8>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int64_t pairs = resident_pairs<MODE, FP8>(smem, stream);
  if (tiles_bound < pairs) pairs = tiles_bound;
  if (pairs < 1) pairs = 1;
  grouped_gemm_pair_kernel<MODE, FP8><<<(unsigned)(2 * pairs), kThreads<FP8>, smem, stream>>>(ta, ta64, tb, p);
  return cudaGetLastError();
}

// Both expert GEMMs on CTA pairs.  FP8: `a` holds E4M3 codes with per-row
// scales a.sa, the weights are E4M3 blobs (codes, then per-row scales), and h
// is re-quantised per token row between the two GEMMs.
template <bool FP8>
cudaError_t run(const GroupedFfnArgs& a, cudaStream_t stream) {
  if (a.rows == 0) return cudaSuccess;
  const int G = a.offsets ? a.G : 1;
  // 256-row m-blocks: at most rows / 256 + one partial block per group
  const int64_t mb_bound = (a.rows + 2 * ROWS - 1) / (2 * ROWS) + (a.offsets ? a.G : 0);
  const uint64_t lim = a.wait_limit_ns ? a.wait_limit_ns : 2000000000ull;
  const int eb = FP8 ? 1 : 2;
  const bool gelu = a.act == kEpiGELU;
  const int64_t w1_rows = (gelu ? 1 : 2) * (int64_t)a.G * a.f;
  const float* s1 = FP8 ? reinterpret_cast<const float*>(static_cast<const uint8_t*>(a.w_gate_up) +
                                                         e4m3_codes_bytes(w1_rows, a.d))
                        : nullptr;
  CUtensorMap mA, mA64, mB1;
  cudaError_t e;
  if (!make_map(&mA, a.a, a.rows, a.d, ROWS, eb) || !make_map(&mA64, a.a, a.rows, a.d, ROWS / 2, eb))
    return cudaErrorInvalidValue;
  if (gelu) {
    // GEMM-1 + GELU: tile = 256 rows x 256 up columns, B halves of 128 rows
    if (!make_map(&mB1, a.w_gate_up, w1_rows, a.d, 128, eb)) return cudaErrorInvalidValue;
    Params p1{a.offsets, G, a.rows, a.d, a.f, (a.f + 255) / 256, (int64_t)a.f, 0, a.h, a.f, a.status, lim, a.sa,
              s1};
    e = launch<MODE_GELU, FP8>(mA, mA64, mB1, p1, mb_bound * p1.nt, stream);
  } else {
    // GEMM-1 + SwiGLU: tile = 256 rows x 128 h columns (128 gate + 128 up B rows)
    if (!make_map(&mB1, a.w_gate_up, w1_rows, a.d, 64, eb)) return cudaErrorInvalidValue;
    Params p1{a.offsets, G, a.rows, a.d, a.f, (a.f + 127) / 128, 2 * (int64_t)a.f, a.f, a.h, a.f, a.status, lim,
              a.sa, s1};
    e = launch<MODE_SWIGLU, FP8>(mA, mA64, mB1, p1, mb_bound * p1.nt, stream);
  }
  if (e != cudaSuccess) return e;
  const void* a2 = a.h;
  const float* sa2 = nullptr;
  if (FP8) {  // h -> E4M3 codes and per-token scales
    e = launch_quantize_e4m3(a.h, a.rows, a.offsets ? a.offsets + a.G : nullptr, a.f, a.hq, a.sh, stream);
    if (e != cudaSuccess) return e;
    a2 = a.hq;
    sa2 = a.sh;
  }
  const float* s2 = FP8 ? reinterpret_cast<const float*>(static_cast<const uint8_t*>(a.w_down) +
                                                         e4m3_codes_bytes((int64_t)a.G * a.d, a.f))
                        : nullptr;
  // GEMM-2: tile = 256 rows x 256 output columns
  CUtensorMap mA2, mA2h, mB2;
  if (!make_map(&mA2, a2, a.rows, a.f, ROWS, eb) || !make_map(&mA2h, a2, a.rows, a.f, ROWS / 2, eb) ||
      !make_map(&mB2, a.w_down, (uint64_t)a.G * a.d, a.f, 128, eb))
    return cudaErrorInvalidValue;
  Params p2{a.offsets, G, a.rows, a.f, a.d, (a.d + 255) / 256, (int64_t)a.d, 0, a.y, a.d, a.status, lim, sa2, s2};
  return launch<MODE_PLAIN, FP8>(mA2, mA2h, mB2, p2, mb_bound * p2.nt, stream);
}

}  // namespace pair
}  // namespace tc

cudaError_t launch_grouped_ffn_pair(const GroupedFfnArgs& a, cudaStream_t stream) {
  return a.fp8 ? tc::pair::run<true>(a, stream) : tc::pair::run<false>(a, stream);
}

}  // namespace moe
