// Grouped expert GEMMs of the decode regime (a few tokens per expert) on the
// sm_100a tensor cores, with the operands swapped: an expert's weight rows are
// the MMA's M operand (128 rows) and its tokens the N operand, so the MMA width
// follows the expert's token count (rounded up to 16, at most 64 per unit)
// instead of a fixed 128-row token tile: an expert with 3 tokens costs an MMA
// of width 16, and the kernel is a stream of the touched experts' weights.
//
// "Mixture of Experts: why a model with 671 billion parameters uses only 37",
// "How data centres handle it" (tokens grouped by expert, all expert
// multiplies in one launch over a stacked weight matrix); "Mixture of experts:
// how MoE works and what it
// costs", "What mixture of experts costs in compute" (decode per-expert
// batches are small and memory bound).  Expert FFN: "Mixture of Experts
// Explained: Routers, Active Parameters and VRAM" (a gated feed-forward block
// with three matrices), read as SwiGLU.
//
//   GEMM-1 (SwiGLU): h^T[f-block, tokens] = [Wg; Wu][64+64 rows] x_perm^T;
//     accumulator rows 0..63 are gate rows, 64..127 the matching up rows; the
//     epilogue pairs them through shared memory and writes h[tokens, f].
//   GEMM-1 (GELU, the two-matrix expert): h^T = GELU(Wu[128 rows] x_perm^T).
//   GEMM-2 (plain):  y^T[d-block, tokens] = Wd[128 rows] h^T.
//
// A unit is (expert, weight-row block j, token chunk of up to 64 tokens; an
// expert's tokens are cut into chunks of equal size).  Inside an expert the
// units run over blocks of 8 chunks, then j, then the chunk, so units running
// together share weight blocks and token chunks through L2.
//
// Schedule (stream-K): the reduction steps of all units, laid end to end, are
// cut into one equal contiguous range per CTA, so every CTA streams the same
// number of weight bytes whatever the routing.  A unit cut between CTAs is
// finished by the last contributor to arrive: each writes its fp32 partial
// tile (at most two per CTA: its first and last unit), adds its step count to
// the unit's counter, and the one that completes the count sums the partials
// in CTA order -- a fixed order, so results are deterministic -- and runs the
// epilogue.  Nothing waits on another CTA.
//
// The same kernel with 256-token units and one whole unit per CTA at a time
// was measured for large batches and ran 1.3-1.7x slower than the
// token-rows-as-M kernel of grouped_gemm_tc.cu, which large batches use.
//
// Persistent, warp-specialised CTA (192 threads): warp 0 TMA producer, warp 1
// TMEM allocator and single-thread tcgen05.mma issuer, warps 2-5 epilogue;
// two accumulators of 64 columns so the epilogue of one unit overlaps the
// main loop of the next.  Every wait is bounded; on expiry the CTA raises an
// abort flag and the device status word, drains its own copies and MMAs,
// frees its tensor memory and returns.
#include <algorithm>
#include <cmath>

#include "kernels.cuh"
#include "pdl.cuh"
#include "tc_primitives.cuh"

namespace moe {
namespace tc {
namespace {

constexpr int S_BK = 64;
constexpr int S_BM = 128;                   // weight rows per MMA (SwiGLU: 64 gate + 64 up)
constexpr int S_THREADS = 192;
constexpr int S_XG = 17;                    // pitch (floats) of a gate/up exchange row: 16 tokens + 1
constexpr int S_HP = 136;                   // pitch (bf16) of a staged output row: 128 columns + 8
// epilogue staging: exchange [2][64][S_XG] fp32, then outputs [32][S_HP] bf16
constexpr int S_STAGE_BYTES = 2 * 64 * S_XG * 4 + 32 * S_HP * 2;
constexpr int S_CB = 8;                     // token chunks per block in the unit order
constexpr int S_A_BYTES = S_BM * S_BK * 2;  // 16 KiB
constexpr int kDevInternal = 7;             // status word: internal size check failed

constexpr int BN = kDecodeTokens;           // most tokens per unit (MMA N <= 64)
constexpr int STAGES = 8;
constexpr int B_BYTES = BN * S_BK * 2;      // 8 KiB
constexpr int TMEM_COLS = 2 * BN;           // two accumulators

struct SwapParams {
  const int32_t* offsets;  // [G+1] token-row offsets, or null: one group of `rows`
  int G;
  int64_t rows;            // token rows of B and of the output
  int K;                   // reduction length
  int n_out;               // output columns (f or d)
  int J;                   // weight-row blocks per group
  int64_t a_group_rows;    // weight rows per group (2f or d)
  int up_off;              // f (SwiGLU)
  __nv_bfloat16* out;      // [rows, n_out]
  int64_t ldo;
  float* partial;          // [2 * gridDim.x][128][BN] fp32 partial tiles
  int* counters;           // one per unit; zero on entry, zero on exit
  int64_t counter_cap;     // units the counters (and the schedule) allow
  int* status;
  uint64_t wait_limit_ns;
  const float* sx;         // FP8: per-token scales of the B operand
  const float* sw;         // FP8: per-row scales of the weight tensor
};

size_t swap_smem_bytes(int G) {
  return 1024 + (size_t)STAGES * (S_A_BYTES + B_BYTES) + S_STAGE_BYTES + 256 + 2 * sizeof(int) * (size_t)(G + 1);
}

// Named barrier of the four epilogue warps (barrier 1, 128 threads).
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// Same barrier, returning whether any of the 128 threads passed true: the
// epilogue warps use it to take their loop-exit decision together.
__device__ __forceinline__ bool epi_bar_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pin, pout;\n\t"
      "setp.ne.u32 pin, %1, 0;\n\t"
      "bar.red.or.pred pout, 1, 128, pin;\n\t"
      "selp.u32 %0, 1, 0, pout;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

struct Unit {
  int g, j, chunk;
  int row0;     // first row of the chunk inside its group
  int n_valid;  // tokens of this chunk (1..BN)
  int nmma;     // MMA N: n_valid rounded up to 16
};

// unit -> (group, weight block, token chunk)
__device__ __forceinline__ Unit decode_unit(int64_t u, int J, const int* cum, const int* off, int G, int bn) {
  int lo = 0, hi = G;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if ((int64_t)cum[mid] * J <= u) lo = mid;
    else hi = mid;
  }
  Unit r;
  r.g = lo;
  const int nch = cum[lo + 1] - cum[lo];
  const int64_t local = u - (int64_t)cum[lo] * J;
  const int cb = (int)(local / ((int64_t)S_CB * J));
  const int64_t rest = local - (int64_t)cb * S_CB * J;
  const int nb = min(S_CB, nch - cb * S_CB);  // chunks in this block
  r.j = (int)(rest / nb);
  r.chunk = cb * S_CB + (int)(rest % nb);
  // the group's rows split into nch chunks of equal size (a multiple of 16,
  // at most bn), the last one shorter: no chunk is a sliver next to a full one
  const int n = off[lo + 1] - off[lo];
  const int cs = ((n + nch - 1) / nch + 15) & ~15;
  r.row0 = r.chunk * cs;
  r.n_valid = min(cs, n - r.row0);
  r.nmma = (r.n_valid + 15) & ~15;
  return r;
}

// First reduction step of CTA c's range when `total` steps are cut into `parts`.
__device__ __forceinline__ int64_t range_start(int64_t c, int64_t total, int64_t parts) { return c * total / parts; }
// The CTA whose range holds step i.
__device__ __forceinline__ int64_t range_owner(int64_t i, int64_t total, int64_t parts) {
  return ((i + 1) * parts - 1) / total;
}

// Calls f(unit, kb0, kb1, first) for this CTA's segments in order, until f returns false.
template <typename F>
__device__ __forceinline__ void for_each_segment(int64_t n_units, int kb_count, F&& f) {
  const int64_t total = n_units * kb_count, parts = gridDim.x;
  const int64_t begin = range_start(blockIdx.x, total, parts), end = range_start(blockIdx.x + 1, total, parts);
  for (int64_t pos = begin; pos < end;) {
    const int64_t u = pos / kb_count;
    const int kb0 = (int)(pos - u * kb_count);
    const int kb1 = (end - pos < (int64_t)(kb_count - kb0)) ? kb0 + (int)(end - pos) : kb_count;
    const bool first = pos == begin;
    pos += kb1 - kb0;
    if (!f(u, kb0, kb1, first)) return;
  }
}

// FP8: weights and tokens are E4M3 codes; a stage's 128-byte K slice holds 128
// of them (kind::f8f6f4) and the epilogue applies the weight-row and token scales.
template <int EPI, bool FP8>
__global__ void __launch_bounds__(S_THREADS, 1)
    grouped_gemm_swap_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX64,
                             const __grid_constant__ CUtensorMap tmX16, const SwapParams p) {
  constexpr bool SWIGLU = EPI == kEpiSwiGLU;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * S_A_BYTES;
  float* xg = reinterpret_cast<float*>(sB + STAGES * B_BYTES);  // [64][S_XG] gate values, tokens 16..31
  float* xu = xg + 64 * S_XG;                                    // [64][S_XG] up values, tokens 0..15
  __nv_bfloat16* hs = reinterpret_cast<__nv_bfloat16*>(xu + 64 * S_XG);  // [32][S_HP] staged outputs
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + STAGES * B_BYTES + S_STAGE_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = bars + 2 * STAGES + 2;
  uint64_t* drain = bars + 2 * STAGES + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* reducer_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);
  int* fill_par = reinterpret_cast<int*>(tmem_slot + 3);  // [STAGES]
  int* s_off = fill_par + STAGES;                          // [G+1]
  int* s_cum = s_off + (p.G + 1);                          // [G+1] cumulative token chunks

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int G = p.G;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
      fill_par[s] = -1;
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&tfull[a]), 1);
      mbar_init(smem_u32(&tempty[a]), 128);
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX64);
    tma_prefetch_desc(&tmX16);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  if (p.offsets) {
    for (int g = threadIdx.x; g <= G; g += S_THREADS) s_off[g] = p.offsets[g];
  } else if (threadIdx.x == 0) {
    s_off[0] = 0;
    s_off[1] = (int)p.rows;
  }
  __syncthreads();
  if (warp == 0) {  // cumulative BN-token chunks per group
    int carry = 0;
    if (lane == 0) s_cum[0] = 0;
    for (int base = 0; base < G; base += 32) {
      const int g = base + lane;
      int v = 0;
      if (g < G) v = max(0, (s_off[g + 1] - s_off[g] + BN - 1) / BN);
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += u;
      }
      if (g < G) s_cum[g + 1] = carry + v;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Programmatic launch (pdl.cuh): wait here, after the set-up, for the
  // predecessor (GEMM-1 for GEMM-2, the gather for GEMM-1 of a chained layer
  // step), then let the successor be scheduled: its CTAs take the SMs this
  // grid frees.  The set-up above reads only the offsets of the dispatch,
  // which finished before the predecessor passed its own wait.
  grid_dependency_wait();
  if (threadIdx.x == 0) grid_launch_dependents();

  const uint32_t tmem_base = *tmem_slot;
  constexpr int KB = FP8 ? 2 * S_BK : S_BK;  // elements per 128-byte K slice
  const int kb_count = (p.K + KB - 1) / KB;
  int64_t n_units = (int64_t)s_cum[G] * p.J;
  if (n_units > p.counter_cap) {  // the host sized the schedule for fewer units: do nothing
    if (threadIdx.x == 0) set_status(p.status, kDevInternal);
    n_units = 0;
  }

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      for_each_segment(n_units, kb_count, [&](int64_t u, int kb0, int kb1, bool) {
        const Unit un = decode_unit(u, p.J, s_cum, s_off, G, BN);
        const int w_row = (int)((int64_t)un.g * p.a_group_rows + (int64_t)un.j * (SWIGLU ? S_BM / 2 : S_BM));
        const int x_row = s_off[un.g] + un.row0;
        const uint32_t tx = S_A_BYTES + (uint32_t)un.nmma * S_BK * 2;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_bounded(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, p.wait_limit_ns, p.status))
            return false;
          const uint32_t fb = smem_u32(&full[stage]);
          mbar_expect_tx(fb, tx);
          fill_par[stage] = (int)phase;
          const uint32_t a_dst = smem_u32(sA + stage * S_A_BYTES);
          if (SWIGLU) {  // 64 gate rows, then the 64 matching up rows
            tma_load_2d(a_dst, &tmW, fb, kb * KB, w_row);
            tma_load_2d(a_dst + S_A_BYTES / 2, &tmW, fb, kb * KB, w_row + p.up_off);
          } else {
            tma_load_2d(a_dst, &tmW, fb, kb * KB, w_row);
          }
          const uint32_t b_dst = smem_u32(sB + stage * B_BYTES);
          int b = 0;
          for (; b + 64 <= un.nmma; b += 64) tma_load_2d(b_dst + b * 128, &tmX64, fb, kb * KB, x_row + b);
          for (; b < un.nmma; b += 16) tma_load_2d(b_dst + b * 128, &tmX16, fb, kb * KB, x_row + b);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        return true;
      });
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for_each_segment(n_units, kb_count, [&](int64_t u, int kb0, int kb1, bool) {
        const Unit un = decode_unit(u, p.J, s_cum, s_off, G, BN);
        const uint32_t idesc = idesc_f32acc<FP8>(S_BM, un.nmma);
        if (!mbar_wait_bounded(smem_u32(&tempty[acc]), acc_phase ^ 1u, abort_flag, p.wait_limit_ns, p.status))
          return false;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_bounded(smem_u32(&full[stage]), phase, abort_flag, p.wait_limit_ns, p.status)) return false;
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * S_A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * B_BYTES);
          mma_kslice<FP8>(d_tmem, a0, b0, idesc, kb == kb0);
          mma_commit(smem_u32(&empty[stage]));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        mma_commit(smem_u32(&tfull[acc]));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
        return true;
      });
    }
  } else {
    // -------------------------------------------------- epilogue (warps 2..5)
    const int q = warp & 3;
    const int r = q * 32 + lane;  // accumulator row = weight row inside the block
    const bool leader = (warp == 2 && lane == 0);
    int acc = 0;
    uint32_t acc_phase = 0;

    // Final epilogue of 32 token columns [32 cc, 32 cc + 32) of a unit.  The
    // outputs are staged token-major in shared memory and leave in coalesced
    // 16-byte stores.  SwiGLU: a gate row and its up row sit in different
    // warps, so gate rows finish tokens 0..15 and up rows tokens 16..31, each
    // taking the other half's partner values through shared memory.
    auto finish = [&](const Unit& un, float (&v)[32], int cc) {
      const int nv = min(32, un.n_valid - 32 * cc);
      const int64_t row0 = (int64_t)s_off[un.g] + un.row0 + 32 * cc;
      if (FP8) {  // accumulator * weight-row scale * token scale
        const int feat = SWIGLU ? un.j * 64 + (r & 63) : un.j * S_BM + r;
        const int64_t wrow = (int64_t)un.g * p.a_group_rows + (SWIGLU && r >= 64 ? p.up_off : 0) + feat;
        const float sw = feat < p.n_out ? p.sw[wrow] : 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= i < nv ? sw * p.sx[row0 + i] : 0.f;
      }
      int ncols, col0;
      if (SWIGLU) {
        const int f = r & 63;
        if (r < 64) {
#pragma unroll
          for (int i = 0; i < 16; ++i) xg[f * S_XG + i] = v[16 + i];
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) xu[f * S_XG + i] = v[i];
        }
        epi_bar();
        if (r < 64) {
#pragma unroll
          for (int i = 0; i < 16; ++i) hs[i * S_HP + f] = __float2bfloat16_rn(silu_f(v[i]) * xu[f * S_XG + i]);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            hs[(16 + i) * S_HP + f] = __float2bfloat16_rn(silu_f(xg[f * S_XG + i]) * v[16 + i]);
        }
        ncols = 64;
        col0 = un.j * 64;
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) hs[i * S_HP + r] = __float2bfloat16_rn(EPI == kEpiGELU ? gelu_f(v[i]) : v[i]);
        ncols = S_BM;
        col0 = un.j * S_BM;
      }
      epi_bar();
      const int segs = ncols / 8;  // 16-byte segments per token row
      for (int c = r; c < 32 * segs; c += 128) {
        const int tok = c / segs, sg = c % segs;
        const int col = col0 + sg * 8;
        const int64_t row = row0 + tok;
        if (tok < nv && row < p.rows) {
          const __nv_bfloat16* src = hs + tok * S_HP + sg * 8;
          __nv_bfloat16* dst = p.out + row * p.ldo + col;
          if (col + 8 <= p.n_out) {
            *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
          } else {
            for (int e = 0; e < 8; ++e)
              if (col + e < p.n_out) dst[e] = src[e];
          }
        }
      }
      epi_bar();  // the staging buffers are free again
    };

    for_each_segment(n_units, kb_count, [&](int64_t u, int kb0, int kb1, bool first) {
      const Unit un = decode_unit(u, p.J, s_cum, s_off, G, BN);
      const bool got = mbar_wait_bounded(smem_u32(&tfull[acc]), acc_phase, abort_flag, p.wait_limit_ns, p.status);
      if (epi_bar_any(!got || *abort_flag)) return false;  // every epilogue warp leaves together
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      const int nc32 = (un.nmma + 31) / 32;
      float v[32];
      if (kb0 == 0 && kb1 == kb_count) {  // the whole unit is here
        for (int cc = 0; cc < nc32; ++cc) {
          uint32_t raw[32];
          tmem_ld32(tb + 32 * cc, raw);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(raw[i]);
          finish(un, v, cc);
        }
        tc_fence_before();
        mbar_arrive(smem_u32(&tempty[acc]));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
        return true;
      }
      // part of a unit: publish this CTA's partial; the contributor that
      // completes the unit's step count sums them all
      const int64_t slot = 2 * (int64_t)blockIdx.x + (first ? 0 : 1);
      float* prow = p.partial + (slot * S_BM + r) * BN;
      for (int cc = 0; cc < nc32; ++cc) {
        uint32_t raw[32];
        tmem_ld32(tb + 32 * cc, raw);
        tmem_ld_wait();
        float4* dst = reinterpret_cast<float4*>(prow + 32 * cc);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (32 * cc + 4 * i < un.nmma)
            dst[i] = make_float4(__uint_as_float(raw[4 * i]), __uint_as_float(raw[4 * i + 1]),
                                 __uint_as_float(raw[4 * i + 2]), __uint_as_float(raw[4 * i + 3]));
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&tempty[acc]));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
      __threadfence();
      epi_bar();
      if (leader) *reducer_flag = (atomicAdd(&p.counters[u], kb1 - kb0) + (kb1 - kb0) == kb_count);
      epi_bar();
      // (the leader rewrites the flag only after the next segment's
      // epi_bar_any, which every reader has passed by then)
      if (!*reducer_flag) return true;
      __threadfence();
      const int64_t total = n_units * kb_count, parts = gridDim.x;
      const int64_t c0 = range_owner(u * kb_count, total, parts);
      const int64_t c1 = range_owner(u * kb_count + kb_count - 1, total, parts);
      for (int cc = 0; cc < nc32; ++cc) {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
        for (int64_t c = c0; c <= c1; ++c) {  // contributors in CTA order = K order
          const int64_t cs = range_start(c, total, parts);
          if (range_start(c + 1, total, parts) == cs) continue;  // empty range: no partial
          const int64_t s2 = 2 * c + (cs / kb_count == u ? 0 : 1);
          const float4* src = reinterpret_cast<const float4*>(p.partial + (s2 * S_BM + r) * BN + 32 * cc);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            if (32 * cc + 4 * i < un.nmma) {
              const float4 w4 = __ldcg(src + i);
              v[4 * i] += w4.x;
              v[4 * i + 1] += w4.y;
              v[4 * i + 2] += w4.z;
              v[4 * i + 3] += w4.w;
            }
          }
        }
        finish(un, v, cc);
      }
      if (leader) p.counters[u] = 0;  // ready for the next launch
      return true;
    });
  }

  if (warp == 0 && lane == 0 && !*abort_flag) {
    // every stage filled has been released by its MMAs (their completion
    // arrivals target this CTA's barriers, which must outlive them)
    for (int s = 0; s < STAGES; ++s)
      if (fill_par[s] >= 0) drain_wait(smem_u32(&empty[s]), (uint32_t)fill_par[s]);
  }
  __syncthreads();
  if (*abort_flag) {
    if (warp == 0 && lane == 0) {
      for (int s = 0; s < STAGES; ++s)
        if (fill_par[s] >= 0) drain_wait(smem_u32(&full[s]), (uint32_t)fill_par[s]);
    }
    if (warp == 1 && lane == 0) {
      mma_commit(smem_u32(drain));
      drain_wait(smem_u32(drain), 0);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// chained: the launch is programmatic (pdl.cuh) and finds its unit counters at
// zero: GEMM-2 after GEMM-1 (directly, or behind the 8-bit re-quantisation
// of h), whose units' last contributors reset every counter they used, or
// GEMM-1 of a layer step that cleared the counters ahead (moe_forward).
// Otherwise the counters are cleared first (a launch that timed out may leave
// some set).
template <int EPI, bool FP8>
cudaError_t launch_swap(const CUtensorMap& tw, const CUtensorMap& tx64, const CUtensorMap& tx16,
                        const SwapParams& p, int grid, bool chained, cudaStream_t stream) {
  auto kernel = grouped_gemm_swap_kernel<EPI, FP8>;
  const size_t smem = swap_smem_bytes(p.G);
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (!chained) {
    e = cudaMemsetAsync(p.counters, 0, sizeof(int) * (size_t)p.counter_cap, stream);
    if (e != cudaSuccess) return e;
  }
  return launch_maybe_chained(kernel, dim3((unsigned)grid), dim3(S_THREADS), smem, stream, chained, tw, tx64, tx16,
                              p);
}

// Units of one GEMM, bounded from the row count (the chunking is per group).
int64_t unit_bound(int64_t rows, int G, int bn, int J) { return ((rows + bn - 1) / bn + G) * (int64_t)J; }

// Both GEMMs of the expert FFN with one schedule.  FP8: `a` holds E4M3 codes
// with per-row scales a.sa, the weights are E4M3 blobs (codes, then per-row
// scales), and h is re-quantised per token row between the two GEMMs.
template <bool FP8>
cudaError_t run_swap(const GroupedFfnArgs& a, cudaStream_t stream) {
  const int G = a.offsets ? a.G : 1;
  const uint64_t lim = a.wait_limit_ns ? a.wait_limit_ns : 2000000000ull;
  const int sms = device_sm_count();
  const int eb = FP8 ? 1 : 2;
  const bool gelu = a.act == kEpiGELU;
  const int J1 = gelu ? (a.f + 127) / 128 : (a.f + 63) / 64, J2 = (a.d + 127) / 128;
  const int64_t cap1 = unit_bound(a.rows, G, BN, J1), cap2 = unit_bound(a.rows, G, BN, J2);
  if (cap1 > a.counter_cap || cap2 > a.counter_cap) return cudaErrorInvalidValue;
  const int grid = std::max(1, std::min(sms, kDecodeMaxCtas));
  // GEMM-1: SwiGLU weight blocks of 64 gate + 64 up rows, or GELU blocks of
  // 128 up rows; tokens of x_perm
  const int64_t w1_rows = (gelu ? 1 : 2) * (int64_t)a.f;
  const float* s1 = FP8 ? reinterpret_cast<const float*>(static_cast<const uint8_t*>(a.w_gate_up) +
                                                         e4m3_codes_bytes((int64_t)a.G * w1_rows, a.d))
                        : nullptr;
  CUtensorMap w1, x1a, x1b;
  if (!make_map(&w1, a.w_gate_up, (uint64_t)a.G * w1_rows, a.d, gelu ? S_BM : 64, eb) ||
      !make_map(&x1a, a.a, a.rows, a.d, 64, eb) || !make_map(&x1b, a.a, a.rows, a.d, 16, eb))
    return cudaErrorInvalidValue;
  SwapParams p1{a.offsets, G, a.rows, a.d, a.f, J1, w1_rows, a.f, static_cast<__nv_bfloat16*>(a.h), a.f,
                a.partial, a.counters, a.counter_cap, a.status, lim, a.sa, s1};
  cudaError_t e = gelu ? launch_swap<kEpiGELU, FP8>(w1, x1a, x1b, p1, grid, a.chained, stream)
                       : launch_swap<kEpiSwiGLU, FP8>(w1, x1a, x1b, p1, grid, a.chained, stream);
  if (e != cudaSuccess) return e;
  const void* b2 = a.h;
  const float* sx2 = nullptr;
  if (FP8) {  // h -> E4M3 codes and per-token scales
    e = launch_quantize_e4m3(a.h, a.rows, a.offsets ? a.offsets + a.G : nullptr, a.f, a.hq, a.sh, stream);
    if (e != cudaSuccess) return e;
    b2 = a.hq;
    sx2 = a.sh;
  }
  const float* s2 = FP8 ? reinterpret_cast<const float*>(static_cast<const uint8_t*>(a.w_down) +
                                                         e4m3_codes_bytes((int64_t)a.G * a.d, a.f))
                        : nullptr;
  // GEMM-2: weight blocks of 128 down rows, tokens of h
  CUtensorMap w2, x2a, x2b;
  if (!make_map(&w2, a.w_down, (uint64_t)a.G * a.d, a.f, S_BM, eb) || !make_map(&x2a, b2, a.rows, a.f, 64, eb) ||
      !make_map(&x2b, b2, a.rows, a.f, 16, eb))
    return cudaErrorInvalidValue;
  SwapParams p2{a.offsets, G, a.rows, a.f, a.d, J2, (int64_t)a.d, 0, static_cast<__nv_bfloat16*>(a.y), a.d,
                a.partial, a.counters, a.counter_cap, a.status, lim, sx2, s2};
  return launch_swap<kEpiNone, FP8>(w2, x2a, x2b, p2, grid, true, stream);
}

}  // namespace
}  // namespace tc

bool use_decode_ffn(int64_t rows, int G, bool grouped) {
  double touched = grouped ? G * (1.0 - std::pow(1.0 - 1.0 / G, (double)rows)) : 1.0;
  if (touched < 1.0) touched = 1.0;
  return (double)rows / touched <= kDecodeTokens;
}

// Partial tiles of the decode schedule: two [128][kDecodeTokens] fp32 tiles per CTA.
int64_t decode_partial_slots() { return 2 * (int64_t)kDecodeMaxCtas; }

// Units (expert, weight block, token chunk) of either GEMM of the decode schedule.
int64_t decode_counter_cap(int64_t rows, int G, int d, int f) {
  return tc::unit_bound(rows, G, kDecodeTokens, std::max((f + 63) / 64, (d + 127) / 128));
}

cudaError_t launch_grouped_ffn_bf16_decode(const GroupedFfnArgs& a, cudaStream_t stream) {
  if (a.rows == 0) return cudaSuccess;
  if (a.partial == nullptr || a.counters == nullptr || a.partial_slots < decode_partial_slots())
    return cudaErrorInvalidValue;
  return a.fp8 ? tc::run_swap<true>(a, stream) : tc::run_swap<false>(a, stream);
}


}  // namespace moe
