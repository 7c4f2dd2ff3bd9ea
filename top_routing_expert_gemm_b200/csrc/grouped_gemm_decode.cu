// Grouped expert GEMMs for the decode regime (a few tokens per expert), on
// the sm_100a tensor cores with the operands swapped: the expert's weight rows
// are the MMA's M operand (128 rows) and its handful of tokens the N operand
// (64 columns), so every MMA row is a real weight row and the kernel streams
// each touched expert's weights exactly once.
//
// "Mixture of experts: how MoE works and what it costs", "What mixture of
// experts costs in compute" (decode per-expert batches are small and memory
// bound) and "How batching changes the mixture of experts math" (at small
// batch a step reads only the touched experts); "Mixture of Experts: why a
// model with 671 billion parameters uses only 37", "Prefill vs. decode".
//
//   GEMM-1 (SwiGLU): h^T[f-block, tokens] = [Wg; Wu][64+64 rows] x_perm^T,
//     the even half of the accumulator rows are gate rows, the odd half the
//     matching up rows; the epilogue pairs them through shared memory and
//     writes h[tokens, f].
//   GEMM-2 (plain):  y^T[d-block, tokens] = Wd[128 rows] h^T.
//
// Work unit = (expert, 64-token chunk, weight-row block, K split).  With too
// few output tiles to fill the GPU the reduction is split S ways: every split
// writes its fp32 partial tile to scratch, and the last split to finish (an
// atomic count per output tile) sums the partials in split order -- a fixed
// order, so results are deterministic -- before the epilogue.
//
// Warp roles, bounded waits and the abort/drain protocol are those of the
// large-batch kernel (grouped_gemm_tc.cu).
#include <cmath>

#include "kernels.cuh"
#include "tc_primitives.cuh"

namespace moe {
namespace tc {
namespace {

constexpr int D_STAGES = 8;
constexpr int D_BK = 64;
constexpr int D_BM = 128;                   // weight rows per MMA (SwiGLU: 64 gate + 64 up)
constexpr int D_BN = 64;                    // tokens per unit (MMA N)
constexpr int D_A_BYTES = D_BM * D_BK * 2;  // 16 KiB
constexpr int D_B_BYTES = D_BN * D_BK * 2;  // 8 KiB
constexpr int D_TMEM_COLS = 128;            // two 64-column accumulators
constexpr int D_THREADS = 192;
constexpr int D_XPITCH = D_BN + 1;          // padded row of the gate/up exchange buffer
constexpr int D_MAX_SPLITS = 16;

struct DecodeParams {
  const int32_t* offsets;  // [G+1] token-row offsets, or null: one group of `rows`
  int G;
  int64_t rows;            // token rows of B and of the output
  int K;                   // reduction length
  int n_out;               // output columns (f or d)
  int J;                   // weight-row blocks per group
  int S;                   // requested K splits
  int64_t a_group_rows;    // weight rows per group (2f or d)
  int up_off;              // f (SwiGLU)
  __nv_bfloat16* out;      // [rows, n_out]
  int64_t ldo;
  float* partial;          // split partials: slots of [128][64] fp32
  int64_t partial_slots;
  int* counters;           // one per output unit; zero on entry, zero on exit
  int64_t counter_cap;
  int* status;
  uint64_t wait_limit_ns;
};

size_t decode_smem_bytes(int G) {
  return 1024 + (size_t)D_STAGES * (D_A_BYTES + D_B_BYTES) + sizeof(float) * 64 * D_XPITCH + 256 +
         2 * sizeof(int) * (size_t)(G + 1);
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

// output unit -> (group, token chunk, weight-row block)
__device__ __forceinline__ void decode_unit(int64_t u, int J, const int* cum, int G, int& g, int& chunk, int& j) {
  int lo = 0, hi = G;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if ((int64_t)cum[mid] * J <= u) lo = mid;
    else hi = mid;
  }
  g = lo;
  const int64_t local = u - (int64_t)cum[lo] * J;
  chunk = (int)(local / J);
  j = (int)(local % J);
}

template <bool SWIGLU>
__global__ void __launch_bounds__(D_THREADS, 1)
    grouped_gemm_decode_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                               const DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + D_STAGES * D_A_BYTES;
  float* xbuf = reinterpret_cast<float*>(sB + D_STAGES * D_B_BYTES);  // [64][D_XPITCH] up values
  uint64_t* bars = reinterpret_cast<uint64_t*>(xbuf + 64 * D_XPITCH);
  uint64_t* full = bars;
  uint64_t* empty = bars + D_STAGES;
  uint64_t* tfull = bars + 2 * D_STAGES;
  uint64_t* tempty = bars + 2 * D_STAGES + 2;
  uint64_t* drain = bars + 2 * D_STAGES + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * D_STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* reducer_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);
  int* fill_par = reinterpret_cast<int*>(tmem_slot + 3);  // [D_STAGES]
  int* s_off = fill_par + D_STAGES;                        // [G+1]
  int* s_cum = s_off + (p.G + 1);                          // [G+1] cumulative token chunks

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int G = p.G;

  if (threadIdx.x == 0) {
    for (int s = 0; s < D_STAGES; ++s) {
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
    tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), D_TMEM_COLS);
    tmem_relinquish();
  }
  if (p.offsets) {
    for (int g = threadIdx.x; g <= G; g += D_THREADS) s_off[g] = p.offsets[g];
  } else if (threadIdx.x == 0) {
    s_off[0] = 0;
    s_off[1] = (int)p.rows;
  }
  __syncthreads();
  if (warp == 0) {  // cumulative 64-token chunks per group
    int carry = 0;
    if (lane == 0) s_cum[0] = 0;
    for (int base = 0; base < G; base += 32) {
      const int g = base + lane;
      int v = 0;
      if (g < G) v = max(0, (s_off[g + 1] - s_off[g] + D_BN - 1) / D_BN);
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

  const uint32_t tmem_base = *tmem_slot;
  const int64_t n_out_units = (int64_t)s_cum[G] * p.J;
  const int kb_count = (p.K + D_BK - 1) / D_BK;
  // splits actually used: bounded by the scratch, the counters and the K blocks
  int S = p.S < 1 ? 1 : p.S;
  if (S > kb_count) S = kb_count;
  if (S > 1 && (n_out_units * S > p.partial_slots || n_out_units > p.counter_cap)) {
    S = (int)(p.partial_slots / (n_out_units > 0 ? n_out_units : 1));
    if (n_out_units > p.counter_cap || S < 2) S = 1;
  }
  const int64_t total = n_out_units * S;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      for (int64_t t = blockIdx.x; t < total; t += gridDim.x) {
        const int64_t ou = t / S;
        const int s = (int)(t % S);
        int g, chunk, j;
        decode_unit(ou, p.J, s_cum, G, g, chunk, j);
        const int w_row = (int)((int64_t)g * p.a_group_rows + (int64_t)j * (SWIGLU ? D_BM / 2 : D_BM));
        const int x_row = s_off[g] + chunk * D_BN;
        const int kb0 = (int)((int64_t)s * kb_count / S), kb1 = (int)((int64_t)(s + 1) * kb_count / S);
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_bounded(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, p.wait_limit_ns, p.status)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&full[stage]);
          mbar_expect_tx(fb, D_A_BYTES + D_B_BYTES);
          fill_par[stage] = (int)phase;
          if (SWIGLU) {  // 64 gate rows, then the 64 matching up rows
            tma_load_2d(smem_u32(sA + stage * D_A_BYTES), &tmW, fb, kb * D_BK, w_row);
            tma_load_2d(smem_u32(sA + stage * D_A_BYTES + D_A_BYTES / 2), &tmW, fb, kb * D_BK, w_row + p.up_off);
          } else {
            tma_load_2d(smem_u32(sA + stage * D_A_BYTES), &tmW, fb, kb * D_BK, w_row);
          }
          tma_load_2d(smem_u32(sB + stage * D_B_BYTES), &tmX, fb, kb * D_BK, x_row);
          if (++stage == D_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      const uint32_t idesc = idesc_bf16_f32(D_BM, D_BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const int s = (int)(t % S);
        const int kb0 = (int)((int64_t)s * kb_count / S), kb1 = (int)((int64_t)(s + 1) * kb_count / S);
        if (!mbar_wait_bounded(smem_u32(&tempty[acc]), acc_phase ^ 1u, abort_flag, p.wait_limit_ns, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * D_BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_bounded(smem_u32(&full[stage]), phase, abort_flag, p.wait_limit_ns, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * D_A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * D_B_BYTES);
#pragma unroll
          for (int kk = 0; kk < D_BK / 16; ++kk)
            mma_bf16(d_tmem, smem_desc_sw128(a0 + kk * 32), smem_desc_sw128(b0 + kk * 32), idesc,
                     (kb != kb0 || kk != 0) ? 1u : 0u);
          mma_commit(smem_u32(&empty[stage]));
          if (++stage == D_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(smem_u32(&tfull[acc]));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
    }
  } else {
    // -------------------------------------------------- epilogue (warps 2..5)
    const int q = warp & 3;
    const int r = q * 32 + lane;  // accumulator row = weight row inside the block
    const bool first = (warp == 2 && lane == 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int64_t t = blockIdx.x; t < total; t += gridDim.x) {
      const int64_t ou = t / S;
      const int s = (int)(t % S);
      int g, chunk, j;
      decode_unit(ou, p.J, s_cum, G, g, chunk, j);
      const bool got = mbar_wait_bounded(smem_u32(&tfull[acc]), acc_phase, abort_flag, p.wait_limit_ns, p.status);
      if (epi_bar_any(!got || *abort_flag)) break;  // every epilogue warp leaves together
      tc_fence_after();
      float v[D_BN];
      {
        uint32_t raw[32];
        const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * D_BN);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          tmem_ld32(tb + h * 32, raw);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 32; ++c) v[h * 32 + c] = __uint_as_float(raw[c]);
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&tempty[acc]));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;

      if (S > 1) {
        // publish this split's partial tile; the last split to arrive reduces
        float4* dst = reinterpret_cast<float4*>(p.partial + ((ou * S + s) * D_BM + r) * D_BN);
#pragma unroll
        for (int c = 0; c < D_BN / 4; ++c) dst[c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
        __threadfence();
        epi_bar();
        if (first) *reducer_flag = (atomicAdd(&p.counters[ou], 1) == S - 1);
        epi_bar();
        if (!*reducer_flag) continue;
        __threadfence();
#pragma unroll
        for (int c = 0; c < D_BN; ++c) v[c] = 0.f;
        for (int s2 = 0; s2 < S; ++s2) {  // fixed order: deterministic sums
          const float4* src = reinterpret_cast<const float4*>(p.partial + ((ou * S + s2) * D_BM + r) * D_BN);
#pragma unroll
          for (int c = 0; c < D_BN / 4; ++c) {
            const float4 w4 = __ldcg(src + c);
            v[4 * c] += w4.x;
            v[4 * c + 1] += w4.y;
            v[4 * c + 2] += w4.z;
            v[4 * c + 3] += w4.w;
          }
        }
        if (first) p.counters[ou] = 0;  // leave the counter ready for the next call
      }

      const int n_g = s_off[g + 1] - s_off[g];
      const int n_valid = min(D_BN, n_g - chunk * D_BN);
      const int64_t row0 = (int64_t)s_off[g] + (int64_t)chunk * D_BN;
      if (SWIGLU) {
        if (r >= 64) {
#pragma unroll
          for (int c = 0; c < D_BN; ++c) xbuf[(r - 64) * D_XPITCH + c] = v[c];
        }
        epi_bar();
        const int col = j * 64 + r;
        if (r < 64 && col < p.n_out) {
#pragma unroll
          for (int c = 0; c < D_BN; ++c) {
            const int64_t row = row0 + c;
            if (c < n_valid && row >= 0 && row < p.rows)
              p.out[row * p.ldo + col] = __float2bfloat16_rn(silu_f(v[c]) * xbuf[r * D_XPITCH + c]);
          }
        }
        epi_bar();  // the exchange buffer is free again
      } else {
        const int col = j * D_BM + r;
        if (col < p.n_out) {
#pragma unroll
          for (int c = 0; c < D_BN; ++c) {
            const int64_t row = row0 + c;
            if (c < n_valid && row >= 0 && row < p.rows) p.out[row * p.ldo + col] = __float2bfloat16_rn(v[c]);
          }
        }
      }
    }
  }

  if (warp == 0 && lane == 0 && !*abort_flag) {
    for (int s = 0; s < D_STAGES; ++s)
      if (fill_par[s] >= 0) drain_wait(smem_u32(&empty[s]), (uint32_t)fill_par[s]);
  }
  __syncthreads();
  if (*abort_flag) {
    if (warp == 0 && lane == 0) {
      for (int s = 0; s < D_STAGES; ++s)
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
    tmem_dealloc(tmem_base, D_TMEM_COLS);
  }
}

// Expected output tiles of one GEMM under uniform routing.
int64_t expected_units(int64_t rows, int G, bool grouped, int J) {
  double touched = grouped ? G * (1.0 - std::pow(1.0 - 1.0 / G, (double)rows)) : 1.0;
  if (touched < 1.0) touched = 1.0;
  const double per = (double)rows / touched;
  return (int64_t)std::ceil(touched) * (int64_t)std::ceil(per / D_BN) * J;
}

// K splits minimising (waves of units) x (weight bytes per unit + partial bytes per unit).
int choose_splits(int64_t units, int kb_count, int ctas) {
  int best = 1;
  double best_cost = 1e300;
  for (int s = 1; s <= D_MAX_SPLITS && s <= kb_count / 2; ++s) {
    const int64_t waves = (units * s + ctas - 1) / ctas;
    const double bytes = (double)D_A_BYTES * kb_count / s + (s > 1 ? 2.0 * D_BM * D_BN * 4 : 0.0);
    const double cost = (double)waves * bytes;
    if (cost < best_cost * 0.98) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

template <bool SWIGLU>
cudaError_t launch_decode(const CUtensorMap& tw, const CUtensorMap& tx, const DecodeParams& p, cudaStream_t stream) {
  const size_t smem = decode_smem_bytes(p.G);
  cudaError_t e = cudaFuncSetAttribute(grouped_gemm_decode_kernel<SWIGLU>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t units = (p.rows + D_BN - 1) / D_BN + (p.offsets ? p.G : 0);  // bound on token chunks
  int64_t grid = device_sm_count();
  if (units * p.J * p.S < grid) grid = units * p.J * p.S;
  if (grid < 1) grid = 1;
  grouped_gemm_decode_kernel<SWIGLU><<<(unsigned)grid, D_THREADS, smem, stream>>>(tw, tx, p);
  return cudaGetLastError();
}

}  // namespace
}  // namespace tc

bool use_decode_ffn(int64_t rows, int G, bool grouped) {
  double touched = grouped ? G * (1.0 - std::pow(1.0 - 1.0 / G, (double)rows)) : 1.0;
  if (touched < 1.0) touched = 1.0;
  return (double)rows / touched <= tc::D_BN;
}

// Split-K scratch: enough [128][64] fp32 partial tiles to split every output
// tile D_MAX_SPLITS ways, capped at 1536 tiles (48 MiB).  The kernel lowers its
// split count when a batch routes to more experts than the scratch covers.
int64_t decode_partial_slots(int64_t rows, int G, bool grouped, int d, int f) {
  (void)grouped;
  const int64_t chunks = (rows + tc::D_BN - 1) / tc::D_BN + G;
  const int64_t J = std::max<int64_t>((f + 63) / 64, (d + 127) / 128);
  return std::min<int64_t>(chunks * J * tc::D_MAX_SPLITS, 1536);
}

int64_t decode_counter_cap(int64_t rows, int G, int d, int f) {
  const int64_t chunks = (rows + tc::D_BN - 1) / tc::D_BN + G;
  const int64_t J = std::max<int64_t>((f + 63) / 64, (d + 127) / 128);
  return chunks * J;
}

cudaError_t launch_grouped_ffn_bf16_decode(const GroupedFfnArgs& a, cudaStream_t stream) {
  using namespace tc;
  if (a.rows == 0) return cudaSuccess;
  if (a.partial == nullptr || a.counters == nullptr) return cudaErrorInvalidValue;
  const int G = a.offsets ? a.G : 1;
  const int ctas = device_sm_count();
  const uint64_t lim = a.wait_limit_ns ? a.wait_limit_ns : 2000000000ull;
  cudaError_t e = cudaMemsetAsync(a.counters, 0, sizeof(int) * (size_t)a.counter_cap, stream);
  if (e != cudaSuccess) return e;
  // GEMM-1 + SwiGLU: weight blocks of 64 gate + 64 up rows, tokens of x_perm
  const int J1 = (a.f + 63) / 64;
  const int S1 = choose_splits(expected_units(a.rows, G, a.offsets != nullptr, J1), (a.d + D_BK - 1) / D_BK, ctas);
  CUtensorMap w1, x1;
  if (!make_map(&w1, a.w_gate_up, (uint64_t)a.G * 2 * a.f, a.d, 64) || !make_map(&x1, a.a, a.rows, a.d, D_BN))
    return cudaErrorInvalidValue;
  DecodeParams p1{a.offsets, G, a.rows, a.d, a.f, J1, S1, 2 * (int64_t)a.f, a.f,
                  static_cast<__nv_bfloat16*>(a.h), a.f, a.partial, a.partial_slots, a.counters, a.counter_cap,
                  a.status, lim};
  e = launch_decode<true>(w1, x1, p1, stream);
  if (e != cudaSuccess) return e;
  // GEMM-2: weight blocks of 128 down rows, tokens of h
  const int J2 = (a.d + 127) / 128;
  const int S2 = choose_splits(expected_units(a.rows, G, a.offsets != nullptr, J2), (a.f + D_BK - 1) / D_BK, ctas);
  CUtensorMap w2, x2;
  if (!make_map(&w2, a.w_down, (uint64_t)a.G * a.d, a.f, D_BM) || !make_map(&x2, a.h, a.rows, a.f, D_BN))
    return cudaErrorInvalidValue;
  DecodeParams p2{a.offsets, G, a.rows, a.f, a.d, J2, S2, (int64_t)a.d, 0, static_cast<__nv_bfloat16*>(a.y), a.d,
                  a.partial, a.partial_slots, a.counters, a.counter_cap, a.status, lim};
  return launch_decode<false>(w2, x2, p2, stream);
}

}  // namespace moe
