// Grouped expert GEMMs on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// "Mixture of Experts: why a model with 671 billion parameters uses only 37",
// "How data centres handle it": tokens grouped by their assigned expert and
// all expert multiplies run in a single launch over a stacked weight matrix.
// Expert FFN: "Mixture of Experts Explained: Routers, Active Parameters and
// VRAM" (a gated feed-forward block with three matrices), read as SwiGLU.
//
//   GEMM-1 (MODE_SWIGLU): h[rows, f] = SiLU(A Wg^T) * (A Wu^T), one launch
//     over every expert; each 128 x N accumulator holds N/2 gate columns and
//     the matching N/2 up columns (the B tile is the gate rows followed by the
//     up rows), so the SwiGLU is applied in the epilogue straight out of
//     tensor memory and only h (bf16) reaches HBM.
//   GEMM-1 (MODE_GELU, the two-matrix expert): h[rows, f] = GELU(A Wu^T).
//   GEMM-2 (MODE_PLAIN):  y[rows, d] = h Wd^T.
//   Router (MODE_ROUTER): logits = x W_r^T with N = E rounded up to 16; the
//     epilogue keeps the top k per row and writes ids and gate weights (one
//     CTA per 128-token tile; see the epilogue).
//
// Persistent, warp-specialised CTA (one CTA per SM):
//   warp 0     TMA producer: ring of (A 128x64, B Nx64) bf16 tiles (128x128
//              and Nx128 with 8-bit operands), 128-byte swizzle, mbarrier
//              transaction counts; four stages of N = 256, or five of N = 224
//              where that width pads the output less (bf16 only)
//   warp 1     TMEM allocator and single-thread tcgen05.mma issuer
//              (M=128, N<=256, K=16 per instruction (32 for 8-bit), fp32
//              accumulators)
//   warps 2..  epilogue: tcgen05.ld of their 32-lane quarter, SwiGLU / bf16
//              conversion, masked 16-byte stores; four warps in bf16, eight
//              with 8-bit operands and in the router (kThreads)
// Two 256-column accumulators (all 512 TMEM columns) let the epilogue of tile
// i overlap the main loop of tile i+1.
//
// Tiles are (group, n-tile, m-tile) with the m-tile fastest, read from the
// device offsets at kernel start (no host sync): CTAs that run together share
// one expert's weight panel, so it crosses HBM about once while its row
// blocks are still in L2.  An expert with more than 16 m-tiles (a hot expert
// of skewed routing) is walked in blocks of 16 m-tiles, so its token rows do
// not fall out of L2 between weight panels.  Rows past a group's end are
// computed on whatever the TMA box holds (the next group's rows or zero fill)
// and never stored.
//
// Every wait is bounded (Params::wait_limit_ns).  On expiry the CTA raises a
// shared abort flag and the device status word, lets its in-flight TMA loads
// and MMAs land, frees its tensor memory and returns.
#include <cudaTypedefs.h>

#include "kernels.cuh"
#include "tc_primitives.cuh"

namespace moe {
namespace tc {

// ---------------------------------------------------------------- tensor maps (host)
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

// row-major [rows, cols] tensor of bf16 or 8-bit elements, box = box_rows x
// one 128-byte swizzle row (64 bf16 or 128 e4m3)
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows, int elem_bytes) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * (uint64_t)elem_bytes};
  cuuint32_t box[2] = {128u / (cuuint32_t)elem_bytes, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt = elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


namespace {

constexpr int BM = 128, BK = 64;
constexpr int MODE_SWIGLU = 0, MODE_PLAIN = 1, MODE_ROUTER = 2, MODE_GELU = 3;

// warp 0 TMA, warp 1 MMA, then the epilogue warps: four (one per TMEM lane
// quarter) with bf16 operands; eight (two per quarter, alternate 32-column
// chunks) with 8-bit ones, whose K loop is half as long per tile, so that the
// epilogue of a tile still fits under the next tile's main loop, and in the
// router, whose per-row top-k selection is a serial chain of compares that
// two threads per row halve
template <bool FP8, int MODE>
constexpr int kThreads = (FP8 || MODE == MODE_ROUTER) ? 320 : 192;
constexpr int BN_MMA = 256;
constexpr int A_BYTES = BM * BK * 2;       // 16 KiB
constexpr int TMEM_COLS = 2 * BN_MMA;      // two accumulators
// Operand ring of an MMA width NB: four stages of N = 256 (48 KiB each), or
// five of N = 224 (44 KiB each: a quarter more bytes in flight), which the
// bf16 expert GEMMs take where 224 columns per tile pad the output less
template <int NB>
constexpr int kStages = NB == 224 ? 5 : 4;
template <int NB>
constexpr int kBBytes = NB * BK * 2;
struct Params {
  const int32_t* offsets;  // [G+1] device, or null: one group of `rows` rows
  int G;
  int64_t rows;            // rows of A and of the output
  int K;                   // reduction length
  int N;                   // output columns
  int nt;                  // n-tiles per group
  int64_t b_group_rows;    // rows of B per group (2f or d)
  int up_off;              // row offset of the up half inside a group (f)
  void* out;
  int64_t ldo;
  int* status;
  uint64_t wait_limit_ns;
  int n_mma;               // MMA N (256, or the padded expert count of the router)
  // 8-bit operands only: per-row scales of A (tokens) and of B (weight rows,
  // indexed like the rows of the B tensor map)
  const float* sa;
  const float* sb;
  // router epilogue only
  const float* bias;       // [E] or null
  int32_t* ids;            // [rows, k]
  float* wts;              // [rows, k]
  int E, k, gating, bias_select_only;
  // 8-bit GEMM-1 only: per row, the largest |h| stored, as bf16 bits (an
  // atomic maximum over the row's tiles; zero on entry), or null
  uint32_t* row_amax;
};

// router: the tile's logits are staged in shared memory over the drained
// operand ring, 260 floats per row (16-byte rows that start on different banks)
constexpr int kLogStride = 260;
static_assert(128 * kLogStride * 4 <= kStages<256> * (A_BYTES + kBBytes<256>), "router logits fit over the ring");
constexpr size_t kRouterBarBytes = 8;  // one mbarrier

template <int NB>
size_t smem_bytes(int G, int E) {
  return 1024 + (size_t)kStages<NB> * (A_BYTES + kBBytes<NB>) + 256 + 2 * sizeof(int) * (size_t)(G + 1) +
         sizeof(float) * (size_t)E + (E > 0 ? 8 + kRouterBarBytes : 0);
}

// m-tiles per block of the tile order: an expert with more m-tiles than this
// runs them block by block, so its token rows in flight (one block, 2048
// rows) stay in L2 while every weight panel passes over them
constexpr int kMBlock = 16;

// tile t -> (group, m-tile, n-tile): group g owns tiles [cum[g]*nt, cum[g+1]*nt);
// inside it, blocks of kMBlock m-tiles, then the n-tile, then the m-tile
__device__ __forceinline__ void decode_tile(int64_t t, int nt, const int* cum, int G, int& g, int& mt, int& ntile) {
  int lo = 0, hi = G;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if ((int64_t)cum[mid] * nt <= t) lo = mid;
    else hi = mid;
  }
  g = lo;
  const int mtiles = cum[lo + 1] - cum[lo];
  const int64_t local = t - (int64_t)cum[lo] * nt;
  const int mb = (int)(local / ((int64_t)kMBlock * nt));
  const int64_t rest = local - (int64_t)mb * kMBlock * nt;
  const int nb = min(kMBlock, mtiles - mb * kMBlock);  // m-tiles in this block
  ntile = (int)(rest / nb);
  mt = mb * kMBlock + (int)(rest % nb);
}


// FP8: A and B are E4M3 codes; a stage's 128-byte K slice holds 128 of them
// (kind::f8f6f4, K = 32 per MMA) instead of 64 bf16, and the epilogue scales
// each accumulator by its token's and its weight row's scale.
template <int MODE, int KMAX, bool FP8, int NB>
__global__ void __launch_bounds__(kThreads<FP8, MODE>, 1)
    grouped_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const Params p) {
  constexpr int STAGES = kStages<NB>, B_BYTES = kBBytes<NB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + STAGES * B_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = bars + 2 * STAGES + 2;
  uint64_t* drain = bars + 2 * STAGES + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* fill_par = reinterpret_cast<int*>(tmem_slot + 2);  // [STAGES]
  int* s_off = fill_par + STAGES;                          // [G+1]
  int* s_cum = s_off + (p.G + 1);                          // [G+1]
  float* s_bias = reinterpret_cast<float*>(s_cum + (p.G + 1));  // [E], router only
  // router hand-off (after s_bias, 8-byte aligned)
  uint64_t* lrdy = reinterpret_cast<uint64_t*>((reinterpret_cast<uintptr_t>(s_bias + p.E) + 7) & ~uintptr_t(7));
  float* s_log = reinterpret_cast<float*>(smem);  // router: [128][kLogStride] logits over the ring

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
      mbar_init(smem_u32(&tempty[a]), kThreads<FP8, MODE> - 64);
    }
    mbar_init(smem_u32(drain), 1);
    if (MODE == MODE_ROUTER) {
      mbar_init(smem_u32(lrdy), kThreads<FP8, MODE> - 64);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  if (MODE == MODE_ROUTER)
    for (int e = threadIdx.x; e < p.E; e += kThreads<FP8, MODE>) s_bias[e] = p.bias ? p.bias[e] : 0.f;
  if (p.offsets) {
    for (int g = threadIdx.x; g <= G; g += kThreads<FP8, MODE>) s_off[g] = p.offsets[g];
  } else if (threadIdx.x == 0) {
    s_off[0] = 0;
    s_off[1] = (int)p.rows;
  }
  __syncthreads();
  if (warp == 0) {  // cumulative m-tile counts, 32 groups per step
    int carry = 0;
    if (lane == 0) s_cum[0] = 0;
    for (int base = 0; base < G; base += 32) {
      const int g = base + lane;
      int v = 0;
      if (g < G) v = max(0, (s_off[g + 1] - s_off[g] + BM - 1) / BM);
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
  const int64_t total = (int64_t)s_cum[G] * p.nt;
  constexpr int KB = FP8 ? 2 * BK : BK;  // elements per 128-byte K slice
  const int kb_count = (p.K + KB - 1) / KB;
  const int n_mma = p.n_mma;
  const int bno = MODE == MODE_SWIGLU ? n_mma / 2 : n_mma;  // output columns per tile

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      for (int64_t t = blockIdx.x; t < total; t += gridDim.x) {
        int g, mt, ntile;
        decode_tile(t, p.nt, s_cum, G, g, mt, ntile);
        const int a_row = s_off[g] + mt * BM;
        const int b_row = (int)((int64_t)g * p.b_group_rows + (int64_t)ntile * bno);
        bool ok = true;
        for (int kb = 0; kb < kb_count; ++kb) {
          if (!mbar_wait_bounded(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, p.wait_limit_ns, p.status)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&full[stage]);
          mbar_expect_tx(fb, A_BYTES + n_mma * BK * 2);
          fill_par[stage] = (int)phase;
          tma_load_2d(smem_u32(sA + stage * A_BYTES), &tmA, fb, kb * KB, a_row);
          if (MODE == MODE_SWIGLU) {  // gate rows, then the matching up rows (bno is a multiple of 8)
            tma_load_2d(smem_u32(sB + stage * B_BYTES), &tmB, fb, kb * KB, b_row);
            tma_load_2d(smem_u32(sB + stage * B_BYTES + bno * 128), &tmB, fb, kb * KB, b_row + p.up_off);
          } else {
            tma_load_2d(smem_u32(sB + stage * B_BYTES), &tmB, fb, kb * KB, b_row);
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
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      const uint32_t idesc = idesc_f32acc<FP8>(BM, n_mma);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < total && ok; t += gridDim.x) {
        if (!mbar_wait_bounded(smem_u32(&tempty[acc]), acc_phase ^ 1u, abort_flag, p.wait_limit_ns, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN_MMA);
        for (int kb = 0; kb < kb_count; ++kb) {
          if (!mbar_wait_bounded(smem_u32(&full[stage]), phase, abort_flag, p.wait_limit_ns, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * B_BYTES);
          mma_kslice<FP8>(d_tmem, a0, b0, idesc, kb == 0);
          mma_commit(smem_u32(&empty[stage]));
          if (++stage == STAGES) {
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
    // -------------------------------------------------- epilogue (warps 2..)
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    constexpr int kPerQuarter = (kThreads<FP8, MODE> - 64) / 128;  // epilogue warps per lane quarter
    const int part = (warp - 2) >> 2;                         // which of them this warp is
    const int r = q * 32 + lane;
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
    // 32-byte stores when every row segment a chunk writes starts on 32
    // bytes: the output's base, the row pitch and the tile's first column (a
    // multiple of bno) decide
    const bool st32 = (p.ldo % 16) == 0 && (bno % 16) == 0 && (reinterpret_cast<uintptr_t>(p.out) % 32) == 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t l_phase = 0;  // router: logits staged
    for (int64_t t = blockIdx.x; t < total; t += gridDim.x) {
      int g, mt, ntile;
      decode_tile(t, p.nt, s_cum, G, g, mt, ntile);
      if (!mbar_wait_bounded(smem_u32(&tfull[acc]), acc_phase, abort_flag, p.wait_limit_ns, p.status)) break;
      tc_fence_after();
      const int rows_g = s_off[g + 1] - s_off[g];
      const int lr = mt * BM + r;
      const int64_t grow = (int64_t)s_off[g] + lr;
      const bool ok = lr < rows_g && grow >= 0 && grow < p.rows;
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN_MMA);
      const int col_base = ntile * bno;
      const int col_lim = min(p.N, col_base + bno);  // this tile's columns (bno need not be a multiple of 32)
      __nv_bfloat16* orow = out + grow * p.ldo + col_base;
      // 8-bit operands: this row's token scale; weight-row scales of the tile's columns
      const float s_row = FP8 && ok ? p.sa[grow] : 1.f;
      const float* sg = FP8 ? p.sb + (int64_t)g * p.b_group_rows + col_base : nullptr;
      if (MODE != MODE_ROUTER) {
        // SwiGLU mode: gate in accumulator columns [0, bno), up in [bno, 2 bno);
        // plain mode: the bno output columns
        constexpr bool kRowMax = FP8 && (MODE == MODE_SWIGLU || MODE == MODE_GELU);
        uint32_t amax_bits = 0;  // kRowMax: the largest |h| this thread stores, as bf16 bits
#pragma unroll 1
        for (int c = 32 * part; c < bno; c += 32 * kPerQuarter) {
          uint32_t v[32], u[32];
          tmem_ld32(tb + c, v);
          if (MODE == MODE_SWIGLU) tmem_ld32(tb + bno + c, u);
          tmem_ld_wait();
          if (ok) {
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
            if (kRowMax && p.row_amax) {  // over the stored columns, as the re-quantisation reads them
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const int cc = col_base + c + 2 * j;
                if (cc < col_lim) amax_bits = max(amax_bits, pk[j] & 0x7FFFu);
                if (cc + 1 < col_lim) amax_bits = max(amax_bits, (pk[j] >> 16) & 0x7FFFu);
              }
            }
            if (col_base + c + 32 <= col_lim) {
              if (st32) {  // two whole 32-byte sectors
                st_global_32B(orow + c, pk);
                st_global_32B(orow + c + 16, pk + 8);
              } else {
                uint4* dst = reinterpret_cast<uint4*>(orow + c);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                  dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
              }
            } else {
              // a chunk past the tile's last column (the fourth of a 112-column
              // SwiGLU tile): its first 16 columns as one 32-byte store when they
              // are all in, the rest one by one
              const bool head = st32 && col_base + c + 16 <= col_lim;
              if (head) st_global_32B(orow + c, pk);
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                if (head && j < 8) continue;
                const int cc = col_base + c + 2 * j;
                if (cc < col_lim) orow[c + 2 * j] = __ushort_as_bfloat16((unsigned short)(pk[j] & 0xFFFFu));
                if (cc + 1 < col_lim) orow[c + 2 * j + 1] = __ushort_as_bfloat16((unsigned short)(pk[j] >> 16));
              }
            }
          }
        }
        if (kRowMax && p.row_amax && ok && amax_bits) atomicMax(p.row_amax + grow, amax_bits);
      } else {
        // Router: keep the top k of kappa = logit + bias over the E columns of
        // each row, then the gate weights of the chosen experts.  The CTA owns
        // this one tile (the router launch has a CTA per tile), so its operand
        // ring is drained: each thread stages its row's logits there (the two
        // warps of a lane quarter alternate 32-column chunks), then each warp
        // selects for 16 rows, four at a time (independent chains of shuffles
        // that the scheduler interleaves): lane l holds columns l, l+32, ...,
        // and k rounds of a warp-wide (kappa desc, index asc) maximum pick the
        // experts in order.
#pragma unroll 1
        for (int c = 32 * part; c < p.n_mma; c += 32 * kPerQuarter) {
          uint32_t v[32];
          tmem_ld32(tb + c, v);
          tmem_ld_wait();
          float4* dst = reinterpret_cast<float4*>(s_log + r * kLogStride + c);
#pragma unroll
          for (int j = 0; j < 8; ++j)  // n_mma is a multiple of 16
            if (c + 4 * j < p.n_mma)
              dst[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                   __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
        }
        mbar_arrive(smem_u32(lrdy));
        const bool lok = mbar_wait_bounded(smem_u32(lrdy), l_phase, abort_flag, p.wait_limit_ns, p.status);
        l_phase ^= 1u;
        if (!lok) break;
        constexpr int R = 4;                       // rows in flight per warp
        constexpr int kEpiWarps = kThreads<FP8, MODE> / 32 - 2;
        const int E = p.E, k = p.k;
        const bool all_e = p.gating == 0 || p.gating == 3;  // softmax over all E: needs the denominator
        const int64_t row0 = (int64_t)s_off[g] + (int64_t)mt * BM;
#pragma unroll 1
        for (int rb = (warp - 2) * R; rb < BM; rb += kEpiWarps * R) {
          float key[R][8], lg[R][8], mx[R], z[R], key0[R], sel_key[R], sel_val[R];
          int sel_idx[R];
#pragma unroll
          for (int q2 = 0; q2 < R; ++q2) {
#pragma unroll
            for (int m = 0; m < 8; ++m) {
              const int c = lane + 32 * m;
              lg[q2][m] = c < E ? s_log[(rb + q2) * kLogStride + c] : 0.f;
              key[q2][m] = c < E ? lg[q2][m] + s_bias[c] : -INFINITY;
            }
            mx[q2] = key[q2][0];
#pragma unroll
            for (int m = 1; m < 8; ++m) mx[q2] = fmaxf(mx[q2], key[q2][m]);
            z[q2] = 0.f;
            key0[q2] = sel_key[q2] = sel_val[q2] = 0.f;
            sel_idx[q2] = 0;
          }
#pragma unroll
          for (int off = 16; off > 0; off >>= 1)
#pragma unroll
            for (int q2 = 0; q2 < R; ++q2) mx[q2] = fmaxf(mx[q2], __shfl_xor_sync(0xffffffffu, mx[q2], off));
          if (all_e) {
#pragma unroll
            for (int q2 = 0; q2 < R; ++q2)
#pragma unroll
              for (int m = 0; m < 8; ++m)
                if (lane + 32 * m < E) z[q2] += expf(key[q2][m] - mx[q2]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
#pragma unroll
              for (int q2 = 0; q2 < R; ++q2) z[q2] += __shfl_xor_sync(0xffffffffu, z[q2], off);
          }
#pragma unroll 1
          for (int s = 0; s < k; ++s) {
            float bk[R];
            int bi[R];
#pragma unroll
            for (int q2 = 0; q2 < R; ++q2) {
              bk[q2] = key[q2][0];
              bi[q2] = lane;
#pragma unroll
              for (int m = 1; m < 8; ++m)
                if (ranks_before(key[q2][m], lane + 32 * m, bk[q2], bi[q2])) {
                  bk[q2] = key[q2][m];
                  bi[q2] = lane + 32 * m;
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
              for (int q2 = 0; q2 < R; ++q2) {
                const float ok2 = __shfl_xor_sync(0xffffffffu, bk[q2], off);
                const int oi = __shfl_xor_sync(0xffffffffu, bi[q2], off);
                if (ranks_before(ok2, oi, bk[q2], bi[q2])) {
                  bk[q2] = ok2;
                  bi[q2] = oi;
                }
              }
            }
#pragma unroll
            for (int q2 = 0; q2 < R; ++q2) {
              // the owner lane of the winner takes it out and hands over its raw logit
              const int owner = bi[q2] & 31, mw = bi[q2] >> 5;
              float cand = 0.f;
#pragma unroll
              for (int m = 0; m < 8; ++m) cand = m == mw ? lg[q2][m] : cand;
              const float bv = __shfl_sync(0xffffffffu, cand, owner);
              if (lane == owner) {
#pragma unroll
                for (int m = 0; m < 8; ++m) key[q2][m] = m == mw ? -INFINITY : key[q2][m];
              }
              if (s == 0) key0[q2] = bk[q2];
              if (lane == s) {
                sel_key[q2] = bk[q2];
                sel_idx[q2] = bi[q2];
                sel_val[q2] = bv;
              }
            }
          }
          float wv[R], den[R];
#pragma unroll
          for (int q2 = 0; q2 < R; ++q2) {
            wv[q2] = 0.f;
            if (lane < k) {
              if (all_e) wv[q2] = expf(sel_key[q2] - mx[q2]) / z[q2];
              else if (p.gating == 1) wv[q2] = expf(sel_key[q2] - key0[q2]);
              else wv[q2] = 1.0f / (1.0f + expf(-(p.bias_select_only ? sel_val[q2] : sel_key[q2])));
            }
            den[q2] = wv[q2];
          }
#pragma unroll
          for (int off = 16; off > 0; off >>= 1)
#pragma unroll
            for (int q2 = 0; q2 < R; ++q2) den[q2] += __shfl_xor_sync(0xffffffffu, den[q2], off);
#pragma unroll
          for (int q2 = 0; q2 < R; ++q2) {
            const int64_t grow_r = row0 + rb + q2;
            if (lane < k && grow_r < p.rows) {
              p.ids[grow_r * k + lane] = sel_idx[q2];
              p.wts[grow_r * k + lane] = p.gating == 3 ? wv[q2] : wv[q2] / den[q2];  // rule 3: not renormalised
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&tempty[acc]));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  if (warp == 0 && lane == 0 && !*abort_flag) {
    // every stage filled has been released by its MMAs (their completion
    // arrivals target this CTA's barriers, which must outlive them)
    for (int s = 0; s < STAGES; ++s)
      if (fill_par[s] >= 0) drain_wait(smem_u32(&empty[s]), (uint32_t)fill_par[s]);
  }
  __syncthreads();
  if (*abort_flag) {
    // let this CTA's own asynchronous copies and MMAs land before its shared
    // and tensor memory are released
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

template <int MODE, int KMAX, bool FP8 = false, int NB = 256>
cudaError_t launch_mode(const CUtensorMap& ta, const CUtensorMap& tb, const Params& p, int64_t tiles_bound,
                        cudaStream_t stream) {
  const size_t smem = smem_bytes<NB>(p.G, MODE == MODE_ROUTER ? p.E : 0);
  cudaError_t e = cudaFuncSetAttribute(grouped_gemm_tc_kernel<MODE, KMAX, FP8, NB>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int64_t grid = device_sm_count();
  if (tiles_bound < grid) grid = tiles_bound;
  // the router's epilogue stages a tile's logits over the operand ring, so
  // each CTA takes exactly one tile (tiles_bound is then the tile count)
  if (MODE == MODE_ROUTER) grid = tiles_bound;
  if (grid < 1) grid = 1;
  grouped_gemm_tc_kernel<MODE, KMAX, FP8, NB><<<(unsigned)grid, kThreads<FP8, MODE>, smem, stream>>>(ta, tb, p);
  return cudaGetLastError();
}

}  // namespace
}  // namespace tc

namespace tc {
namespace {
// The five-stage ring of N = 224 where it pads the output columns strictly
// less than N = 256 (SwiGLU: 112 against 128 output columns per tile), with
// bf16 operands, and where the group offsets fit beside it in shared memory.
// Measured on the layer shapes: both GEMMs of 2880 output columns (25.7 tiles
// of 112 against 22.5 of 128; 12.9 of 224 against 11.25 of 256) ran 2.8-4.5%
// faster; where 256 divides the output the narrower tile only costs, and the
// 8-bit kernel ran 6% slower with it.
bool deep_ring(int cols, bool swiglu, bool fp8, int G) {
  if (fp8 || smem_bytes<224>(G, 0) > (size_t)device_smem_per_block()) return false;
  const int o256 = swiglu ? 128 : 256, o224 = swiglu ? 112 : 224;
  const int64_t pad256 = (int64_t)((cols + o256 - 1) / o256) * o256 - cols;
  const int64_t pad224 = (int64_t)((cols + o224 - 1) / o224) * o224 - cols;
  return pad224 < pad256;
}

template <int MODE, bool FP8>
cudaError_t launch_ffn(bool deep, const CUtensorMap& ta, const CUtensorMap& tb, const Params& p, int64_t tiles_bound,
                       cudaStream_t stream) {
  if constexpr (!FP8) {
    if (deep) return launch_mode<MODE, 1, false, 224>(ta, tb, p, tiles_bound, stream);
  }
  return launch_mode<MODE, 1, FP8, 256>(ta, tb, p, tiles_bound, stream);
}

// Both expert GEMMs with token rows as M.  FP8: `a` holds E4M3 codes with
// per-row scales a.sa, the weights are E4M3 blobs (codes, then per-row
// scales), and h is re-quantised per token row between the two GEMMs.
template <bool FP8>
cudaError_t run_tc(const GroupedFfnArgs& a, cudaStream_t stream) {
  if (a.rows == 0) return cudaSuccess;
  const int G = a.offsets ? a.G : 1;
  const int64_t mt_bound = (a.rows + BM - 1) / BM + (a.offsets ? a.G : 0);
  const uint64_t lim = a.wait_limit_ns ? a.wait_limit_ns : 2000000000ull;
  const int eb = FP8 ? 1 : 2;
  const bool gelu = a.act == kEpiGELU;
  const bool deep1 = deep_ring(a.f, !gelu, FP8, G);
  const int n1 = deep1 ? 224 : BN_MMA;
  const int64_t w1_rows = (gelu ? 1 : 2) * (int64_t)a.G * a.f;
  const float* s1 = FP8 ? reinterpret_cast<const float*>(static_cast<const uint8_t*>(a.w_gate_up) +
                                                         e4m3_codes_bytes(w1_rows, a.d))
                        : nullptr;
  CUtensorMap mA1, mB1;
  cudaError_t e;
  // 8-bit: GEMM-1's epilogue leaves each row's largest |h| in sh (as bf16
  // bits), so the re-quantisation of h reads h once
  uint32_t* row_amax = FP8 ? reinterpret_cast<uint32_t*>(a.sh) : nullptr;
  if (FP8) {
    e = cudaMemsetAsync(a.sh, 0, sizeof(float) * (size_t)a.rows, stream);
    if (e != cudaSuccess) return e;
  }
  if (gelu) {
    // GEMM-1 + GELU: tile = 128 rows x n1 up columns
    if (!make_map(&mA1, a.a, a.rows, a.d, BM, eb) || !make_map(&mB1, a.w_gate_up, w1_rows, a.d, n1, eb))
      return cudaErrorInvalidValue;
    Params p1{a.offsets, G, a.rows, a.d, a.f, (a.f + n1 - 1) / n1, (int64_t)a.f, 0, a.h, a.f, a.status, lim, n1,
              a.sa, s1};
    p1.row_amax = row_amax;
    e = launch_ffn<MODE_GELU, FP8>(deep1, mA1, mB1, p1, mt_bound * p1.nt, stream);
  } else {
    // GEMM-1 + SwiGLU: tile = 128 rows x (n1/2 gate + n1/2 up) columns
    if (!make_map(&mA1, a.a, a.rows, a.d, BM, eb) || !make_map(&mB1, a.w_gate_up, w1_rows, a.d, n1 / 2, eb))
      return cudaErrorInvalidValue;
    Params p1{a.offsets, G, a.rows, a.d, a.f, (a.f + n1 / 2 - 1) / (n1 / 2), 2 * (int64_t)a.f, a.f, a.h, a.f,
              a.status, lim, n1, a.sa, s1};
    p1.row_amax = row_amax;
    e = launch_ffn<MODE_SWIGLU, FP8>(deep1, mA1, mB1, p1, mt_bound * p1.nt, stream);
  }
  if (e != cudaSuccess) return e;
  const void* a2 = a.h;
  const float* sa2 = nullptr;
  if (FP8) {  // h -> E4M3 codes and per-token scales
    e = launch_quantize_e4m3(a.h, a.rows, a.offsets ? a.offsets + a.G : nullptr, a.f, a.hq, a.sh, stream,
                             row_amax);
    if (e != cudaSuccess) return e;
    a2 = a.hq;
    sa2 = a.sh;
  }
  const float* s2 = FP8 ? reinterpret_cast<const float*>(static_cast<const uint8_t*>(a.w_down) +
                                                         e4m3_codes_bytes((int64_t)a.G * a.d, a.f))
                        : nullptr;
  // GEMM-2: tile = 128 rows x n2 output columns
  const bool deep2 = deep_ring(a.d, false, FP8, G);
  const int n2 = deep2 ? 224 : BN_MMA;
  CUtensorMap mA2, mB2;
  if (!make_map(&mA2, a2, a.rows, a.f, BM, eb) || !make_map(&mB2, a.w_down, (uint64_t)a.G * a.d, a.f, n2, eb))
    return cudaErrorInvalidValue;
  Params p2{a.offsets, G, a.rows, a.f, a.d, (a.d + n2 - 1) / n2, (int64_t)a.d, 0, a.y, a.d, a.status, lim, n2,
            sa2, s2};
  return launch_ffn<MODE_PLAIN, FP8>(deep2, mA2, mB2, p2, mt_bound * p2.nt, stream);
}
}  // namespace
}  // namespace tc

cudaError_t launch_grouped_ffn_bf16_tc(const GroupedFfnArgs& a, cudaStream_t stream) {
  return a.fp8 ? tc::run_tc<true>(a, stream) : tc::run_tc<false>(a, stream);
}

// Router GEMM on the tensor cores with the top-k and gate weights fused into
// the epilogue: one 128-token tile per CTA, N = E rounded up to 16 (the rows of
// W_r past E are zero-filled by the TMA box and never selected).
cudaError_t launch_router_topk_tc(const RouterArgs& a, cudaStream_t stream) {
  using namespace tc;
  if (!a.bf16 || a.E > BN_MMA || a.k > 16) return cudaErrorInvalidValue;
  const int n_mma = ((a.E + 15) / 16) * 16;
  CUtensorMap mA, mB;
  if (!make_map(&mA, a.x, (uint64_t)a.T, a.d, BM) || !make_map(&mB, a.w_router, (uint64_t)a.E, a.d, n_mma))
    return cudaErrorInvalidValue;
  const uint64_t lim = a.wait_limit_ns ? a.wait_limit_ns : 2000000000ull;
  Params p{nullptr, 1, a.T, a.d, a.E, 1, 0, 0, nullptr, 0, a.status, lim, n_mma, nullptr, nullptr,
           a.bias, a.ids, a.w, a.E, a.k, a.gating, a.bias_select_only};
  const int64_t tiles = (a.T + BM - 1) / BM;
  if (a.k <= 2) return launch_mode<MODE_ROUTER, 2>(mA, mB, p, tiles, stream);
  if (a.k <= 4) return launch_mode<MODE_ROUTER, 4>(mA, mB, p, tiles, stream);
  if (a.k <= 8) return launch_mode<MODE_ROUTER, 8>(mA, mB, p, tiles, stream);
  return launch_mode<MODE_ROUTER, 16>(mA, mB, p, tiles, stream);
}

}  // namespace moe
