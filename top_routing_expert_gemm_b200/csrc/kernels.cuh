// Host-side launchers of the MoE kernels (internal to the library; the public
// surface is include/moe.h).  Every launcher is asynchronous on `stream` and
// returns the cudaError_t of its launch(es).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// ---- router + top-k + gate weights (router_topk.cu)
struct RouterArgs {
  const void* x;          // [T, d]
  const void* w_router;   // [E, d]
  const float* bias;      // [E] or null
  int32_t* ids;           // [T, k]
  float* w;               // [T, k]
  int64_t T;
  int d, E, k, gating, bias_select_only;
  bool bf16;
  int* status;
  uint64_t wait_limit_ns;
  // router penalties only: per-block sums [blocks][E + 1] (softmax probabilities
  // of the bias-free logits per expert, then squared log-sum-exp), or null
  float* aux_part;
};
constexpr int kAuxMaxBlocks = 2048;  // router blocks of a penalty pass, at most
// Does the router run on the tensor cores (launch_router_topk_tc)?
inline bool router_uses_tc(bool bf16, int E, int64_t T) { return bf16 && E >= 64 && E <= 256 && T > 64; }
cudaError_t launch_router_topk(const RouterArgs& a, cudaStream_t stream);       // picks one of:
cudaError_t launch_router_topk_simt(const RouterArgs& a, cudaStream_t stream);  // CUDA cores, any dtype
cudaError_t launch_router_topk_tc(const RouterArgs& a, cudaStream_t stream);    // tcgen05, bf16, E <= 256
// The CUDA-core router with the penalty sums (a.aux_part set), then the
// reduction into out[0] = balance loss, out[1] = z-loss.
cudaError_t launch_router_aux_losses(const RouterArgs& a, const int32_t* counts, float* out, cudaStream_t stream);

// ---- dispatch (permute.cu)
struct PermuteArgs {
  const int32_t* ids;     // [T*k]
  const void* x;          // [T, d] or null (skip the gather)
  int32_t* counts;        // [E]
  int32_t* offsets;       // [E+1]
  int32_t* perm;          // [T*k]
  int32_t* row_of;        // [T*k]
  void* x_perm;           // [T*k, d] or null
  int32_t* chunk_counts;  // scratch [E * n_chunks]
  int64_t n_assign;       // T*k
  int k, d, E;
  int elem_bytes;
  int* status;
  int64_t capacity;       // rows each expert keeps (n_assign or more: dropless)
  bool chained;           // the dispatch kernels may be launched programmatically (pdl.cuh)
};
int permute_n_chunks(int64_t n_assign);
cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t stream);

// ---- grouped expert GEMMs
// Rows [offsets[g], offsets[g+1]) of A use weight group g.  offsets == null
// means a single group covering rows [0, rows).
struct GroupedFfnArgs {
  const void* a;          // [rows, d]
  const int32_t* offsets; // [G+1] or null
  const void* w_gate_up;  // [G, 2f, d] (SwiGLU) or [G, f, d] (GELU: up rows only)
  const void* w_down;     // [G, d, f]
  void* h;                // [rows, f] scratch
  void* y;                // [rows, d]
  int64_t rows;           // rows of a / h / y (T*k, or T for a shared expert)
  int G, d, f;
  int act;                // kEpiSwiGLU or kEpiGELU
  int* status;
  uint64_t wait_limit_ns;
  // 8-bit experts (fp8 set): a holds E4M3 codes with per-row scales sa; the
  // weights are E4M3 blobs (codes [rows, cols], then fp32 per-row scales at
  // e4m3_codes_bytes(rows, cols)); hq / sh take h re-quantised per token row
  bool fp8;
  const float* sa;
  uint8_t* hq;
  float* sh;
  // decode kernel only: fp32 partial tiles of units cut between CTAs, and
  // one arrival counter per unit
  float* partial;
  int64_t partial_slots;
  int* counters;
  int64_t counter_cap;
  // decode kernel: the counters were zeroed ahead of this call, so GEMM-1 is
  // launched programmatically after its predecessor (pdl.cuh) with no clearing
  bool chained;
};
constexpr int kDecodeMaxCtas = 160;  // CTAs of one decode-schedule launch, at most
constexpr int kDecodeTokens = 64;    // most tokens per unit of the decode schedule
cudaError_t launch_grouped_ffn_bf16_tc(const GroupedFfnArgs& a, cudaStream_t stream);      // tcgen05, token rows as M
cudaError_t launch_grouped_ffn_bf16_decode(const GroupedFfnArgs& a, cudaStream_t stream);  // tcgen05, weight rows as M
cudaError_t launch_grouped_ffn_f32_simt(const GroupedFfnArgs& a, cudaStream_t stream);      // fp32 CUDA cores
// decode regime: at most kDecodeTokens rows per touched group on average (uniform-routing expectation)
bool use_decode_ffn(int64_t rows, int G, bool grouped);
int64_t decode_partial_slots();  // [128][64] fp32 tiles
int64_t decode_counter_cap(int64_t rows, int G, int d, int f);

// ---- FP8 E4M3 row quantisation (quant_e4m3.cu): per row s = max|x| / 448,
// q = e4m3(x / s); rows past *rows_dev (when given) are left alone.
// amax_bits (may be `scale` itself): each row's max|x| as bf16 bits, known
// ahead, so the row is read once
cudaError_t launch_quantize_e4m3(const void* src, int64_t rows, const int32_t* rows_dev, int cols, uint8_t* q,
                                 float* scale, cudaStream_t stream, const uint32_t* amax_bits = nullptr);
// the dispatch with 8-bit experts: token t of x [T, cols] quantised once, its
// codes and scale written to every kept row row_of[t*k + s]
cudaError_t launch_gather_quantize_e4m3(const void* x, const int32_t* row_of, int k, int64_t T, int cols,
                                        uint8_t* q, float* scale, bool chained, cudaStream_t stream);
inline size_t e4m3_codes_bytes(int64_t rows, int64_t cols) { return ((size_t)(rows * cols) + 255) / 256 * 256; }

// ---- combine (combine.cu)
struct CombineArgs {
  const void* y_perm;     // [T*k, d]
  const int32_t* row_of;  // [T*k]
  const float* w;         // [T, k]
  const void* y_shared;   // [T, d] or null
  void* y;                // [T, d]
  int64_t T;
  int k, d;
  bool bf16;
  bool chained;  // may be launched programmatically after the expert GEMMs (pdl.cuh)
};
cudaError_t launch_combine(const CombineArgs& a, cudaStream_t stream);

int device_sm_count();
int device_smem_per_block();  // opt-in dynamic shared memory per block (227 KiB on B200)

}  // namespace moe
