// The C ABI of include/moe.h: host-side argument checks, workspace carving
// and the launch sequence of the layer on the caller's stream.  Nothing here
// allocates device memory or synchronises, except moe_device_status.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "../../include/moe.h"
#include "common.cuh"
#include "host_guard.cuh"
#include "kernels.cuh"

namespace moe {

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

int device_smem_per_block() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 227 * 1024;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess || n <= 0)
    return 227 * 1024;
  return n;
}

// Router kernel choice: with many experts the router is a real GEMM
// (2*T*d*E flops: 30 GFLOP for T=8192, d=7168, E=256) and runs on the tensor
// cores with the top-k fused into the epilogue; with few experts (or fp32,
// which must not use TF32) W_r fits in shared memory and a warp per token on
// the CUDA cores is cheaper than a 128-token tensor tile; a decode-sized batch
// (at most 64 tokens) gets a block per token on the CUDA cores either way.
cudaError_t launch_router_topk(const RouterArgs& a, cudaStream_t stream) {
  if (router_uses_tc(a.bf16, a.E, a.T)) return launch_router_topk_tc(a, stream);
  return launch_router_topk_simt(a, stream);
}

moe_status check_config(const moe_config* c) {
  if (c == nullptr) return MOE_ERR_INVALID_ARG;
  if (c->T < 0 || c->d_model <= 0 || c->d_ff <= 0 || c->n_experts <= 0 || c->top_k <= 0) return MOE_ERR_INVALID_ARG;
  if (c->d_model % 8 != 0 || c->d_ff % 8 != 0) return MOE_ERR_INVALID_ARG;
  if (c->top_k > c->n_experts) return MOE_ERR_INVALID_ARG;
  if (c->dtype != MOE_F32 && c->dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (c->gating < MOE_SOFTMAX_ALL_RENORM || c->gating > MOE_SOFTMAX_ALL_NO_RENORM) return MOE_ERR_INVALID_ARG;
  if (c->expert_act != MOE_ACT_SWIGLU && c->expert_act != MOE_ACT_GELU) return MOE_ERR_INVALID_ARG;
  if (!(c->capacity_factor >= 0.0f) || std::isinf(c->capacity_factor)) return MOE_ERR_INVALID_ARG;
  if (c->bias_select_only != 0 && c->bias_select_only != 1) return MOE_ERR_INVALID_ARG;
  if (c->wait_limit_ns < 0) return MOE_ERR_INVALID_ARG;
  if (c->weight_format != MOE_W_NATIVE && c->weight_format != MOE_W_E4M3) return MOE_ERR_INVALID_ARG;
  // 8-bit experts: bf16 activations; rows of 8-bit codes must be whole 16-byte lines
  if (c->weight_format == MOE_W_E4M3 &&
      (c->dtype != MOE_BF16 || c->d_model % 16 != 0 || c->d_ff % 16 != 0 ||
       (c->n_shared > 0 && c->d_ff_shared % 16 != 0)))
    return MOE_ERR_UNSUPPORTED;
  if (c->n_shared < 0) return MOE_ERR_INVALID_ARG;
  if (c->n_shared > 0 && (c->d_ff_shared <= 0 || c->d_ff_shared % 8 != 0)) return MOE_ERR_INVALID_ARG;
  if (c->n_experts > kMaxExperts || c->top_k > kMaxTopK || c->n_shared > 1) return MOE_ERR_UNSUPPORTED;
  if (c->T * (int64_t)c->top_k >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  // tensor-map row coordinates are 32-bit
  if ((int64_t)c->n_experts * 2 * c->d_ff >= (int64_t(1) << 31) ||
      (int64_t)c->n_experts * c->d_model >= (int64_t(1) << 31))
    return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

namespace {

constexpr size_t kAlign = 256;
inline size_t up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t elem_bytes(const moe_config* c) { return c->dtype == MOE_BF16 ? 2 : 4; }

// Rows each expert keeps: ceil(T*k/E * capacity_factor) in double, at most T
// (no expert is chosen twice by one token); T*k when dropless.
int64_t capacity_rows(const moe_config* c) {
  if (c->capacity_factor == 0.0f) return c->T * c->top_k;
  const double cap = std::ceil((double)(c->T * c->top_k) / (double)c->n_experts * (double)c->capacity_factor);
  return cap >= (double)c->T ? c->T : (int64_t)cap;
}

struct Carve {
  int* status;
  int32_t *ids, *counts, *offsets, *perm, *row_of, *chunk_counts;
  float* w;
  void *x_perm, *h, *y_perm, *h_s, *y_s;
  float* partial;           // decode split-K partial tiles (bf16 decode regime only)
  int64_t partial_slots;
  int* counters;
  int64_t counter_cap;
  float* aux_part;          // router penalty partial sums [kAuxMaxBlocks][E + 1]
  // 8-bit experts: E4M3 codes and per-row scales of x_perm, h and the shared
  // expert's x and h
  uint8_t *xq, *hq, *xq_s, *hq_s;
  float *sx, *sh, *sx_s, *sh_s;
  size_t total;
};

// Does this config run its routed / shared experts on the decode kernel?
bool decode_routed(const moe_config* c) {
  return c->dtype == MOE_BF16 && use_decode_ffn(c->T * c->top_k, c->n_experts, true);
}
bool decode_shared(const moe_config* c) {
  return c->dtype == MOE_BF16 && c->n_shared > 0 && use_decode_ffn(c->T, 1, false);
}

// Lay out the workspace; with base == nullptr only sizes are computed.
Carve carve(const moe_config* c, void* base) {
  Carve k{};
  uint8_t* b = static_cast<uint8_t*>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) -> void* {
    void* p = b ? b + off : nullptr;
    off += up(bytes);
    return p;
  };
  const int64_t n = c->T * c->top_k;
  const size_t eb = elem_bytes(c);
  k.status = static_cast<int*>(take(16));
  k.ids = static_cast<int32_t*>(take(sizeof(int32_t) * n));
  k.w = static_cast<float*>(take(sizeof(float) * n));
  k.counts = static_cast<int32_t*>(take(sizeof(int32_t) * c->n_experts));
  k.offsets = static_cast<int32_t*>(take(sizeof(int32_t) * (c->n_experts + 1)));
  k.perm = static_cast<int32_t*>(take(sizeof(int32_t) * n));
  k.row_of = static_cast<int32_t*>(take(sizeof(int32_t) * n));
  k.chunk_counts = static_cast<int32_t*>(take(sizeof(int32_t) * (size_t)c->n_experts * permute_n_chunks(n)));
  // with 8-bit experts moe_forward gathers E4M3 codes (xq) and no bf16 copy
  k.x_perm = take(c->weight_format == MOE_W_E4M3 ? 0 : eb * n * c->d_model);
  k.h = take(eb * n * c->d_ff);
  k.y_perm = take(eb * n * c->d_model);
  if (c->n_shared > 0) {
    k.h_s = take(eb * c->T * c->d_ff_shared);
    k.y_s = take(eb * c->T * c->d_model);
  }
  k.aux_part = static_cast<float*>(take(sizeof(float) * (size_t)kAuxMaxBlocks * (c->n_experts + 1)));
  if (c->weight_format == MOE_W_E4M3) {
    k.xq = static_cast<uint8_t*>(take((size_t)n * c->d_model));
    k.sx = static_cast<float*>(take(sizeof(float) * n));
    k.hq = static_cast<uint8_t*>(take((size_t)n * c->d_ff));
    k.sh = static_cast<float*>(take(sizeof(float) * n));
    if (c->n_shared > 0) {
      k.xq_s = static_cast<uint8_t*>(take((size_t)c->T * c->d_model));
      k.sx_s = static_cast<float*>(take(sizeof(float) * c->T));
      k.hq_s = static_cast<uint8_t*>(take((size_t)c->T * c->d_ff_shared));
      k.sh_s = static_cast<float*>(take(sizeof(float) * c->T));
    }
  }
  if (decode_routed(c) || decode_shared(c)) {
    k.partial_slots = decode_partial_slots();
    k.partial = static_cast<float*>(take(sizeof(float) * 128 * kDecodeTokens * (size_t)k.partial_slots));
    k.counter_cap = std::max(decode_counter_cap(n, c->n_experts, c->d_model, c->d_ff),
                             c->n_shared ? decode_counter_cap(c->T, 1, c->d_model, c->d_ff_shared) : 0);
    k.counters = static_cast<int*>(take(sizeof(int) * (size_t)k.counter_cap));
  }
  k.total = off;
  return k;
}

moe_status check_ws(const moe_config* c, const void* ws, size_t ws_bytes) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < carve(c, nullptr).total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

uint64_t wait_limit(const moe_config* c) { return c->wait_limit_ns > 0 ? (uint64_t)c->wait_limit_ns : 2000000000ull; }

// After a call's host checks: the injected launch failure (host_guard.cuh),
// then the switch to the device that owns `p` and the check of the stream.
moe_status enter(DeviceGuard& g, const void* p, cudaStream_t stream) {
  if (launch_failure_injected()) return MOE_ERR_CUDA;
  const moe_status st = g.bind(p);
  return st != MOE_OK ? st : g.check_stream(stream);
}

// a_quantized: 8-bit experts whose input rows are already in xq / sx;
// chained: a layer step that cleared the decode counters ahead and chains its
// launches (pdl.cuh)
cudaError_t run_ffn(const moe_config* c, const Carve& k, const void* a, const int32_t* offsets, int G, int64_t rows,
                    int f, const void* w_gu, const void* w_d, void* h, void* y, cudaStream_t s, bool shared = false,
                    bool a_quantized = false, bool chained = false) {
  GroupedFfnArgs g{a, offsets, w_gu, w_d, h, y, rows, G, c->d_model, f, c->expert_act, k.status, wait_limit(c),
                   false, nullptr, nullptr, nullptr, k.partial, k.partial_slots, k.counters, k.counter_cap,
                   chained};
  if (c->dtype != MOE_BF16) return launch_grouped_ffn_f32_simt(g, s);
  if (c->weight_format == MOE_W_E4M3) {
    // the expert input -> E4M3 codes and per-token scales (only the rows in use)
    uint8_t* xq = shared ? k.xq_s : k.xq;
    float* sx = shared ? k.sx_s : k.sx;
    if (!a_quantized) {
      const cudaError_t e = launch_quantize_e4m3(a, rows, offsets ? offsets + G : nullptr, c->d_model, xq, sx, s);
      if (e != cudaSuccess) return e;
    }
    g.a = xq;
    g.fp8 = true;
    g.sa = sx;
    g.hq = shared ? k.hq_s : k.hq;
    g.sh = shared ? k.sh_s : k.sh;
  }
  if (k.partial != nullptr && use_decode_ffn(rows, G, offsets != nullptr)) return launch_grouped_ffn_bf16_decode(g, s);
  return launch_grouped_ffn_bf16_tc(g, s);
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_workspace_bytes(const moe_config* cfg) {
  if (check_config(cfg) != MOE_OK) return 0;
  return carve(cfg, nullptr).total;
}

size_t moe_e4m3_weight_bytes(int64_t rows, int64_t cols) {
  if (rows < 0 || cols <= 0 || cols % 16 != 0) return 0;
  return e4m3_codes_bytes(rows, cols) + sizeof(float) * (size_t)rows;
}

moe_status moe_quantize_e4m3(const void* src, int64_t rows, int32_t cols, void* blob, moe_stream_t stream) {
  if (rows < 0 || cols <= 0 || cols % 16 != 0) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (!src || !blob || !aligned16(src) || (reinterpret_cast<uintptr_t>(blob) % kAlign) != 0)
    return MOE_ERR_INVALID_ARG;
  DeviceGuard g;
  const moe_status st = enter(g, blob, stream);
  if (st != MOE_OK) return st;
  uint8_t* q = static_cast<uint8_t*>(blob);
  float* sc = reinterpret_cast<float*>(q + e4m3_codes_bytes(rows, cols));
  MOE_CUDA_TRY(launch_quantize_e4m3(src, rows, nullptr, cols, q, sc, stream));
  return MOE_OK;
}

int64_t moe_expert_capacity(const moe_config* cfg) {
  if (check_config(cfg) != MOE_OK) return -1;
  return capacity_rows(cfg);
}

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_TIMEOUT: return "device wait timed out";
    case MOE_ERR_BAD_EXPERT_ID: return "expert id out of range";
  }
  return "unknown status";
}

moe_status moe_router_topk(const moe_config* cfg, const void* x, const void* w_router, const float* logit_bias,
                           int32_t* topk_ids, float* topk_w, void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!x || !w_router || !topk_ids || !topk_w || !aligned16(x) || !aligned16(w_router) || !aligned16(topk_ids) ||
      !aligned16(topk_w) || (logit_bias && !aligned16(logit_bias)))
    return MOE_ERR_INVALID_ARG;
  DeviceGuard g;
  if ((st = enter(g, ws, stream)) != MOE_OK) return st;
  Carve k = carve(cfg, ws);
  RouterArgs a{x, w_router, logit_bias, topk_ids, topk_w, cfg->T, cfg->d_model, cfg->n_experts, cfg->top_k,
               cfg->gating, cfg->bias_select_only, cfg->dtype == MOE_BF16, k.status, wait_limit(cfg)};
  MOE_CUDA_TRY(launch_router_topk(a, stream));
  return MOE_OK;
}

moe_status moe_router_aux_losses(const moe_config* cfg, const void* x, const void* w_router, const int32_t* counts,
                                 float* out, void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
  if (!counts || !out || !aligned16(counts) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  if (cfg->T > 0 && (!x || !w_router || !aligned16(x) || !aligned16(w_router))) return MOE_ERR_INVALID_ARG;
  DeviceGuard g;
  if ((st = enter(g, ws, stream)) != MOE_OK) return st;
  if (cfg->T == 0) {
    MOE_CUDA_TRY(cudaMemsetAsync(out, 0, 2 * sizeof(float), stream));
    return MOE_OK;
  }
  Carve k = carve(cfg, ws);
  // the selection itself is recomputed into the workspace and discarded
  RouterArgs a{x, w_router, nullptr, k.ids, k.w, cfg->T, cfg->d_model, cfg->n_experts, cfg->top_k,
               cfg->gating, cfg->bias_select_only, cfg->dtype == MOE_BF16, k.status, wait_limit(cfg), k.aux_part};
  MOE_CUDA_TRY(launch_router_aux_losses(a, counts, out, stream));
  return MOE_OK;
}

moe_status moe_permute(const moe_config* cfg, const int32_t* topk_ids, const void* x, int32_t* counts,
                       int32_t* offsets, int32_t* perm, int32_t* row_of, void* x_perm, void* ws, size_t ws_bytes,
                       moe_stream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
  if (!counts || !offsets || !aligned16(counts) || !aligned16(offsets)) return MOE_ERR_INVALID_ARG;
  if (cfg->T > 0 && (!topk_ids || !perm || !row_of || !x || !x_perm || !aligned16(topk_ids) || !aligned16(perm) ||
                     !aligned16(row_of) || !aligned16(x) || !aligned16(x_perm)))
    return MOE_ERR_INVALID_ARG;
  DeviceGuard g;
  if ((st = enter(g, ws, stream)) != MOE_OK) return st;
  Carve k = carve(cfg, ws);
  PermuteArgs a{topk_ids, x, counts, offsets, perm, row_of, x_perm, k.chunk_counts, cfg->T * cfg->top_k,
                cfg->top_k, cfg->d_model, cfg->n_experts, (int)elem_bytes(cfg), k.status, capacity_rows(cfg)};
  MOE_CUDA_TRY(launch_permute(a, stream));
  return MOE_OK;
}

moe_status moe_grouped_ffn(const moe_config* cfg, const void* x_perm, const int32_t* offsets, const void* w_gate_up,
                           const void* w_down, void* y_perm, void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!x_perm || !offsets || !w_gate_up || !w_down || !y_perm || !aligned16(x_perm) || !aligned16(offsets) ||
      !aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(y_perm))
    return MOE_ERR_INVALID_ARG;
  DeviceGuard g;
  if ((st = enter(g, ws, stream)) != MOE_OK) return st;
  Carve k = carve(cfg, ws);
  MOE_CUDA_TRY(run_ffn(cfg, k, x_perm, offsets, cfg->n_experts, cfg->T * cfg->top_k, cfg->d_ff, w_gate_up, w_down,
                       k.h, y_perm, stream));
  return MOE_OK;
}

moe_status moe_combine(const moe_config* cfg, const void* y_perm, const int32_t* row_of, const float* topk_w,
                       const void* y_shared, void* y, moe_stream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (!y_perm || !row_of || !topk_w || !y || !aligned16(y_perm) || !aligned16(row_of) || !aligned16(topk_w) ||
      !aligned16(y) || (y_shared && !aligned16(y_shared)))
    return MOE_ERR_INVALID_ARG;
  DeviceGuard g;
  if ((st = enter(g, y, stream)) != MOE_OK) return st;
  CombineArgs a{y_perm, row_of, topk_w, y_shared, y, cfg->T, cfg->top_k, cfg->d_model, cfg->dtype == MOE_BF16};
  MOE_CUDA_TRY(launch_combine(a, stream));
  return MOE_OK;
}

moe_status moe_forward(const moe_config* cfg, const void* x, const void* w_router, const float* logit_bias,
                       const void* w_gate_up, const void* w_down, const void* ws_gate_up, const void* ws_down,
                       void* y, int32_t* opt_topk_ids, float* opt_topk_w, int32_t* opt_counts, void* ws,
                       size_t ws_bytes, moe_stream_t stream) {
  return moe_forward_traced(cfg, x, w_router, logit_bias, w_gate_up, w_down, ws_gate_up, ws_down, y, opt_topk_ids,
                            opt_topk_w, opt_counts, ws, ws_bytes, stream, nullptr);
}

moe_status moe_forward_traced(const moe_config* cfg, const void* x, const void* w_router, const float* logit_bias,
                              const void* w_gate_up, const void* w_down, const void* ws_gate_up,
                              const void* ws_down, void* y, int32_t* opt_topk_ids, float* opt_topk_w,
                              int32_t* opt_counts, void* ws, size_t ws_bytes, moe_stream_t stream,
                              const moe_event_t* stage_events) {
  // stage boundary i: record stage_events[i] (when given) on the stream
  auto mark = [&](int i) -> cudaError_t {
    if (stage_events == nullptr || stage_events[i] == nullptr) return cudaSuccess;
    return cudaEventRecord(stage_events[i], stream);
  };
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  if ((st = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return st;
  if (cfg->T == 0) {  // nothing to read or write: clear the status word and the optional counts
    if (opt_counts && !aligned16(opt_counts)) return MOE_ERR_INVALID_ARG;
    DeviceGuard g;
    if ((st = enter(g, ws, stream)) != MOE_OK) return st;
    MOE_CUDA_TRY(cudaMemsetAsync(ws, 0, 16, stream));
    if (opt_counts) MOE_CUDA_TRY(cudaMemsetAsync(opt_counts, 0, sizeof(int32_t) * cfg->n_experts, stream));
    return MOE_OK;
  }
  if (!x || !w_router || !w_gate_up || !w_down || !y || !aligned16(x) || !aligned16(w_router) ||
      !aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(y) || (logit_bias && !aligned16(logit_bias)) ||
      (opt_topk_ids && !aligned16(opt_topk_ids)) || (opt_topk_w && !aligned16(opt_topk_w)) ||
      (opt_counts && !aligned16(opt_counts)))
    return MOE_ERR_INVALID_ARG;
  if (cfg->n_shared > 0 && (!ws_gate_up || !ws_down || !aligned16(ws_gate_up) || !aligned16(ws_down)))
    return MOE_ERR_INVALID_ARG;
  DeviceGuard g;
  if ((st = enter(g, ws, stream)) != MOE_OK) return st;
  if ((st = g.same_device(x)) != MOE_OK) return st;
  Carve k = carve(cfg, ws);
  MOE_CUDA_TRY(mark(0));
  MOE_CUDA_TRY(cudaMemsetAsync(k.status, 0, 16, stream));
  // The launches of the step are chained (pdl.cuh): each kernel after the
  // router may be scheduled while its predecessor finishes.  The decode
  // kernels' unit counters are cleared here, ahead of the chain, instead of
  // by a clearing launch in front of GEMM-1.
  if (k.counters) MOE_CUDA_TRY(cudaMemsetAsync(k.counters, 0, sizeof(int) * (size_t)k.counter_cap, stream));
  int32_t* ids = opt_topk_ids ? opt_topk_ids : k.ids;
  float* w = opt_topk_w ? opt_topk_w : k.w;
  int32_t* counts = opt_counts ? opt_counts : k.counts;
  RouterArgs ra{x, w_router, logit_bias, ids, w, cfg->T, cfg->d_model, cfg->n_experts, cfg->top_k,
                cfg->gating, cfg->bias_select_only, cfg->dtype == MOE_BF16, k.status, wait_limit(cfg)};
  MOE_CUDA_TRY(launch_router_topk(ra, stream));
  MOE_CUDA_TRY(mark(1));
  // 8-bit experts: the dispatch writes no bf16 copy; each token is quantised
  // once, straight from x, and its codes go to its rows
  const bool e4m3 = cfg->weight_format == MOE_W_E4M3;
  PermuteArgs pa{ids, x, counts, k.offsets, k.perm, k.row_of, e4m3 ? nullptr : k.x_perm, k.chunk_counts,
                 cfg->T * cfg->top_k, cfg->top_k, cfg->d_model, cfg->n_experts, (int)elem_bytes(cfg), k.status,
                 capacity_rows(cfg), true};
  MOE_CUDA_TRY(launch_permute(pa, stream));
  if (e4m3)
    MOE_CUDA_TRY(
        launch_gather_quantize_e4m3(x, k.row_of, cfg->top_k, cfg->T, cfg->d_model, k.xq, k.sx, true, stream));
  MOE_CUDA_TRY(mark(2));
  MOE_CUDA_TRY(run_ffn(cfg, k, k.x_perm, k.offsets, cfg->n_experts, cfg->T * cfg->top_k, cfg->d_ff, w_gate_up,
                       w_down, k.h, k.y_perm, stream, false, e4m3, true));
  MOE_CUDA_TRY(mark(3));
  if (cfg->n_shared > 0)
    MOE_CUDA_TRY(run_ffn(cfg, k, x, nullptr, 1, cfg->T, cfg->d_ff_shared, ws_gate_up, ws_down, k.h_s, k.y_s, stream,
                         true, false, true));
  MOE_CUDA_TRY(mark(4));
  CombineArgs ca{k.y_perm, k.row_of, w, cfg->n_shared > 0 ? k.y_s : nullptr, y, cfg->T, cfg->top_k,
                 cfg->d_model, cfg->dtype == MOE_BF16, true};
  MOE_CUDA_TRY(launch_combine(ca, stream));
  MOE_CUDA_TRY(mark(5));
  return MOE_OK;
}

moe_status moe_device_status(const void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (ws == nullptr || ws_bytes < 16 || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0) return MOE_ERR_INVALID_ARG;
  MOE_CUDA_TRY(cudaStreamSynchronize(stream));
  int v = 0;
  MOE_CUDA_TRY(cudaMemcpy(&v, ws, sizeof(int), cudaMemcpyDeviceToHost));
  if (v == kDevTimeout) return MOE_ERR_TIMEOUT;
  if (v == kDevBadExpertId) return MOE_ERR_BAD_EXPERT_ID;
  return v == 0 ? MOE_OK : MOE_ERR_CUDA;
}

}  // extern "C"
