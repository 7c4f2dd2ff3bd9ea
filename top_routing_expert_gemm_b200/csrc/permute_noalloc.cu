// moe_permute_noalloc: the dispatch step (stable counting sort + row gather)
// for callers that cannot hand the library a workspace.
//
// Some callers have no way to obtain device scratch at the moment they
// dispatch tokens: a plug-in whose host framework owns every device
// allocation and only passes it tensors, a serving loop whose memory policy
// forbids allocation once it has started (an allocation there can stall or
// synchronise the device), or code that must not fail on an out-of-memory
// error mid-step.  This entry point takes only the inputs and outputs; its
// per-(expert, chunk) histogram lives in a fixed array compiled into the
// library instead of in a caller-provided workspace.
#include <atomic>

#include <cuda_runtime.h>

#include "../../include/moe.h"
#include "common.cuh"
#include "host_guard.cuh"
#include "kernels.cuh"

namespace moe {
namespace {

// Scratch of the no-allocation dispatch: the per-(expert, chunk) histogram and
// starting rows.  Every GPU that loads the library holds these 256 KiB until
// the process exits.
constexpr int64_t kNoAllocScratchInts = 65536;
static __device__ __align__(256) int32_t g_permute_scratch[kNoAllocScratchInts];

// Device address of g_permute_scratch per device ordinal, looked up on the
// first call made with that device current.
constexpr int kMaxDevices = 64;
std::atomic<int32_t*> g_scratch_addr[kMaxDevices];

cudaError_t scratch_address(int32_t** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  int32_t* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    void* addr = nullptr;
    e = cudaGetSymbolAddress(&addr, g_permute_scratch);
    if (e != cudaSuccess) return e;
    p = static_cast<int32_t*>(addr);
    g_scratch_addr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace moe

extern "C" moe_status moe_permute_noalloc(const moe_config* cfg, const int32_t* topk_ids, const void* x,
                                          int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* row_of,
                                          void* x_perm, moe_stream_t stream) {
  using namespace moe;
  moe_status st = check_config(cfg);  // the same statuses as moe_permute; allocates nothing
  if (st != MOE_OK) return st;
  const int64_t n = cfg->T * cfg->top_k;
  const int64_t need = (int64_t)cfg->n_experts * permute_n_chunks(n);
  if (need > kNoAllocScratchInts) return MOE_ERR_UNSUPPORTED;
  if (!counts || !offsets || !aligned16(counts) || !aligned16(offsets)) return MOE_ERR_INVALID_ARG;
  if (cfg->T > 0 && (!topk_ids || !perm || !row_of || !x || !x_perm || !aligned16(topk_ids) || !aligned16(perm) ||
                     !aligned16(row_of) || !aligned16(x) || !aligned16(x_perm)))
    return MOE_ERR_INVALID_ARG;
  if (launch_failure_injected()) return MOE_ERR_CUDA;
  // run on the device that owns the outputs; the caller's current device is
  // restored when the guard goes out of scope
  DeviceGuard g;
  if ((st = g.bind(counts)) != MOE_OK) return st;
  if ((st = g.check_stream(stream)) != MOE_OK) return st;
  int32_t* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
  // The histogram pass writes every (expert, chunk) entry this call later
  // reads, so nothing left by an earlier call needs clearing.
  const int64_t cap = moe_expert_capacity(cfg);
  PermuteArgs a{topk_ids, x, counts, offsets, perm, row_of, x_perm, scratch, n, cfg->top_k, cfg->d_model,
                cfg->n_experts, cfg->dtype == MOE_BF16 ? 2 : 4, nullptr, cap};
  return launch_permute(a, stream) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
