// Shared device helpers of the sm_100a MoE kernels: numeric conversions,
// vector loads, the device status word and bounded waits.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// status word values written by kernels (mirrors moe_status in include/moe.h)
constexpr int kDevTimeout = 5;
constexpr int kDevBadExpertId = 6;

constexpr int kMaxExperts = 1024;
constexpr int kMaxTopK = 16;

// ---------------------------------------------------------------- element types
template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f(float v) { return v; }
  static __device__ __forceinline__ float from_f(float v) { return v; }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

// 16-byte vector of elements of T (8 bf16 or 4 fp32)
template <typename T> struct Vec16 {
  static constexpr int N = 16 / sizeof(T);
  T v[N];
};

template <typename T>
__device__ __forceinline__ Vec16<T> ld16(const T* p) {
  Vec16<T> r;
  *reinterpret_cast<uint4*>(r.v) = __ldg(reinterpret_cast<const uint4*>(p));
  return r;
}
template <typename T>
__device__ __forceinline__ void st16(T* p, const Vec16<T>& r) {
  *reinterpret_cast<uint4*>(p) = *reinterpret_cast<const uint4*>(r.v);
}

// One 32-byte store (eight 32-bit words) to a 32-byte-aligned global address:
// a whole L2 sector per instruction
__device__ __forceinline__ void st_global_32B(void* p, const uint32_t* w) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]),
               "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// SiLU(z) = z / (1 + e^-z), written with the CUDA math library's expf
__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + expf(-z)); }
// GELU(z) = z * Phi(z) = z/2 * (1 + erf(z / sqrt 2)), with the CUDA math library's erff
__device__ __forceinline__ float gelu_f(float z) { return 0.5f * z * (1.0f + erff(z * 0.70710678118654752f)); }

// expert activations (moe_expert_act) and the epilogue of the second GEMM
constexpr int kEpiSwiGLU = 0, kEpiGELU = 1, kEpiNone = 2;

// A timed-out wait overrides any other code (later kernels of the same call
// may then read unfinished outputs and report those too); any other code
// only fills an empty word, so the first failure is the one reported.
__device__ __forceinline__ void set_status(int* status, int code) {
  if (status == nullptr) return;
  if (code == kDevTimeout) atomicExch(status, code);
  else atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- top-k helpers
// Keep the KMAX largest keys seen so far, sorted descending.  A new key only
// displaces strictly smaller ones, so among equal keys the earlier (lower
// expert index, when fed in ascending index order) stays ahead.
template <int KMAX>
struct TopK {
  float key[KMAX];
  int idx[KMAX];
  float val[KMAX];  // payload carried with each key (the raw logit)
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int j = 0; j < KMAX; ++j) { key[j] = -INFINITY; idx[j] = 0x7fffffff; val[j] = 0.f; }
  }
  __device__ __forceinline__ void push(float k, int i, float v = 0.f) {
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      const bool sw = k > key[j] || (k == key[j] && i < idx[j]);
      const float tk = key[j], tv = val[j];
      const int ti = idx[j];
      key[j] = sw ? k : tk;
      idx[j] = sw ? i : ti;
      val[j] = sw ? v : tv;
      k = sw ? tk : k;
      i = sw ? ti : i;
      v = sw ? tv : v;
    }
  }
};

// (key desc, index asc) ordering: true when (ka, ia) ranks before (kb, ib)
__device__ __forceinline__ bool ranks_before(float ka, int ia, float kb, int ib) {
  return ka > kb || (ka == kb && ia < ib);
}

}  // namespace moe

#define MOE_CUDA_TRY(expr)                                  \
  do {                                                      \
    cudaError_t _e = (expr);                                \
    if (_e != cudaSuccess) return MOE_ERR_CUDA;             \
  } while (0)
