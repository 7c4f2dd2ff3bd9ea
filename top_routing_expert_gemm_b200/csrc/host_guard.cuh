// Host-side helpers shared by the C-ABI entry points: the configuration check,
// the scoped switch to the device that owns a call's buffers, and the
// launch-failure injection hook used by the failure tests.
#pragma once

#include <cuda_runtime.h>

#include <cstdlib>
#include <cstring>

#include "../../include/moe.h"

namespace moe {

// Shapes, enums and the build's limits (moe_api.cu).
moe_status check_config(const moe_config* c);

// Makes the device that owns a call's buffers current for the duration of
// the call and puts the caller's current device back when it goes out of
// scope, so an entry point never leaves the calling thread on another device.
class DeviceGuard {
 public:
  DeviceGuard() = default;
  DeviceGuard(const DeviceGuard&) = delete;
  DeviceGuard& operator=(const DeviceGuard&) = delete;
  ~DeviceGuard() {
    if (prev_ >= 0) cudaSetDevice(prev_);
  }

  // Switch to the device of `p` (device or managed memory; anything else is
  // MOE_ERR_INVALID_ARG).  The first switch remembers the device to restore.
  moe_status bind(const void* p) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
      const cudaError_t e = cudaGetLastError();
      return e == cudaErrorInvalidValue ? MOE_ERR_INVALID_ARG : MOE_ERR_CUDA;
    }
    if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged) return MOE_ERR_INVALID_ARG;
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return MOE_ERR_CUDA;
    if (cur != at.device) {
      if (cudaSetDevice(at.device) != cudaSuccess) return MOE_ERR_CUDA;
      if (prev_ < 0) prev_ = cur;
    }
    device_ = at.device;
    return MOE_OK;
  }

  // `p` must live on the device bound before (MOE_ERR_INVALID_ARG otherwise).
  moe_status same_device(const void* p) const {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
      cudaGetLastError();
      return MOE_ERR_INVALID_ARG;
    }
    if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged) return MOE_ERR_INVALID_ARG;
    return at.device == device_ ? MOE_OK : MOE_ERR_INVALID_ARG;
  }

  // A stream created on another device than the bound one cannot run this
  // call's kernels: MOE_ERR_INVALID_ARG.  The legacy and per-thread default
  // streams (and NULL) belong to whichever device is current.
  moe_status check_stream(cudaStream_t s) const {
    if (s == nullptr || s == cudaStreamLegacy || s == cudaStreamPerThread) return MOE_OK;
    int sd = -1;
    if (cudaStreamGetDevice(s, &sd) != cudaSuccess) {
      cudaGetLastError();
      return MOE_ERR_INVALID_ARG;
    }
    return sd == device_ ? MOE_OK : MOE_ERR_INVALID_ARG;
  }

 private:
  int prev_ = -1;
  int device_ = -1;
};

// Launch-failure injection for failure tests: with the environment variable
// MOE_FAULT set to "launch", every entry point that would launch work returns
// MOE_ERR_CUDA after its host-side argument checks and before any CUDA call.
// Nothing is injected on the device.
inline bool launch_failure_injected() {
  const char* v = std::getenv("MOE_FAULT");
  return v != nullptr && std::strcmp(v, "launch") == 0;
}

}  // namespace moe
