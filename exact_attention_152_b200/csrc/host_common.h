// Host-side helpers shared by the forward and backward translation units of
// libattn: error text, device capability check, pointer checks, and the
// status word of the backward kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <string>

#include "attn.h"

namespace eab {

// Text of the last ATTN_ERR_CUDA on this thread (attn_last_error).
inline thread_local std::string t_last_error;

inline int cuda_fail(cudaError_t e, const char* what) {
  t_last_error = std::string(what) + ": " + cudaGetErrorString(e);
  return ATTN_ERR_CUDA;
}

constexpr int kMaxDeviceCount = 64;

// ATTN_OK when the current device is compute capability 10.0 (B200), probed
// once per device.
inline int check_device() {
  struct DeviceInfo {
    bool probed = false;
    bool supported = false;
  };
  static std::mutex mu;
  static DeviceInfo info[kMaxDeviceCount];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDeviceCount) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(mu);
  DeviceInfo& di = info[dev];
  if (!di.probed) {
    int major = 0, minor = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    di.supported = (major == 10 && minor == 0);
    di.probed = true;
  }
  return di.supported ? ATTN_OK : ATTN_ERR_UNSUPPORTED;
}

// Unique ID of the calling thread's current CUDA context (false if none or
// if the driver cannot tell).  A module-scope __device__ variable's address
// belongs to the copy of the module loaded into one context, so an address
// looked up once stays valid only while this ID is unchanged.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

inline bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}


inline bool ranges_overlap(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

inline bool misaligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) != 0;
}

// Status-word bits reported by attn_status_sync: a pipeline wait ran out
// (ATTN_ERR_TIMEOUT), bad packed-sequence offsets (ATTN_ERR_INVALID_ARG), a
// kernel that could not run as launched (ATTN_ERR_CUDA, text in t_last_error).
constexpr unsigned int kStatusWordTimeout = 1u;
constexpr unsigned int kStatusWordBadSeqlens = 2u;
constexpr unsigned int kStatusWordLaunch = 8u;

// Reads and clears the backward kernels' per-device status word (after the
// caller synchronised `stream`); defined with those kernels.
int bwd_status_take(cudaStream_t stream, unsigned int* status);

}  // namespace eab
