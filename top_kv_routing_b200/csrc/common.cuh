// Shared host/device helpers of the MSA hot-path libraries (not part of the ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>

#include "msa_common.h"

// Each library defines its own thread-local last-error buffer and accessor.
#define MSA_DEFINE_LAST_ERROR(accessor)                                              \
  static thread_local char g_msa_last_error[512] = "";                               \
  extern "C" const char* accessor(void) { return g_msa_last_error; }                 \
  static msa_status msa_fail(msa_status st, const char* fmt, ...) {                  \
    va_list ap;                                                                      \
    va_start(ap, fmt);                                                               \
    vsnprintf(g_msa_last_error, sizeof(g_msa_last_error), fmt, ap);                  \
    va_end(ap);                                                                      \
    return st;                                                                       \
  }                                                                                  \
  static msa_status msa_ok() {                                                       \
    g_msa_last_error[0] = 0;                                                         \
    return MSA_OK;                                                                   \
  }

#define MSA_CUDA_TRY(expr)                                                                 \
  do {                                                                                     \
    cudaError_t e_ = (expr);                                                               \
    if (e_ != cudaSuccess) return msa_fail(MSA_ERR_CUDA, "%s: %s", #expr, cudaGetErrorString(e_)); \
  } while (0)

namespace msa {

// Returns 1 when the current device is sm_100 (B200), 0 when it is another device and
// -1 when no device can be queried.  Cached per device ordinal.
inline int current_device_is_sm100(int* dev_out) {
  static int cache[64];  // 0 unknown, 1 yes, 2 no
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (dev_out) *dev_out = dev;
  if (dev >= 0 && dev < 64 && cache[dev]) return cache[dev] == 1;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return -1;
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return -1;
  const int ok = (major == 10 && minor == 0) ? 1 : 2;
  if (dev >= 0 && dev < 64) cache[dev] = ok;
  return ok == 1;
}

inline int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

__device__ __forceinline__ void set_err(int32_t* dev_err, uint32_t bit) {
  if (dev_err) atomicOr(reinterpret_cast<unsigned int*>(dev_err), bit);
}

// bf16x2 (packed in a 32-bit word, low half = first element) -> two floats, exactly.
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

__device__ __forceinline__ uint32_t float2_to_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Largest d with off[d] <= x, for off non-decreasing with off[0] <= x < off[n].
__device__ __forceinline__ int upper_doc(const int64_t* __restrict__ off, int n, int64_t x) {
  int lo = 0, hi = n;  // invariant: off[lo] <= x < off[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(off + mid) <= x) lo = mid; else hi = mid;
  }
  return lo;
}

// cos/sin of pos * w for an fp64 angle, reduced to [-pi, pi] in fp64 and evaluated in fp64.
__device__ __forceinline__ void angle_sincos(double pos, double w, float* c, float* s) {
  const double two_pi = 6.283185307179586476925286766559;
  double a = pos * w;
  a = a - two_pi * rint(a / two_pi);
  double sd, cd;
  sincos(a, &sd, &cd);
  *c = (float)cd;
  *s = (float)sd;
}

}  // namespace msa
