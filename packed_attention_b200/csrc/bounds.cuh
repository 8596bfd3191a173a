// The device-side error word and the range checks of the checked build.
//
// Kernels record a fault they detect in g_device_error (first fault wins;
// mf_get_device_error reads and clears it). Built with -DMF_CHECKED
// (libmfattn_checked.so), every global-memory index the kernels compute is
// compared with the extent of its buffer before the access: an index outside
// records MF_ERR_BOUNDS and the access is skipped, so a wrong index shows up
// as a status instead of a fault or a silent overwrite. The product build
// compiles the checks away.
#pragma once

#include <cstddef>
#include <cstdint>

#include "../../include/mf_attn.h"

namespace mf {

__device__ int32_t g_device_error;

__device__ __forceinline__ void record_error(mf_status s) {
  atomicCAS(&g_device_error, 0, static_cast<int32_t>(s));
}

#ifdef MF_CHECKED
constexpr bool kChecked = true;

// 0 <= i < n, else MF_ERR_BOUNDS is recorded.
__device__ __forceinline__ bool in_bounds(long long i, long long n) {
  if (i >= 0 && i < n) return true;
  record_error(MF_ERR_BOUNDS);
  return false;
}

// [p, p + bytes) inside [base, base + size), else MF_ERR_BOUNDS is recorded.
__device__ __forceinline__ bool in_span(const void* p, size_t bytes, const void* base,
                                        size_t size) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(p), b = reinterpret_cast<uintptr_t>(base);
  if (a >= b && a + bytes <= b + size) return true;
  record_error(MF_ERR_BOUNDS);
  return false;
}
#else
constexpr bool kChecked = false;

__device__ __forceinline__ constexpr bool in_bounds(long long, long long) { return true; }
__device__ __forceinline__ constexpr bool in_span(const void*, size_t, const void*, size_t) {
  return true;
}
#endif

}  // namespace mf
