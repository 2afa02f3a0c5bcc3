// Shared host/device helpers of libcca (sm_100a only).
#pragma once

#include <cuda_runtime.h>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <string>

#include "../../include/cca.h"

namespace cca {

// ------------------------------------------------------------------ host side
// Per-thread last error message and launch counter (see cca_last_error and
// cca_take_launch_count in cca.h).
std::string &last_error();
int64_t &launch_counter();

inline cca_status fail(cca_status st, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  last_error() = buf;
  return st;
}

// Check the launch that was just issued; count it on success.
inline cca_status launched(const char *what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    return fail(CCA_ERR_CUDA, "%s: launch failed: %s", what, cudaGetErrorString(e));
  }
  ++launch_counter();
  return CCA_OK;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int num_sms();  // SM count of the current device (cached per device)

#define CCA_TRY(expr)                 \
  do {                                \
    cca_status _st = (expr);          \
    if (_st != CCA_OK) return _st;    \
  } while (0)

// ------------------------------------------------------------------ device side
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

}  // namespace cca
