// Shared host/device helpers of libkdverify.so: error plumbing, argument checks,
// device attribute cache.  No arithmetic of the verify step lives here.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include "kd_verify.h"

namespace kd {

// Last CUDA error text, per host thread, for kd_strerror(KD_ELAUNCH).
void set_cuda_error(cudaError_t e, const char* where);

// KD_ELAUNCH when `e` is an error (recording its text), else KD_OK.
inline int cuda_status(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return KD_OK;
  set_cuda_error(e, where);
  return KD_ELAUNCH;
}

// Status of the launch just enqueued.
inline int launch_status(const char* where) { return cuda_status(cudaGetLastError(), where); }

// Checks that the current device is an sm_100 part and returns its SM count.
int device_sms(int* sms);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shapes every call shares.
inline bool shapes_ok(int B, int n) { return B >= 1 && n >= 1 && n <= KD_MAX_NODES; }

// Cache addressing: 16-byte aligned base, stride a multiple of 8 bf16, wide enough.
inline bool cache_ok(const void* c_kv, const void* k_rope, int64_t sc, int64_t sr, int64_t cap) {
  return c_kv && k_rope && aligned16(c_kv) && aligned16(k_rope) && sc >= KD_D_C && sr >= KD_D_R &&
         (sc % 8) == 0 && (sr % 8) == 0 && cap >= 1;
}

__device__ __forceinline__ void raise_dev_error(int32_t* word, int bits) {
  if (word) atomicOr(word, bits);
}

}  // namespace kd
