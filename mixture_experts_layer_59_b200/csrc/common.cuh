// Shared device/host helpers of the MoE library (no torch types anywhere).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <string>

#include "../../include/moe.h"

namespace moe {

// ---------------------------------------------------------------- host errors
void set_error(const std::string& msg);
int fail(int code, const std::string& msg);
int cuda_fail(cudaError_t e, const char* what);

#define MOE_CHECK_LAUNCH(what)                                  \
  do {                                                          \
    cudaError_t _e = cudaGetLastError();                        \
    if (_e != cudaSuccess) return ::moe::cuda_fail(_e, what);   \
  } while (0)

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Measurement hook: while profiling is enabled (moe_profile_enable), every
// kernel launch of the library is bracketed by CUDA events on its stream.
struct ProfScope {
  const char* name;
  cudaStream_t stream;
  cudaEvent_t start = nullptr;
  ProfScope(const char* n, cudaStream_t s);
  ~ProfScope();
};

// Bump allocator over a caller workspace.
struct Carve {
  char* base;
  size_t cap;
  size_t used = 0;
  bool ok = true;
  Carve(void* p, size_t n) : base(static_cast<char*>(p)), cap(n) {}
  template <class T>
  T* take(size_t count) {
    size_t off = align_up(used, 256);
    size_t bytes = align_up(count * sizeof(T), 256);
    if (base == nullptr || off + bytes > cap) { ok = false; used = off + bytes; return nullptr; }
    used = off + bytes;
    return reinterpret_cast<T*>(base + off);
  }
};

// Bytes a Carve sequence needs (same arithmetic, no pointer).
struct Sizer {
  size_t used = 0;
  template <class T>
  T* take(size_t count) {
    used = align_up(used, 256) + align_up(count * sizeof(T), 256);
    return nullptr;
  }
};

// ---------------------------------------------------------------- device status
// Device address of the library's status word (one per device).  Kernels
// whose bounded waits expire, or that meet an invalid index, record a code
// there; moe_check_status() reads and clears it.
int* status_ptr();

__device__ __forceinline__ void record_status(int* st, int code) {
  if (st) atomicCAS(st, 0, code);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- numerics
__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }

template <class T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// Round an fp32 value to bf16 and back (the value a bf16 tensor would hold).
__device__ __forceinline__ float bf16_round(float v) {
  return __bfloat162float(__float2bfloat16_rn(v));
}

// silu(z) = z * sigmoid(z); silu'(z) = sigmoid(z) * (1 + z * (1 - sigmoid(z))).
__device__ __forceinline__ float sigmoid_f(float z) { return 1.0f / (1.0f + expf(-z)); }
__device__ __forceinline__ float silu_f(float z) { return z * sigmoid_f(z); }
__device__ __forceinline__ float silu_grad_f(float z) {
  float s = sigmoid_f(z);
  return s * (1.0f + z * (1.0f - s));
}

// Expert owning row r: the segment [offsets[e], offsets[e+1]) containing r.
__device__ __forceinline__ int row_expert(const int32_t* offsets, int E, int r) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (offsets[mid] <= r) lo = mid; else hi = mid - 1;
  }
  return lo;
}

}  // namespace moe
