// common.cuh -- shared definitions of libvit's kernels and host code.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace vit {

// Upper bound of any single bounded wait inside a kernel (mbarrier phase,
// peer flag).  Every kernel of this library finishes in milliseconds; a wait
// this long means a lost arrival, and the kernel records VIT_ERR_TIMEOUT in
// the device status word and winds down instead of spinning.
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;  // 2 s

// Device status word values (mirror vit_status codes).
constexpr int kDevOk = 0;
constexpr int kDevTimeout = 6;
constexpr int kDevBounds = 7;

// Programmatic dependent launch: a kernel launched with launch_pdl() may
// start while the previous kernel of its stream is still running.  It calls
// pdl_trigger() at entry (its own dependents may then be scheduled; a grid is
// only launched once every CTA of its predecessor has started, so this cannot
// starve the running grid of SMs) and pdl_wait() before its first access to
// global memory, which returns once the previous grid has completed and its
// writes are visible.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void report_status(int *status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// ---------------------------------------------------------------- element io
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// Two fp32 -> packed bf16x2 (low half = first argument), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// GELU, tanh form: 0.5 u (1 + tanh(sqrt(2/pi) (u + 0.044715 u^3))).
__device__ __forceinline__ float gelu_tanh_f32(float u) {
  const float k0 = 0.7978845608028654f;  // sqrt(2/pi)
  const float k1 = 0.044715f;
  float t = tanhf(k0 * (u + k1 * u * u * u));
  return 0.5f * u * (1.0f + t);
}

}  // namespace vit
