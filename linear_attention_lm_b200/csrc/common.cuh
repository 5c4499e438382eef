// common.cuh -- shared device helpers for the Based attention kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "based.h"

namespace based {

// q/k feature dimension and the Taylor feature count 1 + d + d*d.
constexpr int kD = 16;
constexpr int kF = 1 + kD + kD * kD;  // 273
// phi scales for d = 16: d^(-1/4) = 1/2 and 1/(sqrt(2) sqrt(d)) = 1/(4 sqrt 2).
constexpr float kLinScale = 0.5f;
constexpr float kQuadScale = 0.17677669529663687f;

// Device status word: kernels that give up on a bounded wait record the first
// error here (atomicCAS from BASED_OK); the host reads and clears it.
__device__ int g_device_status = BASED_OK;

__device__ __forceinline__ void record_device_error(int code) {
  atomicCAS(&g_device_status, (int)BASED_OK, code);
}

// Test hook (based_debug_stall): which input load the first CTA of a kernel
// leaves out, so that the wait for it runs out; 0 = none.
constexpr int kStallNone = 0;
constexpr int kStallLinattnV = 1;  // linear-attention prefill: the V tile of its second chunk
constexpr int kStallWindowV = 2;   // window attention: its V tile
__device__ int g_stall_test = kStallNone;

__device__ __forceinline__ bool stall_test(int which) {
  return blockIdx.x == 0 && *const_cast<const volatile int*>(&g_stall_test) == which;
}

// One Taylor feature of a 16-vector held in shared memory or registers.
__device__ __forceinline__ float phi_feature(const float* x, int f) {
  if (f == 0) return 1.0f;
  if (f <= kD) return x[f - 1] * kLinScale;
  const int i = (f - kD - 1) >> 4, j = (f - kD - 1) & 15;
  return x[i] * x[j] * kQuadScale;
}

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// 2^x by the hardware approximation (PTX ex2.approx.ftz.f32: one special-function
// instruction, relative error about 2^-22, subnormal results flushed to zero).
// Used for softmax weights, which are rounded to bf16 right after.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace based
