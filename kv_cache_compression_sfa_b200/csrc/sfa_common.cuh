// sfa_common.cuh — device helpers shared by the SFA kernels: vector loads of
// the input dtype, warp reductions, the error latch and the acquire/release
// flag accesses of the prefill look-back.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "sfa_internal.h"

namespace sfa {

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

// First error wins; later errors are dropped until the host clears the word.
__device__ __forceinline__ void latch_error(int* err, int code) { atomicCAS(err, 0, code); }

// One exponential-moving-average step, s <- g*s + (1-g)*e.  Used for the
// far-field EWMA [P1 §2.1 eq. S_t] and the EMA field [P3 §2.1 channel 2]; one
// definition so every site rounds the same way.
__device__ __forceinline__ float ewma(float g, float s, float e) {
  return fmaf(g, s, (1.0f - g) * e);
}

// Loads N consecutive elements of the input dtype and widens them to fp32.
template <typename T, int N>
struct VecLoad;

template <>
struct VecLoad<float, 2> {
  __device__ __forceinline__ static void run(const float* p, float* o) {
    const float2 v = *reinterpret_cast<const float2*>(p);
    o[0] = v.x; o[1] = v.y;
  }
};
template <>
struct VecLoad<float, 4> {
  __device__ __forceinline__ static void run(const float* p, float* o) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
  }
};
template <>
struct VecLoad<__nv_bfloat16, 2> {
  __device__ __forceinline__ static void run(const __nv_bfloat16* p, float* o) {
    const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(p);
    const float2 f = __bfloat1622float2(v);
    o[0] = f.x; o[1] = f.y;
  }
};
template <>
struct VecLoad<__nv_bfloat16, 4> {
  __device__ __forceinline__ static void run(const __nv_bfloat16* p, float* o) {
    const uint2 raw = *reinterpret_cast<const uint2*>(p);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
    const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    o[0] = fa.x; o[1] = fa.y; o[2] = fb.x; o[3] = fb.y;
  }
};

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// gpu-scope acquire load / release store of a 32-bit look-back flag.
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_u32(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Polls a flag until it is non-empty, at most `limit` times.  A wait that
// runs out latches SFA_ERR_DEVICE_TIMEOUT and reports kFlagIncl so that the
// caller finishes its work (with invalid data) instead of hanging.
__device__ __forceinline__ unsigned wait_flag(const unsigned* f, unsigned limit, int* err) {
  unsigned v = ld_acquire_u32(f);
  unsigned polls = 0;
  while (v == kFlagEmpty) {
    if (++polls > limit) {
      latch_error(err, SFA_ERR_DEVICE_TIMEOUT);
      return kFlagIncl;
    }
    __nanosleep(128);
    v = ld_acquire_u32(f);
  }
  return v;
}

}  // namespace sfa
