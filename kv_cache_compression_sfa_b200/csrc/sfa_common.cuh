// sfa_common.cuh — device helpers shared by the SFA kernels: vector loads of
// the input dtype, warp reductions, the error latch, mbarriers, bulk and
// asynchronous copies, and programmatic dependent launch.
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

// Maximum over the full warp in one instruction (sm_100a float redux);
// every lane must take part.
__device__ __forceinline__ float warp_max_redux(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// First error wins; later errors are dropped until the host clears the word.
__device__ __forceinline__ void latch_error(int* err, int code) { atomicCAS(err, 0, code); }

// One exponential-moving-average step, s <- g*s + (1-g)*e.  Used for the
// far-field EWMA [P1 §2.1 eq. S_t] and the EMA field [P3 §2.1 channel 2]; one
// definition so every site rounds the same way.
__device__ __forceinline__ float ewma(float g, float s, float e) {
  return fmaf(g, s, (1.0f - g) * e);
}

// Result element i of the enhancement alpha_layer * u for attention output
// x, in the output mode [P3 §2.2]: fp32 or bf16 x + enhancement, or the
// enhancement added to the caller's attention output already in res.  The
// fp32 mode rounds once: fmaf(alpha_layer, u, x).
__device__ __forceinline__ void store_result(int mode, void* res, long long i, float a_l, float u, float x) {
  if (mode == SFA_OUT_F32) {
    static_cast<float*>(res)[i] = fmaf(a_l, u, x);
  } else if (mode == SFA_OUT_BF16) {
    static_cast<__nv_bfloat16*>(res)[i] = __float2bfloat16_rn(fmaf(a_l, u, x));
  } else if (mode == SFA_OUT_ADD_F32) {
    float* r = static_cast<float*>(res) + i;
    *r = fmaf(a_l, u, *r);
  } else {
    __nv_bfloat16* r = static_cast<__nv_bfloat16*>(res) + i;
    *r = __float2bfloat16_rn(fmaf(a_l, u, __bfloat162float(*r)));
  }
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

// Loads one 16-byte vector of the input dtype and widens it: 4 floats or 8
// bf16 values.
template <typename T>
struct Load16;
template <>
struct Load16<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void run(const float* p, float* o) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
  }
};
template <>
struct Load16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void run(const __nv_bfloat16* p, float* o) {
    const uint4 raw = *reinterpret_cast<const uint4*>(p);
    const unsigned w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
      o[2 * i] = f.x;
      o[2 * i + 1] = f.y;
    }
  }
};

template <>
struct VecLoad<float, 8> {
  __device__ __forceinline__ static void run(const float* p, float* o) {
    VecLoad<float, 4>::run(p, o);
    VecLoad<float, 4>::run(p + 4, o + 4);
  }
};
template <>
struct VecLoad<__nv_bfloat16, 8> {
  __device__ __forceinline__ static void run(const __nv_bfloat16* p, float* o) {
    Load16<__nv_bfloat16>::run(p, o);
  }
};

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// ---- shared-memory addresses, mbarriers and 1-D bulk copies (TMA engine) --

__device__ __forceinline__ unsigned smem_u32(const void* p) {
  return static_cast<unsigned>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

// Makes barrier initialisation visible to the async (bulk-copy) proxy.
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Barrier `id` (1..15) among `count` threads (whole warps) of the CTA.
__device__ __forceinline__ void named_bar_sync(unsigned id, unsigned count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Waits for phase `parity` of a barrier, at most `limit` polls.  Returns
// false (and latches SFA_ERR_DEVICE_TIMEOUT) if the wait ran out.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, unsigned parity, unsigned limit,
                                                  int* err) {
  for (unsigned i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  latch_error(err, SFA_ERR_DEVICE_TIMEOUT);
  return false;
}

// Contiguous global -> shared copy by the bulk-copy engine; completion is
// counted in bytes on `bar`.  Both addresses 16-byte aligned, bytes a
// multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// 16-byte global -> shared copy that bypasses the registers (and L1);
// completion is tracked per thread by commit groups.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Waits until at most N of this thread's commit groups are still in flight.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// 3-D tiled bulk tensor load (no multicast) of the box at coordinates
// (x, y, z) of `map` into shared memory, completion counted in bytes on
// `bar`.  x times the element size must be a multiple of 16 bytes; other
// coordinates may lie outside the tensor (those elements read as zero).
__device__ __forceinline__ void tma_load_3d(void* dst, const void* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::
          "r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

// 4-D tiled bulk tensor load (no multicast), as tma_load_3d.
__device__ __forceinline__ void tma_load_4d(void* dst, const void* map, int x, int y, int z, int w,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], [%6];" ::
          "r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w),
          "r"(smem_u32(bar))
      : "memory");
}

// Plain arrive (count 1, no transaction bytes) on a barrier of this CTA.
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Orders this thread's earlier generic-proxy shared-memory accesses before
// later bulk copies (async proxy) into the same bytes.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Split cluster barrier: arrive (release) once this CTA is done reading its
// peers' shared memory, wait (acquire) before leaving.
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// The same for shared memory of other CTAs of the cluster written through
// distributed shared memory.
__device__ __forceinline__ void fence_proxy_async_cluster() {
  asm volatile("fence.proxy.async.shared::cluster;" ::: "memory");
}

// ---- programmatic dependent launch ----------------------------------------
// Everything a kernel reads that an earlier kernel of the stream may write
// must come after pdl_wait(); pdl_trigger() lets the next kernel's CTAs be
// scheduled early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

constexpr unsigned kMbarPollLimit = 1u << 24;

}  // namespace sfa
