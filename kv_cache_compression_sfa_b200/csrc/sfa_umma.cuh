// sfa_umma.cuh — 5th-generation tensor core (tcgen05) helpers for sm_100a:
// tensor-memory allocation, shared-memory matrix descriptors, bf16 MMAs with
// fp32 accumulation in tensor memory, commits to mbarriers and loads of
// accumulator rows.
//
// Operand layout used throughout (no swizzle): a matrix is stored as "core
// matrices" of 8 rows x 16 bytes (8 bf16), 128 contiguous bytes each, rows
// 16 bytes apart.  For a [64 rows x 64 columns] bf16 block the core matrix
// holding rows 8*rg.., columns 8*cg.. sits at byte (cg*8 + rg)*128, so that
//   * as a K-major operand (rows = M or N, columns = K): the next row group
//     is 128 bytes on (stride offset) and the next K group 1024 bytes on
//     (leading offset);
//   * as an MN-major operand (rows = K, columns = M or N): the next MN group
//     is 1024 bytes on (stride offset) and the next K group 128 bytes on
//     (leading offset).
// One stored block can therefore feed both a K-major and an MN-major MMA.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "sfa_common.cuh"

namespace sfa {

constexpr int kBlk = 64;                       // rows/columns of a staged block
constexpr int kBlkBytes = kBlk * kBlk * 2;     // one bf16 block (8 KB)
constexpr int kCoreBytes = 128;

// Byte offset of element (row, col) inside a [64 x 64] bf16 block.
__host__ __device__ __forceinline__ int blk_off(int row, int col) {
  return ((col >> 3) * 8 + (row >> 3)) * kCoreBytes + (row & 7) * 16 + (col & 7) * 2;
}

// Shared-memory matrix descriptor (no swizzle): start address, leading and
// stride byte offsets (all in 16-byte units), descriptor version 1.
__device__ __forceinline__ uint64_t umma_desc(const void* smem, unsigned lbo, unsigned sbo) {
  const unsigned a = smem_u32(smem);
  uint64_t d = static_cast<uint64_t>((a >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  return d;
}

// Instruction descriptor of kind::f16: bf16 A and B, fp32 accumulator,
// A K-major, B K-major or MN-major, shape M x N.
__host__ __device__ __forceinline__ uint32_t umma_idesc_bf16(int M, int N, bool b_mn_major) {
  uint32_t d = 0;
  d |= 1u << 4;   // accumulator fp32
  d |= 1u << 7;   // A bf16
  d |= 1u << 10;  // B bf16
  d |= (b_mn_major ? 1u : 0u) << 16;
  d |= static_cast<uint32_t>(N >> 3) << 17;
  d |= static_cast<uint32_t>(M >> 4) << 24;
  return d;
}

// The same with either operand MN-major (A: bit 15, B: bit 16).
__host__ __device__ __forceinline__ uint32_t umma_idesc_bf16_ab(int M, int N, bool a_mn_major, bool b_mn_major) {
  return umma_idesc_bf16(M, N, b_mn_major) | ((a_mn_major ? 1u : 0u) << 15);
}

// Byte offset of element (row, col) inside a [16 x 64] bf16 block in the
// core-matrix layout (core matrix of rows 8*rg.., columns 8*cg.. at byte
// (cg*2 + rg)*128): as a K-major operand the next row group is 128 bytes
// on and the next K group 256 bytes on.
__host__ __device__ __forceinline__ int blk16_off(int row, int col) {
  return ((col >> 3) * 2 + (row >> 3)) * kCoreBytes + (row & 7) * 16 + (col & 7) * 2;
}
constexpr int kBlk16Bytes = 16 * kBlk * 2;  // one [16 x 64] bf16 block (2 KB)

// D[tmem] (+)= A[smem] * B[smem]; issued by one thread.
__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                          bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(static_cast<uint32_t>(accumulate))
      : "memory");
}

// Arrives once on `bar` when every tcgen05 operation this thread issued so
// far has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Tensor-memory allocation by one whole warp; the base address lands in
// *dst (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// 32 consecutive 32-bit columns of this thread's lane (warp w reads lanes
// 32*(w%4) .. +31; the lane offset is part of taddr).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 16 consecutive 32-bit columns of this thread's lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// 2 consecutive 32-bit columns of this thread's lane.
__device__ __forceinline__ void tmem_ld2(uint32_t taddr, float (&v)[2]) {
  uint32_t r0, r1;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  v[0] = __uint_as_float(r0);
  v[1] = __uint_as_float(r1);
}

// Splits x into bf16 hi = round(x) and lo = round(x - hi): hi + lo carries
// about 16 significant bits of x.
__device__ __forceinline__ void split_bf16(float x, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

// Writes a [64 x 64] fp32 tile (row stride `ld` floats) as hi and lo bf16
// blocks in the core-matrix layout; all threads of the block cooperate.
__device__ __forceinline__ void stage_split_block(const float* src, int ld, unsigned char* hi_blk,
                                                  unsigned char* lo_blk, int tid, int nthreads) {
  for (int i = tid; i < kBlk * kBlk / 4; i += nthreads) {
    const int row = i / (kBlk / 4), c4 = (i % (kBlk / 4)) * 4;
    const float4 v = *reinterpret_cast<const float4*>(src + row * ld + c4);
    __nv_bfloat16 h[4], l[4];
    split_bf16(v.x, h[0], l[0]);
    split_bf16(v.y, h[1], l[1]);
    split_bf16(v.z, h[2], l[2]);
    split_bf16(v.w, h[3], l[3]);
    const int off = blk_off(row, c4);  // 4 consecutive columns: 8 contiguous bytes
    *reinterpret_cast<uint2*>(hi_blk + off) = *reinterpret_cast<const uint2*>(h);
    *reinterpret_cast<uint2*>(lo_blk + off) = *reinterpret_cast<const uint2*>(l);
  }
}

}  // namespace sfa
