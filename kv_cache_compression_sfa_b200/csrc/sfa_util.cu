// sfa_util.cu — set-up kernels: semantic-slot norms and the state header.
#include <cuda_runtime.h>

#include "sfa_common.cuh"
#include "sfa_umma.cuh"

namespace sfa {
namespace {

// One block per (layer, slot): |slot_j| accumulated in double, clamped below
// at the cosine norm floor ([P3 §2.1 channel 3] cosine of x and slot_j).
__global__ void slot_norm_kernel(const float* slots, float* norms, int H) {
  const int row = blockIdx.x;
  const float* s = slots + static_cast<size_t>(row) * H;
  double acc = 0.0;
  for (int i = threadIdx.x; i < H; i += blockDim.x) acc += static_cast<double>(s[i]) * s[i];
  __shared__ double red[256];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) norms[row] = fmaxf(static_cast<float>(sqrt(red[0])), kNormFloor);
}

// Pre-split slot blocks for the prefill pool MMAs: for layer l and 64-column
// chunk c of hidden, a [64 slots x 64 columns] bf16 hi block followed by the
// lo block (slot = hi + lo to about 16 significant bits), both in the
// core-matrix layout of sfa_umma.cuh.  One thread per element.
__global__ void slot_image_kernel(const float* slots, unsigned char* img, int L, int H) {
  const long long n = static_cast<long long>(L) * kSlots * H;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int l = static_cast<int>(i / (static_cast<long long>(kSlots) * H));
    const int rem = static_cast<int>(i % (static_cast<long long>(kSlots) * H));
    const int j = rem / H, h = rem % H;
    const int c = h / kBlk, col = h % kBlk;
    unsigned char* blk = img + (static_cast<size_t>(l) * (H / kBlk) + c) * 2 * kBlkBytes;
    __nv_bfloat16 hi, lo;
    split_bf16(slots[i], hi, lo);
    *reinterpret_cast<__nv_bfloat16*>(blk + blk_off(j, col)) = hi;
    *reinterpret_cast<__nv_bfloat16*>(blk + kBlkBytes + blk_off(j, col)) = lo;
  }
}

__global__ void write_header_kernel(unsigned char* state, StateHeader h) {
  if (threadIdx.x == 0 && blockIdx.x == 0) *reinterpret_cast<StateHeader*>(state) = h;
}

}  // namespace

cudaError_t launch_slot_norms(const float* slots, float* norms, int L, int H, cudaStream_t s) {
  slot_norm_kernel<<<L * kSlots, 256, 0, s>>>(slots, norms, H);
  return cudaGetLastError();
}

cudaError_t launch_slot_image(const float* slots, unsigned char* img, int L, int H, cudaStream_t s) {
  slot_image_kernel<<<592, 256, 0, s>>>(slots, img, L, H);
  return cudaGetLastError();
}

cudaError_t launch_write_header(unsigned char* state, StateHeader h, cudaStream_t s) {
  write_header_kernel<<<1, 32, 0, s>>>(state, h);
  return cudaGetLastError();
}

}  // namespace sfa
