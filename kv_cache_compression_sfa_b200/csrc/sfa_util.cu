// sfa_util.cu — set-up kernels: semantic-slot norms and the state header.
#include <cuda_runtime.h>

#include "sfa_common.cuh"

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

__global__ void write_header_kernel(unsigned char* state, StateHeader h) {
  if (threadIdx.x == 0 && blockIdx.x == 0) *reinterpret_cast<StateHeader*>(state) = h;
}

}  // namespace

cudaError_t launch_slot_norms(const float* slots, float* norms, int L, int H, cudaStream_t s) {
  slot_norm_kernel<<<L * kSlots, 256, 0, s>>>(slots, norms, H);
  return cudaGetLastError();
}

cudaError_t launch_write_header(unsigned char* state, StateHeader h, cudaStream_t s) {
  write_header_kernel<<<1, 32, 0, s>>>(state, h);
  return cudaGetLastError();
}

}  // namespace sfa
