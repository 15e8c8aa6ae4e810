// sfa_static_ws.cu — sfa_prefill_static_ws: a prefill entry point that
// allocates nothing.
//
// Some callers cannot hand the operator a workspace.  A custom-op hook inside
// another inference engine may receive only the operator's input and output
// tensors and no allocator, and a serving loop may forbid cudaMalloc in its
// steady state because an allocation can synchronise the device.  For them,
// the prefill's scratch (stream positions, the far state at the end of the
// call and the pool weights of every tile) lives in one file-scope device
// array of fixed size, held by every GPU that loads it until the process
// exits.  The caller still passes inputs, outputs and the state.  The CUDA
// runtime loads a module's device arrays lazily: the array is reserved on a
// device when its address is first looked up, which the first call on that
// device does (it may allocate and synchronise there, once), so that first
// call belongs before any stream capture.
//
// The work itself is exactly sfa_prefill's: this entry point only supplies
// the array's device address as the workspace.
#include <cuda_runtime.h>

#include <mutex>

#include "sfa_internal.h"

namespace {

// Scratch shared by every call on a device (16 MiB: one 512-token prefill of
// a 24-layer, hidden-896 model needs about 3 MB).
constexpr size_t kStaticWorkspaceBytes = SFA_STATIC_WORKSPACE_BYTES;
static __device__ __align__(256) unsigned char g_static_ws[kStaticWorkspaceBytes];

constexpr int kMaxDevices = 64;
std::mutex g_ws_mutex;
void* g_ws_ptr[kMaxDevices] = {};

// Device address of the array on the current device.  The array's name is
// only a host-side stand-in, so the address is looked up once per device,
// with that device current, and cached.
int static_ws_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SFA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_ws_mutex);
  if (g_ws_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_ws) != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return SFA_ERR_CUDA;
    }
    g_ws_ptr[dev] = ptr;
  }
  *out = g_ws_ptr[dev];
  return SFA_OK;
}

}  // namespace

extern "C" {

int sfa_prefill_static_ws(const sfa_handle* h, const void* q, const void* k, const void* v,
                          long long n, int batch, void* state, void* out, void* stream) {
  // the same argument checks, in the same order, as sfa_prefill
  if (n < 0 || batch <= 0 || sfa_prefill_workspace_bytes(h, 1, 1) == 0) return SFA_ERR_INVALID_ARG;
  if (n == 0) return SFA_OK;
  const size_t need = sfa_prefill_workspace_bytes(h, batch, n);
  // 0: a bad handle or a call beyond sfa_prefill's limits; sfa_prefill
  // returns that status without launching anything.
  if (need == 0) return sfa_prefill(h, q, k, v, n, batch, state, out, nullptr, 0, stream);
  if (need > kStaticWorkspaceBytes) return SFA_ERR_WORKSPACE;  // call exceeds the fixed scratch
  void* ws = nullptr;
  const int rc = static_ws_address(&ws);
  if (rc != SFA_OK) return rc;
  // Nothing in the workspace has to start at zero.
  return sfa_prefill(h, q, k, v, n, batch, state, out, ws, kStaticWorkspaceBytes, stream);
}

}  // extern "C"
