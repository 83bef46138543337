// Allocation-free form of archead_logits_lse_argmax.
//
// Some callers cannot call cudaMalloc at the point where they run the head:
// code recorded into a CUDA graph by a framework that forbids allocation
// during capture, allocators that must stay untouched in the middle of a
// serving step, or plug-ins whose host process owns all device memory.  They
// pass inputs and outputs as usual; the scratch space the forward pass needs
// (low-rank prologue output, per-block partials, ticket and status word) comes
// from a fixed array in the library's own device memory instead of a
// caller-provided workspace.
//
// The array is a file-scope __device__ variable of kStaticWorkspaceBytes, so
// every GPU that loads this library holds it until the process exits.  Host
// code cannot use the array's name as a device address; the first call on a
// device (with that device current) fetches the address with
// cudaGetSymbolAddress and clears the status word, so that first call should
// happen before any stream capture.  Every call on a device shares the one
// array: calls that overlap on the GPU (different streams without ordering)
// race on it.
#include <cuda_runtime.h>

#include <mutex>

#include "handle.h"

namespace archead {
namespace {

constexpr size_t kStaticWorkspaceBytes = size_t(2) << 20;   // 2 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

std::mutex g_setup_mutex;
void* g_static_ptr[kMaxDevices] = {};

// Device address of g_static_workspace on `dev` (current), set up once.
int static_workspace(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevices) return ARCHEAD_EUNSUP;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_static_ptr[dev] == nullptr) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_static_workspace);
    if (e != cudaSuccess) return set_cuda_error(e);
    // The status word is sticky: start it at zero.  The completion ticket is
    // reset by every call's prologue.
    e = cudaMemset(p, 0, 256);
    if (e != cudaSuccess) return set_cuda_error(e);
    g_static_ptr[dev] = p;
  }
  *out = g_static_ptr[dev];
  return ARCHEAD_OK;
}

}  // namespace
}  // namespace archead

using namespace archead;

extern "C" ARCHEAD_API size_t archead_static_workspace_capacity(void) { return kStaticWorkspaceBytes; }

extern "C" ARCHEAD_API int archead_logits_lse_argmax_static(const archead_handle* handle, const uint16_t* hidden,
                                                            int32_t T, const int32_t* targets, float* lse,
                                                            int32_t* argmax, float* ce, archead_stream_t stream) {
  if (handle == nullptr || T <= 0) return ARCHEAD_EINVAL;
  const size_t need = archead_workspace_bytes(handle, T);
  if (need == 0) return ARCHEAD_EINVAL;
  if (need > kStaticWorkspaceBytes) return ARCHEAD_ENOMEM;   // T too large for the fixed array
  int dev = -1;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_cuda_error(e);
  if (dev != handle->device) return ARCHEAD_EINVAL;
  void* ws = nullptr;
  const int rc = static_workspace(dev, &ws);
  if (rc != ARCHEAD_OK) return rc;
  return archead_logits_lse_argmax(handle, hidden, T, targets, lse, argmax, ce, ws, kStaticWorkspaceBytes, stream);
}
