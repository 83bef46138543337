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
// code cannot use the array's name as a device address; a call on a device
// (with that device current) whose context has not been seen before fetches
// the address with cudaGetSymbolAddress and clears the status word on the
// caller's stream, so the first call on a device should happen before any
// stream capture.  A later context on the same device (after cudaDeviceReset)
// is detected by its context handle and set up again the same way.  Every
// call on a device shares the one array: calls that overlap on the GPU
// (different streams without ordering) race on it.  The status word is sticky
// (an OR of ARCHEAD_STATUS_* bits since the last clear);
// archead_static_workspace_status reads and optionally clears it.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "handle.h"

namespace archead {
namespace {

constexpr size_t kStaticWorkspaceBytes = size_t(2) << 20;   // 2 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

using CtxGetCurrent = CUresult (*)(CUcontext*);

struct StaticSlot {
  CUcontext ctx;   // context the address below belongs to
  void* ptr;       // device address of g_static_workspace in that context
};

std::mutex g_setup_mutex;
StaticSlot g_slots[kMaxDevices] = {};
CtxGetCurrent g_ctx_get_current = nullptr;

// The current context of the calling thread (driver API, looked up through the
// runtime so that the library needs no link to libcuda).
int current_context(CUcontext* out) {
  if (g_ctx_get_current == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    const cudaError_t e = cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess) return set_cuda_error(e);
    if (q != cudaDriverEntryPointSuccess || fn == nullptr) return ARCHEAD_EUNSUP;
    g_ctx_get_current = reinterpret_cast<CtxGetCurrent>(fn);
  }
  CUcontext c = nullptr;
  if (g_ctx_get_current(&c) != CUDA_SUCCESS) return ARCHEAD_EUNSUP;
  *out = c;   // null when no context is current yet
  return ARCHEAD_OK;
}

// Device address of g_static_workspace on `dev` (current) in the current
// context; the first call in a context clears the status word on `stream`.
int static_workspace(int dev, cudaStream_t stream, void** out) {
  if (dev < 0 || dev >= kMaxDevices) return ARCHEAD_EUNSUP;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  CUcontext ctx = nullptr;
  int rc = current_context(&ctx);
  if (rc != ARCHEAD_OK) return rc;
  StaticSlot& s = g_slots[dev];
  if (ctx == nullptr || s.ptr == nullptr || s.ctx != ctx) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_static_workspace);   // makes the primary context current
    if (e != cudaSuccess) return set_cuda_error(e);
    rc = current_context(&ctx);
    if (rc != ARCHEAD_OK) return rc;
    if (ctx == nullptr) return ARCHEAD_EUNSUP;
    // The status word is sticky: start it at zero, ordered before this call's
    // kernels on the same stream.  The completion ticket is reset by every
    // call's prologue.
    e = cudaMemsetAsync(p, 0, 256, stream);
    if (e != cudaSuccess) return set_cuda_error(e);
    s.ctx = ctx;
    s.ptr = p;
  }
  *out = s.ptr;
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
  const int rc = static_workspace(dev, reinterpret_cast<cudaStream_t>(stream), &ws);
  if (rc != ARCHEAD_OK) return rc;
  return archead_logits_lse_argmax(handle, hidden, T, targets, lse, argmax, ce, ws, kStaticWorkspaceBytes, stream);
}

extern "C" ARCHEAD_API int archead_static_workspace_status(int clear, archead_stream_t stream, uint32_t* status_out) {
  if (status_out == nullptr) return ARCHEAD_EINVAL;
  int dev = -1;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_cuda_error(e);
  void* ws = nullptr;
  const int rc = static_workspace(dev, reinterpret_cast<cudaStream_t>(stream), &ws);
  if (rc != ARCHEAD_OK) return rc;
  return archead_workspace_status(ws, clear, stream, status_out);
}
