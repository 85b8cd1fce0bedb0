// s2o_build_indices_static: the index build with its scratch in a fixed device array that the
// library owns, for callers that cannot allocate device memory themselves.
//
// Who needs this: code that runs where allocating is not allowed or not possible — a plugin or
// operator inside another framework that hands it only its inputs and outputs, a real-time or
// graph-replayed serving path that forbids cudaMalloc (it can synchronise the device and stall
// other streams), or a host that must keep its device memory footprint fixed after start-up.
// Those callers pass Q, K and the index arrays; the scratch lives in this file's static array.
//
// The array is a file-scope __device__ object, so every GPU that loads the library holds
// S2O_STATIC_WORKSPACE_BYTES for it until the process exits. Host code cannot use the symbol's
// name as a device address (on the host it names a stand-in object), so the first call on each
// device looks up the real address with cudaGetSymbolAddress while that device is current, and
// caches it per device together with the unique id of the device's context at that time. A later
// call on a device whose context has been replaced (cudaDeviceReset, or a primary context released
// and created again) finds another id and looks the address up again, so a stale address from a
// destroyed context is never used.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "s2o_internal.h"

namespace s2o {
namespace {

constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_static_workspace[S2O_STATIC_WORKSPACE_BYTES];

std::mutex g_static_mutex;
char *g_static_ptr[kMaxDevices] = {};
unsigned long long g_static_ctx[kMaxDevices] = {};

// Unique id of the calling thread's current context (cuCtxGetId, through the runtime's driver
// entry point query: no link against libcuda). 0 if it cannot be had.
unsigned long long current_context_id() {
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_id || !get_cur || get_cur(&ctx) != CUDA_SUCCESS || !ctx ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the static scratch on the current device: looked up on the first call with
// the device current and again whenever the device's context has changed since.
cudaError_t static_workspace(char **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  // 0 when no context is current on this thread yet (the runtime binds the device's primary
  // context on its first call that needs one): the lookup below then runs, and binds it.
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_static_mutex);
  if (!g_static_ptr[dev] || ctx == 0 || g_static_ctx[dev] != ctx) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_workspace);
    if (e != cudaSuccess) return e;
    g_static_ptr[dev] = static_cast<char *>(p);
    g_static_ctx[dev] = current_context_id();
  }
  *out = g_static_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace s2o

extern "C" s2o_status s2o_build_indices_static(const s2o_config *cfg, const void *q,
                                               const void *k, const s2o_indices *out,
                                               s2o_stream stream) {
  size_t need = 0;
  s2o_status st = s2o_workspace_size(cfg, &need);
  if (st != S2O_OK) return st;
  if (need > (size_t)S2O_STATIC_WORKSPACE_BYTES) return S2O_ERR_WORKSPACE_TOO_SMALL;
  char *ws = nullptr;
  if (s2o::static_workspace(&ws) != cudaSuccess) return S2O_ERR_CUDA;
  // The index build writes every scratch element before it reads it, so stale contents from an
  // earlier call need no clearing.
  return s2o_build_indices(cfg, q, k, out, ws, (size_t)S2O_STATIC_WORKSPACE_BYTES, stream);
}
