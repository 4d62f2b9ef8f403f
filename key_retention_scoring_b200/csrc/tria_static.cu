// tria_compress_pass_static: the compression pass with its scratch carved
// from a fixed device array of this library instead of a caller's workspace.
//
// It exists for callers that cannot hand the library a workspace allocation:
// a serving engine that reserves all free device memory for its KV-cache
// block pool at start-up (a later cudaMalloc would fail or shrink the pool),
// or a decode loop that must not stall other streams (cudaMalloc and
// cudaFree may synchronise the device).  Nothing here allocates: the array is
// part of the library's device image, and each call only enqueues a memset of
// the scratch header, the pass's kernels and an optional status copy.
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/tria.h"

namespace {

static __device__ __align__(256) unsigned char g_scratch[TRIA_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
constexpr size_t kHeaderBytes = 256;  // work counter (bytes 0..3), status flags (4..7)

// The array's device address belongs to a CUDA context: after a device reset
// the next context loads the library's device code again, possibly at
// another address.  So the cached address is keyed by the id of the context
// it was looked up in (cuCtxGetId: unique for the life of the process).
struct ScratchEntry {
  unsigned long long ctx_id;
  void *ptr;
};

std::mutex g_mu;
ScratchEntry g_scratch_of[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// Id of the calling thread's current context; false if there is none yet.
bool current_ctx_id(unsigned long long *id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *a = nullptr, *b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
        qa == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
        qb == cudaDriverEntryPointSuccess) {
      get_current = reinterpret_cast<CtxGetCurrentFn>(a);
      get_id = reinterpret_cast<CtxGetIdFn>(b);
    }
  });
  if (get_current == nullptr || get_id == nullptr) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Address of the array in the current device's context: looked up once per
// context (cudaGetSymbolAddress, which also makes the device's primary
// context current if no context is yet).
tria_status scratch_of_current_device(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return TRIA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return TRIA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  unsigned long long id = 0;
  const bool have_id = current_ctx_id(&id);
  ScratchEntry &e = g_scratch_of[dev];
  if (!have_id || e.ptr == nullptr || e.ctx_id != id) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) return TRIA_ERR_CUDA;
    if (!current_ctx_id(&id)) return TRIA_ERR_CUDA;
    e.ctx_id = id;
    e.ptr = p;
  }
  *out = e.ptr;
  return TRIA_OK;
}

}  // namespace

extern "C" tria_status tria_compress_pass_static(const tria_stats *stats,
                                                 const tria_cache_view *cache,
                                                 const tria_params *params, int32_t *kept_idx,
                                                 int32_t *freed_blocks, int32_t *n_freed,
                                                 int32_t *device_status, tria_stream_t stream) {
  if (stats == nullptr || cache == nullptr || params == nullptr) return TRIA_ERR_INVALID_ARG;
  tria_model_desc desc;
  tria_status st = tria_stats_desc(stats, &desc);
  if (st != TRIA_OK) return st;
  size_t need = 0;
  if ((st = tria_workspace_size(stats, cache, params, 0, desc.n_layers, &need)) != TRIA_OK)
    return st;
  if (need > (size_t)TRIA_STATIC_SCRATCH_BYTES) return TRIA_ERR_WORKSPACE;
  void *ws = nullptr;
  if ((st = scratch_of_current_device(&ws)) != TRIA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the work counter and the status flags must start at zero; every other
  // region is written by the pass's kernels before it is read
  if (cudaMemsetAsync(ws, 0, kHeaderBytes, s) != cudaSuccess) return TRIA_ERR_CUDA;
  st = tria_compress_pass(stats, cache, params, kept_idx, freed_blocks, n_freed, ws,
                          (size_t)TRIA_STATIC_SCRATCH_BYTES, stream);
  if (st != TRIA_OK) return st;
  if (device_status != nullptr &&
      cudaMemcpyAsync(device_status, static_cast<unsigned char *>(ws) + 4, sizeof(int32_t),
                      cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return TRIA_ERR_CUDA;
  return TRIA_OK;
}
