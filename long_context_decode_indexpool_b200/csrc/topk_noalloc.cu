// spx_topk_blocks_noalloc: the top-k block selection for callers that cannot
// hand the library a scratch buffer.
//
// Some callers cannot allocate device memory when they call the layer: a
// framework whose allocator owns every byte of the device, a runtime that
// forbids cudaMalloc on its serving path because it synchronises the whole
// device, or a plugin host that gives kernels their inputs and outputs but no
// scratch.  For them this entry point runs the same kernels as
// spx_topk_blocks, with the multi-level candidate lists kept in one fixed
// array that is part of the library itself (a file-scope __device__ array, so
// every GPU that loads the library holds it until the process exits).
//
// The array's name seen from host code is only a host-side handle, not a
// device address: the device address is looked up once per device with
// cudaGetSymbolAddress (with that device current) and cached for the life of
// the process, which assumes the device is not reset (cudaDeviceReset) in
// between.  That lookup happens inside the first call on each device, so the
// first call on a device should be made before any stream capture begins.
// Devices with an index beyond the cache look the address up on every call.
//
// Every call shares the one array and leaves its contents behind; nothing in
// it has to start at zero (each list count is written before it is read).
// Calls whose kernels overlap on the GPU (other streams, other host threads)
// race on the array: serialise them.
#include <cmath>
#include <cstdint>
#include <mutex>

#include "spx.h"
#include "spx_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_topk_scratch[SPX_TOPK_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_topk_scratch on the current device, or nullptr.
void* scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return nullptr;
  if (dev >= kMaxDevices) {  // not cached
    void* p = nullptr;
    return cudaGetSymbolAddress(&p, g_topk_scratch) == cudaSuccess ? p : nullptr;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_topk_scratch) != cudaSuccess || p == nullptr) return nullptr;
    g_scratch_addr[dev] = p;
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" spx_status spx_topk_blocks_noalloc(const spx_dims* d, int32_t rows, const float* scores,
                                              int64_t score_stride, const int64_t* n_vis,
                                              int64_t max_len, int32_t* idx, int32_t* count,
                                              spx_stream stream) {
  const spx_status st = spx::check_dims(d);
  if (st != SPX_OK) return st;
  if (rows < 1 || rows > 65535 || max_len < 0) return SPX_ERR_SHAPE;
  if (max_len / spx::kPool > (int64_t(1) << 31) - 1) return SPX_ERR_SHAPE;
  if (score_stride < max_len / spx::kPool) return SPX_ERR_SHAPE;
  if (!scores || !n_vis || !idx || !count) return SPX_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(scores) | reinterpret_cast<uintptr_t>(idx) |
       reinterpret_cast<uintptr_t>(count)) & 3u)
    return SPX_ERR_INVALID_ARG;
  const spx::TopkPlan plan = spx::plan_topk(rows, max_len);
  if (plan.ws_bytes > SPX_TOPK_NOALLOC_SCRATCH_BYTES) return SPX_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (plan.ws_bytes > 0) {
    scratch = scratch_address();
    if (!scratch) return SPX_ERR_CUDA;
  }
  const cudaError_t e = spx::launch_topk(plan, scores, score_stride, n_vis, max_len, idx, count,
                                         scratch, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SPX_OK : SPX_ERR_CUDA;
}
