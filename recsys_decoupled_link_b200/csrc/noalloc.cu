// lime_build_qk_cache_noalloc: the QK-cache build for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc: a plug-in hosted by a serving framework
// that owns the whole device memory pool and forbids its plug-ins to allocate,
// or a latency-critical serving loop where cudaMalloc's implicit device
// synchronisation is not acceptable.  They still own their inputs and
// outputs, but cannot provide the workspace lime_build_qk_cache takes.  This
// entry point runs the same cache build with its scratch in a file-scope
// static device array of LIME_NOALLOC_SCRATCH_BYTES bytes instead.
//
// The array is part of the library's device image: every GPU that loads the
// library holds it until the process exits.  Host code cannot use the array's
// name as a device address (on the host it names a stand-in object), so the
// entry point, with the device current, looks its device address up with
// cudaGetSymbolAddress on every call outside a stream capture and keeps it for
// calls made during one; the first call on each device should therefore come
// before any stream capture.  All calls share the one array and
// it keeps the last call's contents: each call clears the status word at its
// head before use, and calls that overlap on the GPU (e.g. on two streams) race
// on it.  Nothing here calls cudaMalloc, cudaFree or an allocating library
// routine.
#include <stdio.h>

#include <mutex>

#include "lime.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[LIME_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

// Device address of g_noalloc_scratch on the current device, nullptr if the
// runtime refuses.  Looked up again on every call made outside a stream
// capture (the address can change if the device's context is reset and the
// module reloaded); a call made while `stream` is capturing uses the address
// the last uncaptured call on this device found, so the first call on a device
// has to come before any capture.
void* scratch_address(cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (cs == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) {
      fprintf(stderr, "liblime: cudaGetSymbolAddress(scratch) failed: %s\n",
              cudaGetErrorString(e));
      return nullptr;
    }
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

namespace lime {
int check_cache_args(const lime_dims* dims, const void* T, int64_t n_items, const void* L,
                     const void* Wq_c, const void* Wk_c, const void* cache_out);
}

extern "C" int lime_build_qk_cache_noalloc(const lime_dims* dims, const void* T,
                                           int64_t n_items, const void* L, const void* Wq_c,
                                           const void* Wk_c, void* cache_out,
                                           cudaStream_t stream) {
  // the same argument checks as lime_build_qk_cache, with the same codes,
  // before the shared array is touched
  int rc = lime::check_cache_args(dims, T, n_items, L, Wq_c, Wk_c, cache_out);
  if (rc != LIME_OK) return rc;
  const size_t need = lime_workspace_bytes(dims, 0, 0);
  if (need > (size_t)LIME_NOALLOC_SCRATCH_BYTES) {
    fprintf(stderr,
            "liblime: lime_build_qk_cache_noalloc needs %zu bytes of scratch, more than its "
            "static maximum of %u bytes; use lime_build_qk_cache with a workspace\n",
            need, (unsigned)LIME_NOALLOC_SCRATCH_BYTES);
    return LIME_ERR_SCRATCH;
  }
  void* scratch = scratch_address(stream);
  if (!scratch) return LIME_ERR_CUDA;
  rc = lime_workspace_init(scratch, LIME_NOALLOC_SCRATCH_BYTES, stream);
  if (rc != LIME_OK) return rc;
  return lime_build_qk_cache(dims, T, n_items, L, Wq_c, Wk_c, cache_out, scratch,
                             LIME_NOALLOC_SCRATCH_BYTES, stream);
}

// The status word of the static array (device-side flags of the last
// lime_build_qk_cache_noalloc call on this device: LIME_FLAG_TIMEOUT when a
// bounded wait gave up and the cache may be partly written), read and cleared
// like lime_get_status reads a workspace's.  Allocation-free; not callable
// while `stream` is capturing (the read synchronises).
extern "C" int lime_noalloc_get_status(cudaStream_t stream, int* flags) {
  if (!flags) return LIME_ERR_ARG;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return LIME_ERR_CUDA;
  if (cs != cudaStreamCaptureStatusNone) return LIME_ERR_ARG;
  void* scratch = scratch_address(stream);
  if (!scratch) return LIME_ERR_CUDA;
  return lime_get_status(scratch, stream, flags);
}
