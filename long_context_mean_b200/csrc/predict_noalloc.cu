// sa_predict_mask_noalloc: mask prediction for callers that cannot allocate
// device memory.
//
// Some callers have no way to obtain a workspace buffer: code that runs
// inside another runtime's memory pool without a handle to it, a plug-in
// that is only handed pre-sized input and output tensors, or a process that
// must not grow its device footprint once it is serving.  For them this file
// keeps the scratch that sa_predict_mask needs (block means, block
// similarities, row counts, sort scratch) in a fixed array that belongs to
// the library itself: it is created when the library is loaded on a device
// and stays until the process exits, on every device that loads the library.
//
// The array holds kNoallocScratchBytes (32 MiB), enough for the mask
// prediction of every workload shipped here (the largest, 32 query heads of
// 131,072 tokens at bq = 128, bk = 64, d = 128, needs about 25 MiB).  Larger
// problems are rejected with SA_ERR_WORKSPACE.  Every call uses the same
// array and leaves its contents behind; each call writes every scratch value
// it reads before reading it, so nothing needs clearing, but two calls whose
// work overlaps on the GPU (different streams, different threads) race on
// the array and must be serialised by the caller.
//
// The device address of the array is looked up with cudaGetSymbolAddress the
// first time the entry point runs on a device (with that device current);
// make that first call before any stream capture begins on the device.  The
// address is kept for the life of the process: after cudaDeviceReset (or any
// other teardown of the device's primary context) the library would hold a
// stale address, so the entry point must not be used across a device reset.
#include <mutex>

#include "sa_internal.cuh"

namespace sa {
namespace {

constexpr size_t kNoallocScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_predict_scratch[kNoallocScratchBytes];

std::mutex g_lookup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_predict_scratch on the current device (looked up once
// per device).
sa_status scratch_on_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return set_error(SA_ERR_CUDA, "no usable CUDA device");
  }
  if (dev < 0 || dev >= kMaxDevices) return set_error(SA_ERR_UNSUPPORTED, "device index %d beyond %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_lookup_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_predict_scratch);
    if (e != cudaSuccess || ptr == nullptr)
      return set_error(SA_ERR_CUDA, "cudaGetSymbolAddress(predict scratch) failed: %s", cudaGetErrorString(e));
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return SA_OK;
}

}  // namespace
}  // namespace sa

using namespace sa;

extern "C" sa_status sa_predict_mask_noalloc(const void* q, const void* k, const sa_shape* shape,
                                             const sa_mask_params* params, sa_mask* out, void* stream) {
  if (!shape || !params) return set_error(SA_ERR_INVALID_ARG, "NULL argument to sa_predict_mask_noalloc");
  const size_t need = sa_predict_mask_workspace(shape, params);
  if (need == 0) return sa_predict_mask(q, k, shape, params, nullptr, 0, out, stream);  // reports the argument error
  if (need > kNoallocScratchBytes)
    return set_error(SA_ERR_WORKSPACE,
                     "sa_predict_mask_noalloc: this shape needs %zu bytes of scratch, more than the %zu bytes "
                     "the library holds; use sa_predict_mask with a caller-provided workspace",
                     need, kNoallocScratchBytes);
  void* ws = nullptr;
  if (sa_status e = scratch_on_current_device(&ws)) return e;
  return sa_predict_mask(q, k, shape, params, ws, kNoallocScratchBytes, out, stream);
}
