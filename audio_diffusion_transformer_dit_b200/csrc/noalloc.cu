// Allocation-free variant of h3b_block_forward.
//
// Some callers cannot allocate device memory: code hosted inside an
// application that owns and accounts for every byte of device memory through
// its own pool, or a latency-critical thread that must not call cudaMalloc
// (it can synchronise the device and has no latency bound).  This entry point
// takes inputs and outputs only and keeps its scratch in a fixed-size array
// that lives in the library's own device image: every GPU that loads this
// code holds H3B_NOALLOC_MAX_BYTES for it until the process exits.
//
// In host code the array's name only stands in for it; its device address is
// looked up once per device with cudaGetSymbolAddress (with that device
// current) on the first call, and that address is what the kernels receive.
// The address is cached for the life of the process: after cudaDeviceReset on
// a device the cached address (like the library's other per-device state) is
// stale, so the library must not be called on that device again.
#include <mutex>

#include "h3b.h"

#include <cuda_runtime.h>

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[H3B_NOALLOC_MAX_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set-up on the
// first call per device).  Returns nullptr if the lookup fails.
void* scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_noalloc_ptr[dev] = p;
  }
  return g_noalloc_ptr[dev];
}

}  // namespace

extern "C" int h3b_block_forward_noalloc(const h3b_dims* dims, const h3b_block_weights* w, float* x, int merged,
                                         void* stream) {
  if (!dims || !w) return H3B_ERR_NULL;
  if (w->dtype != H3B_BF16 && w->dtype != H3B_INT8) return H3B_ERR_DTYPE;
  const size_t need = h3b_workspace_bytes(dims, w->dtype, 0);
  if (need == 0) return H3B_ERR_DIMS;
  if (need > static_cast<size_t>(H3B_NOALLOC_MAX_BYTES)) return H3B_ERR_WORKSPACE;  // beyond the fixed scratch
  void* scratch = scratch_on_current_device();
  if (!scratch) return H3B_ERR_CUDA;
  return h3b_block_forward(dims, w, x, merged, scratch, static_cast<size_t>(H3B_NOALLOC_MAX_BYTES), stream);
}
