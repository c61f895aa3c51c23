// noalloc.cu - chipmunk_mlp_delta_noalloc: the sparse MLP step with its delta
// scratch in a fixed device array of the library, for callers that cannot
// allocate device memory.
//
// The array lives in this translation unit alone, so its module (and with it
// the 64 MiB on each device) is loaded only when this entry point is first
// used, under CUDA's default lazy module loading; with eager loading
// (CUDA_MODULE_LOADING=EAGER) every device that creates a context while the
// library is loaded reserves it.
#include <mutex>

#include "abi_internal.cuh"

namespace {

// In host code this name is a host-side stand-in, not a device address: the
// device address comes from cudaGetSymbolAddress below.
__device__ __align__(256) unsigned char g_noalloc_scratch[CHIPMUNK_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices] = {};

// One-time per-device look-up of the scratch array's device address, with
// that device current (the caller's current device).
chipmunk_status noalloc_scratch(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cm::record_error(CHIPMUNK_ERR_CUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return cm::record_error(CHIPMUNK_ERR_UNSUPPORTED, "device ordinal out of range");
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess)
      return cm::record_error(CHIPMUNK_ERR_CUDA, "cudaGetSymbolAddress(no-alloc scratch) failed: the device may not "
                                                 "have 64 MiB free for the library's fixed scratch array");
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return CHIPMUNK_OK;
}

}  // namespace

extern "C" chipmunk_status chipmunk_mlp_delta_noalloc(const chipmunk_mlp_args *a, chipmunk_stream stream) {
  return cm::mlp_delta_fixed_scratch(a, CHIPMUNK_NOALLOC_SCRATCH_BYTES, noalloc_scratch,
                                     static_cast<cudaStream_t>(stream));
}
