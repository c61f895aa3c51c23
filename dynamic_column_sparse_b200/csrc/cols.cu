// cols.cu - standalone gather / scatter of selected cache columns.
//
// The activation cache is block-column-major ([nb][H][Bt] bf16), so one
// selected column of one token block is a contiguous run of Bt * 2 bytes
// (256 B at Bt = 128). Each run moves as Bt/8 16-byte vectors handled by
// consecutive threads, so every warp access is fully coalesced.
#include "kernels.cuh"
#include "ptx.cuh"

namespace cm {
namespace {

template <bool GATHER>
__global__ void __launch_bounds__(256) cols_kernel(const uint4 *__restrict__ src, uint4 *__restrict__ dst,
                                                   const int32_t *__restrict__ idx, int64_t nb, int64_t H, int vecs,
                                                   int k, const int *status) {
  if (*(volatile const int *)status != kDevOk) return;  // an earlier failure is pending: do nothing
  const int64_t total = nb * k * vecs;
  for (int64_t g = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; g < total;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t run = g / vecs;
    const int v = static_cast<int>(g - run * vecs);
    const int64_t b = run / k;
    const int64_t c = __ldg(idx + run);
    if (c < 0 || c >= H) continue;  // out-of-range index: move nothing
    const int64_t cache_vec = (b * H + c) * vecs + v;
    if (GATHER)
      dst[g] = __ldg(src + cache_vec);
    else
      dst[cache_vec] = __ldg(src + g);
  }
}

cudaError_t launch_cols(bool gather, const uint16_t *src, uint16_t *dst, const int32_t *idx, int64_t nb, int64_t H,
                        int Bt, int k, const int *status, cudaStream_t s) {
  if (nb <= 0 || k <= 0) return cudaSuccess;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int vecs = Bt / 8;
  const int64_t total = nb * k * vecs;
  const int64_t want = (total + 255) / 256;
  const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(want, static_cast<int64_t>(sms) * 8));
  if (gather)
    cols_kernel<true><<<static_cast<unsigned>(grid), 256, 0, s>>>(reinterpret_cast<const uint4 *>(src),
                                                                  reinterpret_cast<uint4 *>(dst), idx, nb, H, vecs, k,
                                                                  status);
  else
    cols_kernel<false><<<static_cast<unsigned>(grid), 256, 0, s>>>(reinterpret_cast<const uint4 *>(src),
                                                                   reinterpret_cast<uint4 *>(dst), idx, nb, H, vecs, k,
                                                                   status);
  return cudaGetLastError();
}

__global__ void selftest_wait_kernel(int *status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  mbar_wait(&bar, 0, status, &abort_flag);  // never signalled: gives up after the wait limit
  __syncthreads();
}

}  // namespace

cudaError_t launch_selftest_wait(int *status, cudaStream_t s) {
  selftest_wait_kernel<<<1, 32, 0, s>>>(status);
  return cudaGetLastError();
}

cudaError_t launch_gather_cols(const uint16_t *a_cache, int64_t nb, int64_t H, int Bt, const int32_t *idx, int k,
                               uint16_t *packed, int *status, cudaStream_t s) {
  return launch_cols(true, a_cache, packed, idx, nb, H, Bt, k, status, s);
}

cudaError_t launch_scatter_cols(const uint16_t *packed, int64_t nb, int64_t H, int Bt, const int32_t *idx, int k,
                                uint16_t *a_cache, int *status, cudaStream_t s) {
  return launch_cols(false, packed, a_cache, idx, nb, H, Bt, k, status, s);
}

}  // namespace cm
