// quant.cu - rows of bf16 values to e4m3 codes with one scale per row (the
// operands of the FP8 form of the sparse MLP step).
//
// For each row: amax = max |x| (fp32), inv = 448 / amax and scale = amax / 448
// (both fp32 divisions rounded to nearest; inv = scale = 1 for an all-zero
// row), code = e4m3(x * inv) rounded to nearest even with saturation at +-448,
// so that x ~ scale * code. One warp per row, 16 elements (two 16-byte bf16
// loads, one 16-byte code store) per lane and step.
#include <cuda_fp8.h>

#include <algorithm>

#include "kernels.cuh"
#include "ptx.cuh"

namespace cm {
namespace {

__global__ void __launch_bounds__(256) quantize_e4m3_rows_kernel(const uint16_t *__restrict__ x, int64_t rows,
                                                                 int64_t cols, uint8_t *__restrict__ codes,
                                                                 float *__restrict__ scales, const int *status) {
  if (*(volatile const int *)status != kDevOk) return;
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t groups = cols / 16;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows;
       row += warps) {
    const uint4 *src = reinterpret_cast<const uint4 *>(x + row * cols);
    float amax = 0.f;
    for (int64_t g = lane; g < groups; g += 32) {
      const uint4 u[2] = {src[2 * g], src[2 * g + 1]};
      const uint32_t *w = reinterpret_cast<const uint32_t *>(u);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        amax = fmaxf(amax, fabsf(__uint_as_float(w[e] << 16)));
        amax = fmaxf(amax, fabsf(__uint_as_float(w[e] & 0xffff0000u)));
      }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 1.f;
    if (lane == 0) scales[row] = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
    uint4 *dst = reinterpret_cast<uint4 *>(codes + row * cols);
    for (int64_t g = lane; g < groups; g += 32) {
      const uint4 u[2] = {src[2 * g], src[2 * g + 1]};
      const uint32_t *w = reinterpret_cast<const uint32_t *>(u);
      uint32_t out[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t word = 0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t pair = w[2 * q + h];
          const float lo = __uint_as_float(pair << 16), hi = __uint_as_float(pair & 0xffff0000u);
          const uint32_t c0 = __nv_cvt_float_to_fp8(__fmul_rn(lo, inv), __NV_SATFINITE, __NV_E4M3);
          const uint32_t c1 = __nv_cvt_float_to_fp8(__fmul_rn(hi, inv), __NV_SATFINITE, __NV_E4M3);
          word |= (c0 | (c1 << 8)) << (16 * h);
        }
        out[q] = word;
      }
      dst[g] = make_uint4(out[0], out[1], out[2], out[3]);
    }
  }
}

}  // namespace

cudaError_t launch_quantize_e4m3_rows(const uint16_t *x, int64_t rows, int64_t cols, uint8_t *codes, float *scales,
                                      int *status, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  const int64_t blocks = std::min<int64_t>((rows + 7) / 8, 148 * 8);
  quantize_e4m3_rows_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(x, rows, cols, codes, scales, status);
  return cudaGetLastError();
}

}  // namespace cm
