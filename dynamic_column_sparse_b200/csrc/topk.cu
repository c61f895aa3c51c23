// topk.cu - per-row top-k column selection (the sparsity identification step).
//
// For each row: the k largest fp32 scores, ties to the lower index, written as
// ascending column indices. Scores become order-preserving uint32 keys; a
// three-pass radix select (11 + 11 + 10 bits, 2048-bin shared histograms)
// finds the exact k-th key tau and how many keys equal to tau are taken;
// a stable block-wide compaction in index order then writes the result.
// One CTA per row (grid-stride). Rows of up to kStagedMaxN scores are staged
// in shared memory once; longer rows are re-read from global memory (L2) by
// each pass.
#include "kernels.cuh"
#include "ptx.cuh"

namespace cm {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxBins = 2048;
constexpr int kItems = 8;             // consecutive elements per thread in the compaction
constexpr int kStagedMaxN = 40960;    // 160 KB of keys in shared memory

__device__ __forceinline__ uint32_t ordered_key(float f) {
  uint32_t b = __float_as_uint(f);
  if (b == 0x80000000u) b = 0u;  // -0 compares equal to +0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Block-wide exclusive scan of a 64-bit value; also returns the block total.
__device__ __forceinline__ uint64_t block_excl_scan(uint64_t v, uint64_t *warp_tot, uint64_t &total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint64_t inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint64_t t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    uint64_t w = lane < kWarps ? warp_tot[lane] : 0;
    uint64_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint64_t t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    if (lane < kWarps) warp_tot[lane] = wi - w;  // exclusive prefix of each warp
    if (lane == kWarps - 1) warp_tot[kWarps] = wi;
  }
  __syncthreads();
  uint64_t res = warp_tot[warp] + inc - v;
  total = warp_tot[kWarps];
  __syncthreads();
  return res;
}

template <bool STAGED>
__global__ void __launch_bounds__(kThreads) topk_kernel(const TopkParams p) {
  extern __shared__ uint32_t staged[];
  __shared__ uint32_t hist[kMaxBins];
  __shared__ uint64_t warp_tot[kWarps + 1];
  __shared__ uint32_t s_digit, s_above;

  const int tid = threadIdx.x;
  const int n = static_cast<int>(p.n);
  const int k = p.k;
  if (*(volatile int *)p.status != kDevOk) return;  // an earlier failure is pending: do nothing

  for (int64_t row = blockIdx.x; row < p.rows; row += gridDim.x) {
    const float *src = p.scores + row * p.ld_scores;
    int32_t *dst = p.idx + row * p.ld_idx;
    if (k >= n) {
      for (int i = tid; i < n; i += kThreads) dst[i] = i;
      continue;
    }
    if (STAGED) {
      for (int i = tid; i < n; i += kThreads) staged[i] = ordered_key(__ldg(src + i));
      __syncthreads();
    }
    uint32_t prefix = 0, mask = 0;
    int kk = k;  // keys still to take among those matching prefix
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
      const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
      const int nbins = pass == 2 ? 1024 : 2048;
      for (int i = tid; i < nbins; i += kThreads) hist[i] = 0;
      __syncthreads();
      for (int i = tid; i < n; i += kThreads) {
        const uint32_t key = STAGED ? staged[i] : ordered_key(__ldg(src + i));
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & (nbins - 1)], 1u);
      }
      __syncthreads();
      // thread t owns bins [nbins - (t+1)*per, nbins - t*per): thread 0 the highest
      const int per = nbins / kThreads;
      const int hi = nbins - tid * per;
      uint32_t local = 0;
      for (int b = hi - 1; b >= hi - per; --b) local += hist[b];
      uint64_t tot;
      const uint32_t above = static_cast<uint32_t>(block_excl_scan(local, warp_tot, tot));
      if (above < static_cast<uint32_t>(kk) && above + local >= static_cast<uint32_t>(kk)) {
        uint32_t cum = above;
        for (int b = hi - 1; b >= hi - per; --b) {
          if (cum + hist[b] >= static_cast<uint32_t>(kk)) {
            s_digit = static_cast<uint32_t>(b);
            s_above = cum;
            break;
          }
          cum += hist[b];
        }
      }
      __syncthreads();
      prefix |= s_digit << shift;
      mask |= static_cast<uint32_t>(nbins - 1) << shift;
      kk -= static_cast<int>(s_above);
      __syncthreads();
    }
    const uint32_t tau = prefix;
    // stable compaction: an element is kept if its key exceeds tau, or equals
    // tau and fewer than kk equal keys precede it
    uint32_t run_gt = 0, run_eq = 0;
    const int tile = kThreads * kItems;
    for (int base = 0; base < n; base += tile) {
      const int first = base + tid * kItems;
      uint32_t keys[kItems];
      uint32_t n_gt = 0, n_eq = 0;
#pragma unroll
      for (int e = 0; e < kItems; ++e) {
        const int i = first + e;
        uint32_t key = 0;
        if (i < n) key = STAGED ? staged[i] : ordered_key(__ldg(src + i));
        keys[e] = key;
        if (i < n) {
          n_gt += key > tau;
          n_eq += key == tau;
        }
      }
      uint64_t tot;
      const uint64_t before = block_excl_scan((static_cast<uint64_t>(n_gt) << 32) | n_eq, warp_tot, tot);
      uint32_t gt_b = run_gt + static_cast<uint32_t>(before >> 32);
      uint32_t eq_b = run_eq + static_cast<uint32_t>(before & 0xffffffffu);
#pragma unroll
      for (int e = 0; e < kItems; ++e) {
        const int i = first + e;
        if (i >= n) break;
        if (keys[e] > tau) {
          const uint32_t pos = gt_b + min(eq_b, static_cast<uint32_t>(kk));
          if (pos < static_cast<uint32_t>(k)) dst[pos] = i;
          ++gt_b;
        } else if (keys[e] == tau) {
          if (eq_b < static_cast<uint32_t>(kk) && gt_b + eq_b < static_cast<uint32_t>(k)) dst[gt_b + eq_b] = i;
          ++eq_b;
        }
      }
      run_gt += static_cast<uint32_t>(tot >> 32);
      run_eq += static_cast<uint32_t>(tot & 0xffffffffu);
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_topk(const TopkParams &p, cudaStream_t s) {
  if (p.rows <= 0 || p.k <= 0) return cudaSuccess;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (p.n <= kStagedMaxN) {
    const size_t smem = static_cast<size_t>(p.n) * sizeof(uint32_t);
    static bool attr_set = false;
    if (!attr_set) {
      cudaError_t e = cudaFuncSetAttribute(topk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           kStagedMaxN * static_cast<int>(sizeof(uint32_t)));
      if (e != cudaSuccess) return e;
      attr_set = true;
    }
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, topk_kernel<true>, kThreads, smem);
    const int64_t grid = std::min<int64_t>(p.rows, static_cast<int64_t>(sms) * std::max(per_sm, 1));
    topk_kernel<true><<<static_cast<unsigned>(grid), kThreads, smem, s>>>(p);
  } else {
    // one CTA per SM keeps every row being scanned resident in L2 between passes
    const int64_t grid = std::min<int64_t>(p.rows, sms);
    topk_kernel<false><<<static_cast<unsigned>(grid), kThreads, 0, s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace cm
