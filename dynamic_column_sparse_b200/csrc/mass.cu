// mass.cu - attention mass of every key per query block, with the top-k of
// each mass row selected inside the same kernel (fused refresh scoring).
//
// For head h and query block b the mass of key j is sum over the block's
// queries i of softmax_i(j) = exp2(s_ij * scale * log2 e - lse_i * log2 e),
// s_ij = q_i . k_j, with lse the dense pass's row log-sum-exp. Persistent CTAs
// walk the (head, query block) tiles head-major (the CTAs running together
// stream the same head's keys, which stay in L2). Per tile, warp 0 loads the
// 128 queries by TMA once and the keys in chunks of 128 through a two-stage
// ring; warp 1 issues D = K Q^T (TMEM lane = key, column = query) into one of
// two TMEM buffers; warps 2-9, one group of four per buffer, sum each key's
// column of exponentials, write the fp32 mass row and build a 4096-bin
// histogram of it (bins of 1/128 octave over [2^-24, 2^8); smaller values
// share bin 0, larger ones the top bin).
//
// Warps 10-13 select on the previous tile's finished row while the others
// compute the next: the histogram gives the bin holding the k-th largest mass;
// one pass over the row copies every mass in that bin or above, with its
// index, in index order into shared memory; three radix passes over those
// candidates find the exact k-th key, and a stable compaction writes the
// ascending indices. When the candidates do not fit, the radix passes and the
// compaction run over the whole row instead. The result is the exact top-k of
// the stored fp32 row, ties to the lower index.
//
// The row goes to the caller's mass tensor when one is given. Otherwise it
// goes to row buffers of the CTA that its tiles reuse, so the mass stays in L2
// and need not travel to HBM and back: two per CTA (tile j uses buffer j mod 2,
// free again once the selection of tile j - 2 is done) when both fit in a
// fraction of L2, else one, and then the mass warps write key chunk c of tile
// j only after the selection warps have read chunk c of tile j - 1 (a
// progress counter in shared memory).
#include <algorithm>

#include "kernels.cuh"
#include "ptx.cuh"
#include "select.cuh"

namespace cm {
namespace {

constexpr int kThreads = 448;          // warp 0 TMA, warp 1 MMA, warps 2-9 mass, warps 10-13 selection
constexpr int kMassThreads = 256;      // two groups of 128, one per TMEM buffer
constexpr int kSelWarp0 = 10;
constexpr int kSelThreads = 128;
using Sel = SelGroup<kSelThreads, 1>;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kTileBytes = 32768;  // 128 x 128 bf16, two 64-column swizzle halves

constexpr int kBins = 4096;
constexpr int kBinBase = 0x8000 + 103 * 128;  // key >> 16 of 2^-24: bin 0
constexpr int kCap = 10240;                   // candidates held in shared memory
constexpr int64_t kTwoSlotBytes = 48ll << 20; // row buffers of all CTAs, two per CTA, up to this size

constexpr uint32_t kQOff = 0;
constexpr uint32_t kKOff = kTileBytes;                   // [2]
constexpr uint32_t kBarOff = kKOff + 2 * kTileBytes;     // 18 barriers, progress, TMEM slot, abort flag
constexpr uint32_t kLseOff = kBarOff + 256;              // [2][128] fp32
constexpr uint32_t kHistOff = kLseOff + 2 * 128 * 4;     // [2][kBins] u32
constexpr uint32_t kCKeyOff = kHistOff + 2 * kBins * 4;  // [kCap] u32
constexpr uint32_t kCIdxOff = kCKeyOff + kCap * 4;       // [kCap] i32
constexpr uint32_t kSelOff = kCIdxOff + kCap * 4;        // scan words, digit results
constexpr uint32_t kSmem = 1024 + kSelOff + 256;
static_assert(kSmem <= 232448, "shared memory of one CTA");

// Floats per row buffer: whole 128-byte lines, so that a row's lines hold no other row.
__host__ __device__ __forceinline__ int64_t mass_row_pad(int64_t T) { return (T + 31) & ~static_cast<int64_t>(31); }

// Row buffers per CTA: two when those of all `grid` CTAs fit in kTwoSlotBytes.
__host__ __device__ __forceinline__ int64_t mass_row_slots(int64_t grid, int64_t T) {
  return 2 * grid * mass_row_pad(T) * 4 <= kTwoSlotBytes ? 2 : 1;
}

__device__ __forceinline__ uint32_t mass_bin(uint32_t key) {
  const int f = static_cast<int>(key >> 16) - kBinBase;
  return static_cast<uint32_t>(min(max(f, 0), kBins - 1));
}

// The smallest key of bin b; bin 0 holds every key below bin 1.
__device__ __forceinline__ uint32_t bin_floor(uint32_t b) {
  return b == 0 ? 0u : (b + static_cast<uint32_t>(kBinBase)) << 16;
}

__device__ __forceinline__ uint64_t ld_acquire_shared(const uint64_t *p) {
  uint64_t v;
  asm volatile("ld.acquire.cta.shared::cta.u64 %0, [%1];" : "=l"(v) : "r"(smem_u32(p)) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_shared(uint64_t *p, uint64_t v) {
  asm volatile("st.release.cta.shared::cta.u64 [%0], %1;" ::"r"(smem_u32(p)), "l"(v) : "memory");
}

// An L2 policy that evicts the lines it touches after others (the live mass rows).
__device__ __forceinline__ uint64_t l2_evict_last_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ void st_global_hint(float *p, float v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(p), "f"(v), "l"(pol) : "memory");
}

// Drops the 128-byte line at p from L2 without writing it back (its data is dead).
__device__ __forceinline__ void discard_l2_line(const void *p) {
  asm volatile("discard.global.L2 [%0], 128;" ::"l"(p) : "memory");
}

__device__ __forceinline__ bool wait_warp(uint64_t *bar, uint32_t parity, int *status, volatile int *abort_flag) {
  const bool ok = mbar_wait(bar, parity, status, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

// Lane 0 waits (bounded, like mbar_wait) until *progress >= need; warp-uniform result.
__device__ __forceinline__ bool wait_progress(const uint64_t *progress, uint64_t need, uint64_t &seen, int *status,
                                              volatile int *abort_flag) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) {
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
      seen = ld_acquire_shared(progress);
      if (seen >= need) break;
      if ((it & 1023u) == 1023u) {
        if (*abort_flag) {
          ok = false;
          break;
        }
        const uint64_t now = globaltimer_ns();
        if (t0 == 0) {
          t0 = now;
        } else if (now - t0 > kWaitLimitNs) {
          atomicCAS(status, kDevOk, kDevWaitTimeout);
          *abort_flag = 1;
          ok = false;
          break;
        }
      }
    }
  }
  seen = __shfl_sync(0xffffffffu, seen, 0);
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok;
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_mass_select_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                            const MassParams p) {
  constexpr uint32_t kIdesc = idesc_bf16(128, 128, false, false);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align_up<1024>(smem_raw);
  uint8_t *sQ = smem + kQOff;
  uint8_t *sK = smem + kKOff;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kBarOff);
  uint64_t *q_full = bars + 0;
  uint64_t *q_empty = bars + 1;
  uint64_t *k_full = bars + 2;      // [2]
  uint64_t *k_empty = bars + 4;     // [2]
  uint64_t *d_full = bars + 6;      // [2]
  uint64_t *d_free = bars + 8;      // [2]
  uint64_t *lse_full = bars + 10;   // [2] the tile's query log-sum-exps are in shared memory
  uint64_t *lse_empty = bars + 12;  // [2]
  uint64_t *row_ready = bars + 14;  // [2] a tile's mass row and histogram are complete
  uint64_t *hist_free = bars + 16;  // [2] the selection is done with a histogram (and zeroed it)
  uint64_t *progress = bars + 18;   // chunks of rows the selection has finished reading
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 19);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  int *start_bad = reinterpret_cast<int *>(bars + 20);  // an earlier failure was pending at entry
  float *lse2 = reinterpret_cast<float *>(smem + kLseOff);
  uint32_t *hist = reinterpret_cast<uint32_t *>(smem + kHistOff);
  uint32_t *ckey = reinterpret_cast<uint32_t *>(smem + kCKeyOff);
  int32_t *cidx = reinterpret_cast<int32_t *>(smem + kCIdxOff);
  uint64_t *warp_tot = reinterpret_cast<uint64_t *>(smem + kSelOff);   // [Sel::kWarps + 1]
  uint32_t *sel_res = reinterpret_cast<uint32_t *>(warp_tot + 16);      // [2]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.T;
  const int nch = (T + 127) / 128;
  const int tiles = p.h * p.nb;
  const bool shared_row = p.mass == nullptr;
  const int64_t row_pad = mass_row_pad(T);
  const int slots = static_cast<int>(mass_row_slots(gridDim.x, T));
  // the mass row of local tile j (global tile t)
  auto row_of = [&](int j, int t) -> float * {
    return shared_row ? p.row_buf + (static_cast<int64_t>(blockIdx.x) * slots + (j % slots)) * row_pad
                      : p.mass + static_cast<size_t>(t) * T;
  };

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&d_full[s], 1);
      mbar_init(&d_free[s], 128);
      mbar_init(&lse_full[s], 32);
      mbar_init(&lse_empty[s], kMassThreads);
      mbar_init(&row_ready[s], kMassThreads);
      mbar_init(&hist_free[s], 1);
    }
    *progress = 0;
    *abort_flag = 0;
    *start_bad = *(volatile int *)p.status != kDevOk;  // read once: every role takes the same branch
    fence_barrier_init();
  }
  for (int i = threadIdx.x; i < 2 * kBins; i += kThreads) hist[i] = 0;
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (*start_bad) {
    // an earlier launch failed: do nothing
  } else if (warp == 0) {
    // ---------------------------------------------------------------- loads
    uint32_t g = 0;
    for (int j = 0, t = blockIdx.x; t < tiles; ++j, t += gridDim.x) {
      const int hh = t / p.nb, b = t % p.nb;
      if (!wait_warp(&lse_empty[j & 1], ((j >> 1) & 1) ^ 1, p.status, abort_flag)) break;
      for (int e = lane; e < 128; e += 32) {
        const int gq = b * 128 + e;
        lse2[(j & 1) * 128 + e] = gq < T ? p.lse[static_cast<size_t>(hh) * T + gq] * kLog2e : INFINITY;
      }
      mbar_arrive(&lse_full[j & 1]);
      if (!wait_warp(q_empty, (j & 1) ^ 1, p.status, abort_flag)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(q_full, kTileBytes);
        tma_load_2d(sQ, &tm_q, q_full, hh * 128, b * 128);
        tma_load_2d(sQ + 16384, &tm_q, q_full, hh * 128 + 64, b * 128);
      }
      bool ok = true;
      for (int i = 0; i < nch; ++i, ++g) {
        const int s = g & 1;
        if (!wait_warp(&k_empty[s], ((g >> 1) & 1) ^ 1, p.status, abort_flag)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&k_full[s], kTileBytes);
          tma_load_2d(sK + s * kTileBytes, &tm_k, &k_full[s], hh * 128, i * 128);
          tma_load_2d(sK + s * kTileBytes + 16384, &tm_k, &k_full[s], hh * 128 + 64, i * 128);
        }
        __syncwarp();
      }
      if (!ok) break;
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    uint32_t g = 0;
    const uint32_t q0 = smem_u32(sQ);
    for (int j = 0, t = blockIdx.x; t < tiles; ++j, t += gridDim.x) {
      if (!wait_warp(q_full, j & 1, p.status, abort_flag)) break;
      tc_fence_after();
      bool ok = true;
      for (int i = 0; i < nch; ++i, ++g) {
        const int s = g & 1;
        if (!wait_warp(&k_full[s], (g >> 1) & 1, p.status, abort_flag) ||
            !wait_warp(&d_free[s], ((g >> 1) & 1) ^ 1, p.status, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t k0 = smem_u32(sK + s * kTileBytes);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            umma_bf16(tmem + s * 128, sdesc_sw128(k0 + off, 16, 1024), sdesc_sw128(q0 + off, 16, 1024), kIdesc,
                      kk > 0);
          }
          umma_commit(&k_empty[s]);
          umma_commit(&d_full[s]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) umma_commit(q_empty);
      __syncwarp();
    }
  } else if (warp < kSelWarp0) {
    // ---------------------------------------------------------------- mass
    const int group = (warp - 2) >> 2;  // takes the chunks that land in TMEM buffer `group`
    const int q = warp & 3;             // TMEM lane quadrant this warp may access
    const int r = q * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    uint32_t g = 0;
    uint64_t seen = 0;
    const uint64_t pol = l2_evict_last_policy();
    for (int j = 0, t = blockIdx.x; t < tiles; ++j, t += gridDim.x) {
      if (!wait_warp(&lse_full[j & 1], (j >> 1) & 1, p.status, abort_flag)) break;
      if (!wait_warp(&hist_free[j & 1], ((j >> 1) & 1) ^ 1, p.status, abort_flag)) break;
      const float *l2 = lse2 + (j & 1) * 128;
      uint32_t *hcur = hist + (j & 1) * kBins;
      float *row = row_of(j, t);
      bool ok = true;
      for (int i = 0; i < nch; ++i, ++g) {
        const int s = g & 1;
        if (s != group) continue;
        if (!wait_warp(&d_full[s], (g >> 1) & 1, p.status, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float v[32];
          tmem_ld32(tmem + lane_off + s * 128 + c * 32, v);
#pragma unroll
          for (int e = 0; e < 32; ++e) sum += exp2_approx(v[e] * p.scale_log2 - l2[c * 32 + e]);
        }
        tc_fence_before();
        mbar_arrive(&d_free[s]);
        const int key = i * 128 + r;
        if (shared_row && slots == 1 && j > 0) {
          const uint64_t need = static_cast<uint64_t>(j - 1) * nch + i + 1;
          if (seen < need && !wait_progress(progress, need, seen, p.status, abort_flag)) {
            ok = false;
            break;
          }
        }
        if (key < T) {
          if (shared_row) {
            st_global_hint(row + key, sum, pol);
          } else {
            row[key] = sum;
          }
        }
        warp_hist_add(hcur, mass_bin(ordered_key(sum)), key < T);
      }
      if (!ok) break;
      mbar_arrive(&lse_empty[j & 1]);
      mbar_arrive(&row_ready[j & 1]);  // releases this thread's row stores and histogram increments
    }
  } else {
    // ---------------------------------------------------------------- selection
    const int st = threadIdx.x - kSelWarp0 * 32;  // 0 .. kSelThreads-1
    const int k = p.k;
    for (int j = 0, t = blockIdx.x; t < tiles; ++j, t += gridDim.x) {
      const bool ok = mbar_wait(&row_ready[j & 1], (j >> 1) & 1, p.status, abort_flag);
      if (!Sel::all(ok)) break;
      const float *row = row_of(j, t);
      int32_t *dst = p.idx + static_cast<size_t>(t) * k;
      uint32_t *hrow = hist + (j & 1) * kBins;
      const uint64_t done_before = static_cast<uint64_t>(j) * nch;
      int read_end = 0;  // elements of a row buffer already read and released
      // Group-wide, after the first `end` elements of the row have been read for the last time: in a
      // row buffer, drops their lines from L2 (dead data is never written back) and publishes the
      // progress that lets the mass warps overwrite them.
      auto tile_done = [&](int end) {
        end = min(end, T);
        if (!shared_row || end <= read_end) return;
        const int64_t l1 = (static_cast<int64_t>(end) + 31) / 32;
        for (int64_t l = read_end / 32 + st; l < l1; l += kSelThreads) discard_l2_line(row + l * 32);
        Sel::sync();
        if (st == 0) {
          const uint64_t c = end >= T ? static_cast<uint64_t>(nch) : static_cast<uint64_t>(end / 128);
          st_release_shared(progress, done_before + c);
        }
        read_end = end;
      };
      if (k >= T) {
        for (int i = st; i < T; i += kSelThreads) dst[i] = i;
      } else if (k > 0) {
        Sel::select_digit(hrow, kBins, k, st, warp_tot, sel_res);
        const uint32_t bin = sel_res[0];
        const uint32_t n_cand = sel_res[1] + hrow[bin];
        const uint32_t lo = bin_floor(bin);
        Sel::sync();
        if (n_cand <= static_cast<uint32_t>(kCap)) {
          // one pass over the row: every key >= lo, in index order, into the candidate buffer
          const bool vec = (reinterpret_cast<uintptr_t>(row) & 15u) == 0;
          uint32_t count = 0;
          for (int base = 0; base < T; base += 4 * kSelThreads) {
            const int e0 = base + 4 * st;
            uint32_t key[4];
            if (vec && e0 + 3 < T) {
              const float4 f = *reinterpret_cast<const float4 *>(row + e0);
              key[0] = ordered_key(f.x);
              key[1] = ordered_key(f.y);
              key[2] = ordered_key(f.z);
              key[3] = ordered_key(f.w);
            } else {
#pragma unroll
              for (int c = 0; c < 4; ++c) key[c] = e0 + c < T ? ordered_key(row[e0 + c]) : 0u;
            }
            uint32_t cnt = 0;
#pragma unroll
            for (int c = 0; c < 4; ++c) cnt += (e0 + c < T && key[c] >= lo) ? 1u : 0u;
            uint64_t tot;
            uint32_t pos = count + static_cast<uint32_t>(Sel::excl_scan(cnt, st, warp_tot, tot));
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              if (e0 + c < T && key[c] >= lo) {
                if (pos < static_cast<uint32_t>(kCap)) {
                  ckey[pos] = key[c];
                  cidx[pos] = e0 + c;
                }
                ++pos;
              }
            }
            count += static_cast<uint32_t>(tot);
            tile_done(base + 4 * kSelThreads);
          }
          Sel::sync();
          const int nc = static_cast<int>(min(count, static_cast<uint32_t>(kCap)));
          int kk = min(k, nc);
          const uint32_t tau = Sel::radix_select([&](int i) { return ckey[i]; }, nc, kk, st, hrow, warp_tot, sel_res);
          Sel::compact([&](int i, uint32_t &key, int32_t &id) { key = ckey[i]; id = cidx[i]; }, nc, tau, kk, k, dst,
                       st, warp_tot, [](int) {});
        } else {
          // too many candidates: the exact select over the whole row, read again for each pass
          int kk = k;
          const uint32_t tau =
              Sel::radix_select([&](int i) { return ordered_key(row[i]); }, T, kk, st, hrow, warp_tot, sel_res);
          Sel::compact([&](int i, uint32_t &key, int32_t &id) { key = ordered_key(row[i]); id = i; }, T, tau, kk, k,
                       dst, st, warp_tot, tile_done);
        }
      }
      tile_done(T);
      // hand the histogram back zeroed
      for (int i = st; i < kBins; i += kSelThreads) hrow[i] = 0;
      Sel::sync();
      if (st == 0) mbar_arrive(&hist_free[j & 1]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 256);
}

}  // namespace

int64_t mass_grid(int64_t tiles) {
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return std::min<int64_t>(tiles, std::max(sms, 1));
}

int64_t mass_row_floats(int64_t T) { return mass_row_pad(T); }

int64_t mass_row_buffers(int64_t tiles, int64_t T) {
  const int64_t grid = mass_grid(tiles);
  return grid * mass_row_slots(grid, T);
}

cudaError_t launch_attn_mass_select(const MassParams &p, const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                                    cudaStream_t s) {
  if (p.h <= 0 || p.nb <= 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(attn_mass_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmem));
  if (e != cudaSuccess) return e;
  const int64_t grid = mass_grid(static_cast<int64_t>(p.h) * p.nb);
  attn_mass_select_kernel<<<static_cast<unsigned>(grid), kThreads, kSmem, s>>>(tm_q, tm_k, p);
  return cudaGetLastError();
}

}  // namespace cm
