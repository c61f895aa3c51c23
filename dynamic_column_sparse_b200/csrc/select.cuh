// select.cuh - building blocks of the exact per-row top-k: order-preserving
// keys, warp-aggregated histogram increments, and a radix select plus stable
// compaction run by a group of warps (a named barrier), so that a kernel can
// give selection to some of its warps while the others keep computing.
//
// Result rule: the k largest fp32 values of a row, ties to the lower index,
// written as ascending indices; -0 equals +0 and NaN orders by its bits.
#pragma once

#include <stdint.h>

namespace cm {

// fp32 -> uint32 whose unsigned order is the numeric order (-0 == +0).
__device__ __forceinline__ uint32_t ordered_key(float f) {
  uint32_t b = __float_as_uint(f);
  if (b == 0x80000000u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// One shared-memory increment of hist[bin] for every lane that has `active`
// set. When all active lanes of the warp share one bin (values that crowd into
// a few bins), a single atomic adds them all; otherwise each lane adds its own.
// Warp-collective: every lane of the warp must call it.
__device__ __forceinline__ void warp_hist_add(uint32_t *hist, uint32_t bin, bool active) {
  const unsigned am = __ballot_sync(0xffffffffu, active);
  if (am == 0u) return;
  const int leader = __ffs(am) - 1;
  const uint32_t lb = __shfl_sync(0xffffffffu, bin, leader);
  if (__all_sync(0xffffffffu, !active || bin == lb)) {
    if ((threadIdx.x & 31) == static_cast<unsigned>(leader)) atomicAdd(&hist[lb], static_cast<uint32_t>(__popc(am)));
  } else if (active) {
    atomicAdd(&hist[bin], 1u);
  }
}

// A group of NT threads (whole warps) that synchronise on named barrier BAR.
// `t` is the thread's index within the group. Every member must make every
// call; decisions that steer a member past a barrier go through all().
template <int NT, int BAR>
struct SelGroup {
  static_assert(NT % 32 == 0 && NT >= 64 && NT <= 1024, "whole warps");
  static constexpr int kWarps = NT / 32;
  static constexpr int kItems = 8;  // consecutive elements per thread in a compaction tile

  __device__ static void sync() { asm volatile("bar.sync %0, %1;" ::"n"(BAR), "n"(NT) : "memory"); }

  // True on every member iff v is true on every member.
  __device__ static bool all(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(v ? 1u : 0u), "n"(BAR), "n"(NT)
        : "memory");
    return r != 0;
  }

  // Exclusive scan of v over the group in member order; total = the sum.
  // warp_tot: kWarps + 1 words of shared memory.
  __device__ static uint64_t excl_scan(uint64_t v, int t, uint64_t *warp_tot, uint64_t &total) {
    const int lane = t & 31, w = t >> 5;
    uint64_t inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint64_t u = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += u;
    }
    if (lane == 31) warp_tot[w] = inc;
    sync();
    if (w == 0) {
      const uint64_t x = lane < kWarps ? warp_tot[lane] : 0;
      uint64_t xi = x;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint64_t u = __shfl_up_sync(0xffffffffu, xi, o);
        if (lane >= o) xi += u;
      }
      if (lane < kWarps) warp_tot[lane] = xi - x;
      if (lane == kWarps - 1) warp_tot[kWarps] = xi;
    }
    sync();
    const uint64_t res = warp_tot[w] + inc - v;
    total = warp_tot[kWarps];
    sync();
    return res;
  }

  // Given the histogram of one digit of the keys still in play (nbins a
  // multiple of NT) and the number kk >= 1 of keys still to take, the digit of
  // the kk-th largest key (res[0]) and how many keys lie in higher digits
  // (res[1]). res lives in shared memory; all members read it after return.
  __device__ static void select_digit(const uint32_t *hist, int nbins, int kk, int t, uint64_t *warp_tot,
                                      uint32_t *res) {
    const int per = nbins / NT;
    const int hi = nbins - t * per;  // member t owns bins [hi - per, hi): member 0 the highest
    uint32_t local = 0;
    for (int b = hi - 1; b >= hi - per; --b) local += hist[b];
    if (t == 0) res[0] = res[1] = 0;
    uint64_t tot;
    const uint32_t above = static_cast<uint32_t>(excl_scan(local, t, warp_tot, tot));
    if (above < static_cast<uint32_t>(kk) && above + local >= static_cast<uint32_t>(kk)) {
      uint32_t cum = above;
      for (int b = hi - 1; b >= hi - per; --b) {
        if (cum + hist[b] >= static_cast<uint32_t>(kk)) {
          res[0] = static_cast<uint32_t>(b);
          res[1] = cum;
          break;
        }
        cum += hist[b];
      }
    }
    sync();
  }

  // Three radix passes (11 + 11 + 10 bits) over the keys key_at(i), i < count,
  // that find the kk-th largest key. Returns it; kk becomes the number of keys
  // equal to it that are taken. hist: 2048 words of shared memory.
  template <typename KeyAt>
  __device__ static uint32_t radix_select(KeyAt key_at, int count, int &kk, int t, uint32_t *hist, uint64_t *warp_tot,
                                          uint32_t *res) {
    const int lane = t & 31, w = t >> 5;
    uint32_t prefix = 0, mask = 0;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
      const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
      const int nbins = pass == 2 ? 1024 : 2048;
      for (int i = t; i < nbins; i += NT) hist[i] = 0;
      sync();
      for (int b0 = w * 32; b0 < count; b0 += NT) {  // warp-uniform
        const int i = b0 + lane;
        const uint32_t key = i < count ? key_at(i) : 0u;
        warp_hist_add(hist, (key >> shift) & static_cast<uint32_t>(nbins - 1), i < count && (key & mask) == prefix);
      }
      sync();
      select_digit(hist, nbins, kk, t, warp_tot, res);
      prefix |= res[0] << shift;
      mask |= static_cast<uint32_t>(nbins - 1) << shift;
      kk -= static_cast<int>(res[1]);
      sync();
    }
    return prefix;
  }

  // Stable compaction over elements 0 .. count-1 in index order: an element is
  // kept if its key exceeds tau, or equals tau and fewer than kk equal keys
  // precede it. load(i, key, id) gives element i's key and output value;
  // after each tile of NT * kItems elements, tile_done(end) is called by every
  // member (end = elements read so far). Writes dst[0 .. k).
  template <typename Load, typename TileDone>
  __device__ static void compact(Load load, int count, uint32_t tau, int kk, int k, int32_t *dst, int t,
                                 uint64_t *warp_tot, TileDone tile_done) {
    uint32_t run_gt = 0, run_eq = 0;
    for (int base = 0; base < count; base += NT * kItems) {
      const int first = base + t * kItems;
      uint32_t keys[kItems];
      int32_t ids[kItems];
      uint32_t n_gt = 0, n_eq = 0;
#pragma unroll
      for (int e = 0; e < kItems; ++e) {
        keys[e] = 0u;
        ids[e] = 0;
        if (first + e < count) {
          load(first + e, keys[e], ids[e]);
          n_gt += keys[e] > tau;
          n_eq += keys[e] == tau;
        }
      }
      uint64_t tot;
      const uint64_t before = excl_scan((static_cast<uint64_t>(n_gt) << 32) | n_eq, t, warp_tot, tot);
      uint32_t gt_b = run_gt + static_cast<uint32_t>(before >> 32);
      uint32_t eq_b = run_eq + static_cast<uint32_t>(before & 0xffffffffu);
#pragma unroll
      for (int e = 0; e < kItems; ++e) {
        if (first + e >= count) break;
        if (keys[e] > tau) {
          const uint32_t pos = gt_b + min(eq_b, static_cast<uint32_t>(kk));
          if (pos < static_cast<uint32_t>(k)) dst[pos] = ids[e];
          ++gt_b;
        } else if (keys[e] == tau) {
          if (eq_b < static_cast<uint32_t>(kk) && gt_b + eq_b < static_cast<uint32_t>(k)) dst[gt_b + eq_b] = ids[e];
          ++eq_b;
        }
      }
      run_gt += static_cast<uint32_t>(tot >> 32);
      run_eq += static_cast<uint32_t>(tot & 0xffffffffu);
      tile_done(min(base + NT * kItems, count));
    }
  }
};

}  // namespace cm
