// topk.cu - per-row top-k column selection (the sparsity identification step).
//
// For each row: the k largest fp32 scores, ties to the lower index, written as
// ascending column indices. Scores become order-preserving uint32 keys; a
// radix select finds the exact k-th key tau and how many keys equal to tau are
// taken; a stable block-wide compaction in index order then writes the result.
//
// Rows of up to kStagedMaxN scores are staged in shared memory once and run a
// three-pass radix select (11 + 11 + 10 bits) there. Longer rows (two in
// flight per SM) first try a sampled threshold: every stride-th float4 of the
// row is read, two radix passes find the top 22 bits of the r-th largest
// sampled key, r set about three standard deviations above the sample's
// expected share of the k largest, and one vectorised pass over the row copies
// every key at or above that (key and index, in index order) into shared memory, each warp appending
// its own segment of the row to its own region; the exact k-th key and the
// output come from the candidates there. If the sample misjudged the row (too
// few or too many candidates), a 12-bit histogram of the whole row finds the
// bucket holding the k-th key and the keys in it or above become the
// candidates. If one warp's region overflows while the row's candidates still
// fit, the regions are laid end to end after a counting pass. A row whose
// candidates do not fit at all, or that is not 16-byte aligned, falls back to
// the general path that re-reads the row from global memory for every radix
// pass. The radix passes over the candidates walk the warps' regions as they
// lie (they need every candidate, in any order); the compaction, which needs
// index order, finds each thread's region once and walks forwards. A warp
// whose active lanes all fall in one histogram bin (scores that crowd into a
// few bins) adds them with one shared-memory atomic.
#include "kernels.cuh"
#include "ptx.cuh"
#include "select.cuh"

namespace cm {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxBins = 2048;
constexpr int kItems = 8;             // consecutive elements per thread in the compaction
constexpr int kStagedMaxN = 40960;    // 160 KB of keys in shared memory
constexpr int kLongBins = 4096;       // first digit of the long-row path: the top 12 key bits
constexpr int kLongCap = 12288;       // long-row candidates held in shared memory (96 KB: two CTAs per SM)
constexpr int kSampleMaxK = 9216;     // the sampled-threshold path serves k up to 3/4 of the candidate buffer

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

// Given the histogram of the digit of the keys still in play and the number kk
// of keys still to take, finds the digit of the kk-th largest key (s_digit)
// and how many keys lie in higher digits (s_above). Block-wide.
__device__ __forceinline__ void select_digit(const uint32_t *hist, int nbins, int kk, uint64_t *warp_tot,
                                             uint32_t &s_digit, uint32_t &s_above) {
  const int tid = threadIdx.x;
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
}

// One tile of the stable compaction: thread t holds the keys of elements
// first .. first + kItems - 1 (of n). An element is kept if its key exceeds
// tau, or equals tau and fewer than kk equal keys precede it; out(pos, e)
// writes output position pos for the thread's item e (element first + e).
template <typename Out>
__device__ __forceinline__ void compact_tile(const uint32_t *keys, int first, int n, uint32_t tau, int kk, int k,
                                             uint32_t &run_gt, uint32_t &run_eq, uint64_t *warp_tot, Out out) {
  uint32_t n_gt = 0, n_eq = 0;
#pragma unroll
  for (int e = 0; e < kItems; ++e) {
    if (first + e < n) {
      n_gt += keys[e] > tau;
      n_eq += keys[e] == tau;
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
      if (pos < static_cast<uint32_t>(k)) out(pos, e);
      ++gt_b;
    } else if (keys[e] == tau) {
      if (eq_b < static_cast<uint32_t>(kk) && gt_b + eq_b < static_cast<uint32_t>(k)) out(gt_b + eq_b, e);
      ++eq_b;
    }
  }
  run_gt += static_cast<uint32_t>(tot >> 32);
  run_eq += static_cast<uint32_t>(tot & 0xffffffffu);
}

// Exact top-k of one row by a three-pass radix select over all n keys (read
// from `staged` shared memory or, if STAGED is false, from global memory on
// every pass), then a stable compaction.
template <bool STAGED>
__device__ void row_generic(const float *src, int32_t *dst, int n, int k, const uint32_t *staged, uint32_t *hist,
                            uint64_t *warp_tot, uint32_t &s_digit, uint32_t &s_above) {
  const int tid = threadIdx.x;
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
    select_digit(hist, nbins, kk, warp_tot, s_digit, s_above);
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
#pragma unroll
    for (int e = 0; e < kItems; ++e) {
      const int i = first + e;
      keys[e] = i < n ? (STAGED ? staged[i] : ordered_key(__ldg(src + i))) : 0u;
    }
    compact_tile(keys, first, n, tau, kk, k, run_gt, run_eq, warp_tot, [&](uint32_t pos, int e) { dst[pos] = first + e; });
  }
  __syncthreads();
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
    row_generic<STAGED>(src, dst, n, k, staged, hist, warp_tot, s_digit, s_above);
  }
}

// Long rows (see the file comment). Dynamic shared memory holds the candidate
// keys and indices: kLongCap entries each, split into one region per warp.
__global__ void __launch_bounds__(kThreads) topk_long_kernel(const TopkParams p) {
  extern __shared__ uint32_t cand[];  // [kLongCap] keys, then [kLongCap] indices
  __shared__ uint32_t hist[kLongBins];
  __shared__ uint64_t warp_tot[kWarps + 1];
  __shared__ uint32_t s_digit, s_above;
  __shared__ uint32_t s_pref[kWarps + 1];  // start of warp w's candidates in the concatenated order
  __shared__ uint32_t s_base[kWarps];      // where warp w's candidates sit in the buffer
  __shared__ int s_overflow;
  constexpr int kRegion = kLongCap / kWarps;
  constexpr int kUnroll = 8;
  uint32_t *ckey = cand;
  int32_t *cidx = reinterpret_cast<int32_t *>(cand + kLongCap);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = static_cast<int>(p.n);
  const int k = p.k;
  if (*(volatile int *)p.status != kDevOk) return;

  for (int64_t row = blockIdx.x; row < p.rows; row += gridDim.x) {
    const float *src = p.scores + row * p.ld_scores;
    int32_t *dst = p.idx + row * p.ld_idx;
    if (k >= n) {
      for (int i = tid; i < n; i += kThreads) dst[i] = i;
      continue;
    }
    if ((reinterpret_cast<uintptr_t>(src) & 15u) != 0) {
      row_generic<false>(src, dst, n, k, nullptr, hist, warp_tot, s_digit, s_above);
      continue;
    }
    const float4 *src4 = reinterpret_cast<const float4 *>(src);
    const int n4 = n >> 2;
    // Warp w takes float4 elements [w seg, (w+1) seg) (the last warp also the
    // < 4 trailing scalars) and appends every key >= lo, with its index, in
    // index order, to its own region of the buffer (region w at s_base[w]). If a
    // region overflows, every warp counts its candidates first, and if they fit
    // the regions are laid end to end and the segments are read a second time.
    // Returns false (block-uniform) if the candidates do not fit at all.
    const int seg = (n4 + kWarps - 1) / kWarps;
    const int f_lo = min(warp * seg, n4), f_hi = min(f_lo + seg, n4);
    // one pass over this warp's segment: counts (write false) or appends into
    // wkey / widx up to cap entries; returns the count, sets over past cap
    auto scan_segment = [&](uint32_t lo, bool write, uint32_t *wkey, int32_t *widx, uint32_t cap,
                            bool &over) -> uint32_t {
      uint32_t wcount = 0;
      over = false;
      // this lane's flagged keys of one step (up to 4, elements base..base+3), in lane order
      auto append = [&](const uint32_t *key, int base, int nvalid) {
        uint32_t flags = 0, cnt = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (c < nvalid && key[c] >= lo) {
            flags |= 1u << c;
            ++cnt;
          }
        uint32_t incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        const uint32_t tot = __shfl_sync(0xffffffffu, incl, 31);
        if (write) {
          if (wcount + tot > cap) {
            over = true;  // warp-uniform
            return;
          }
          uint32_t pos = wcount + incl - cnt;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            if (flags & (1u << c)) {
              wkey[pos] = key[c];
              widx[pos] = base + c;
              ++pos;
            }
        }
        wcount += tot;
      };
      for (int f0 = f_lo; f0 < f_hi && !over; f0 += kUnroll * 32) {
        float4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int f = f0 + u * 32 + lane;
          v[u] = f < f_hi ? __ldg(src4 + f) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          if (over || f0 + u * 32 >= f_hi) break;  // warp-uniform
          const int f = f0 + u * 32 + lane;
          const uint32_t key[4] = {ordered_key(v[u].x), ordered_key(v[u].y), ordered_key(v[u].z), ordered_key(v[u].w)};
          append(key, 4 * f, f < f_hi ? 4 : 0);
        }
      }
      if (warp == kWarps - 1 && !over && 4 * n4 < n) {
        // the (at most 3) trailing scalars, all on lane 0
        const int nt = n - 4 * n4;
        uint32_t key[4] = {0u, 0u, 0u, 0u};
        if (lane == 0)
          for (int c = 0; c < nt; ++c) key[c] = ordered_key(__ldg(src + 4 * n4 + c));
        append(key, 4 * n4, lane == 0 ? nt : 0);
      }
      return wcount;
    };
    auto gather_candidates = [&](uint32_t lo) -> bool {
      if (tid == 0) s_overflow = 0;
      __syncthreads();
      bool over;
      uint32_t wc = scan_segment(lo, true, ckey + warp * kRegion, cidx + warp * kRegion, kRegion, over);
      if (lane == 0) {
        warp_tot[warp] = wc;
        if (over) s_overflow = 1;
      }
      __syncthreads();
      const bool contiguous = s_overflow != 0;
      if (contiguous) {
        wc = scan_segment(lo, false, nullptr, nullptr, 0, over);
        if (lane == 0) warp_tot[warp] = wc;
        __syncthreads();
      }
      if (tid == 0) {
        uint32_t acc = 0;
        for (int w = 0; w < kWarps; ++w) {
          s_pref[w] = acc;
          s_base[w] = contiguous ? acc : static_cast<uint32_t>(w * kRegion);
          acc += static_cast<uint32_t>(warp_tot[w]);
        }
        s_pref[kWarps] = acc;
      }
      __syncthreads();
      if (s_pref[kWarps] > static_cast<uint32_t>(kLongCap)) return false;
      if (contiguous) {
        // the counts add up to at most kLongCap, so the regions laid end to end fit
        scan_segment(lo, true, ckey + s_base[warp], cidx + s_base[warp], static_cast<uint32_t>(kLongCap), over);
        __syncthreads();
      }
      return true;
    };
    // candidate L of the concatenated (index-ordered) list lies in region
    // cand_w(L), which holds candidates s_pref[w] .. s_pref[w+1]-1 from s_base[w] on
    auto cand_w = [&](int L) -> int {
      int w = 0;
#pragma unroll
      for (int step = kWarps / 2; step >= 1; step >>= 1)
        if (static_cast<uint32_t>(L) >= s_pref[w + step]) w += step;
      return w;
    };
    // whether buffer slot j holds a candidate (the radix passes need every
    // candidate, in any order, so they walk the buffer itself)
    auto slot_valid = [&](int j) -> bool {
      if (s_base[kWarps - 1] == s_pref[kWarps - 1]) return j < static_cast<int>(s_pref[kWarps]);  // laid end to end
      const int w = j / kRegion;
      return j - w * kRegion < static_cast<int>(s_pref[w + 1] - s_pref[w]);
    };
    // radix passes over the first `count` keys of `keys` (or, with keys null,
    // over the candidates): from (prefix, mask, kk), the digits of passes
    // p0 .. p1 - 1 of (21: 11 bits, 10: 11 bits, 0: 10 bits)
    auto radix_select = [&](const uint32_t *keys, int count, uint32_t &prefix, uint32_t &mask, int &kk, int p0,
                            int p1) {
#pragma unroll 1
      for (int pass = p0; pass < p1; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const int nbins = pass == 2 ? 1024 : 2048;
        for (int i = tid; i < nbins; i += kThreads) hist[i] = 0;
        __syncthreads();
        const int span = keys ? count : kLongCap;
        for (int b0 = warp * 32; b0 < span; b0 += kThreads) {   // warp-uniform
          const int L = b0 + lane;
          const bool valid = L < span && (keys ? true : slot_valid(L));
          const uint32_t key = valid ? (keys ? keys[L] : ckey[L]) : 0u;
          warp_hist_add(hist, (key >> shift) & static_cast<uint32_t>(nbins - 1), valid && (key & mask) == prefix);
        }
        __syncthreads();
        select_digit(hist, nbins, kk, warp_tot, s_digit, s_above);
        prefix |= s_digit << shift;
        mask |= static_cast<uint32_t>(nbins - 1) << shift;
        kk -= static_cast<int>(s_above);
        __syncthreads();
      }
    };
    // stable compaction over the candidates in index order
    auto compact_candidates = [&](uint32_t tau, int kk) {
      const int count = static_cast<int>(s_pref[kWarps]);
      uint32_t run_gt = 0, run_eq = 0;
      const int tile = kThreads * kItems;
      for (int base = 0; base < count; base += tile) {
        const int first = base + tid * kItems;
        uint32_t keys[kItems];
        int32_t ids[kItems];
        int w = first < count ? cand_w(first) : 0;   // found once, then walked forwards
#pragma unroll
        for (int e = 0; e < kItems; ++e) {
          keys[e] = 0u;
          ids[e] = 0;
          const int L = first + e;
          if (L < count) {
            while (static_cast<uint32_t>(L) >= s_pref[w + 1]) ++w;
            const int j = static_cast<int>(s_base[w]) + (L - static_cast<int>(s_pref[w]));
            keys[e] = ckey[j];
            ids[e] = cidx[j];
          }
        }
        compact_tile(keys, first, count, tau, kk, k, run_gt, run_eq, warp_tot,
                     [&](uint32_t pos, int e) { dst[pos] = ids[e]; });
      }
      __syncthreads();
    };

    // Path 1: a threshold from a sample. Every stride-th float4 of the row is
    // read and the r-th largest sampled key is taken as the lower bound of the
    // candidates, r chosen so that about k + 3 standard deviations of the
    // sample lie above the row's k-th key; then the row is read once.
    bool done = false;
    if (k <= kSampleMaxK && n4 >= 64) {
      const int stride = max(16, (4 * n4 + kLongCap - 1) / kLongCap);
      const int ns = min((n4 + stride - 1) / stride, kLongCap / 4);
      const int m = 4 * ns;
      for (int i = tid; i < ns; i += kThreads) {
        const float4 v = __ldg(src4 + static_cast<size_t>(i) * stride);
        ckey[4 * i] = ordered_key(v.x);
        ckey[4 * i + 1] = ordered_key(v.y);
        ckey[4 * i + 2] = ordered_key(v.z);
        ckey[4 * i + 3] = ordered_key(v.w);
      }
      __syncthreads();
      const float expect = static_cast<float>(k) * static_cast<float>(m) / static_cast<float>(n);
      const int r = min(m, static_cast<int>(ceilf(expect + 3.f * sqrtf(expect))) + 8);
      uint32_t prefix = 0, mask = 0;
      int rr = r;
      radix_select(ckey, m, prefix, mask, rr, 0, 2);
      const uint32_t lo = prefix;   // the top 22 bits of the r-th largest sampled key (the rest zero)
      if (gather_candidates(lo) && s_pref[kWarps] >= static_cast<uint32_t>(k)) {
        uint32_t tau = 0, tmask = 0;
        int kk = k;
        radix_select(nullptr, static_cast<int>(s_pref[kWarps]), tau, tmask, kk, 0, 3);
        compact_candidates(tau, kk);
        done = true;
      }
    }
    if (done) continue;

    // Path 2: a 12-bit histogram of every key finds the bucket holding the
    // k-th key; the keys in it or above are the candidates.
    for (int i = tid; i < kLongBins; i += kThreads) hist[i] = 0;
    __syncthreads();
    for (int base = warp * 32; base < n4; base += kUnroll * kThreads) {   // warp-uniform
      float4 v[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int i = base + lane + u * kThreads;
        v[u] = i < n4 ? __ldg(src4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const bool valid = base + lane + u * kThreads < n4;
        warp_hist_add(hist, ordered_key(v[u].x) >> 20, valid);
        warp_hist_add(hist, ordered_key(v[u].y) >> 20, valid);
        warp_hist_add(hist, ordered_key(v[u].z) >> 20, valid);
        warp_hist_add(hist, ordered_key(v[u].w) >> 20, valid);
      }
    }
    if (warp == 0) {
      const int i = 4 * n4 + lane;
      warp_hist_add(hist, i < n ? ordered_key(__ldg(src + i)) >> 20 : 0u, i < n);
    }
    __syncthreads();
    select_digit(hist, kLongBins, k, warp_tot, s_digit, s_above);
    const uint32_t b1 = s_digit;
    const int kk1 = k - static_cast<int>(s_above);   // keys to take from bucket b1
    const uint32_t n_cand = s_above + hist[b1];       // keys in bucket b1 or above
    __syncthreads();
    if (n_cand > static_cast<uint32_t>(kLongCap) || !gather_candidates(b1 << 20)) {
      row_generic<false>(src, dst, n, k, nullptr, hist, warp_tot, s_digit, s_above);
      continue;
    }
    // the remaining 20 bits (10 + 10) among the candidates of bucket b1
    uint32_t prefix = b1 << 20, mask = 0xfff00000u;
    int kk = kk1;
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
      const int shift = pass == 0 ? 10 : 0;
      for (int i = tid; i < 1024; i += kThreads) hist[i] = 0;
      __syncthreads();
      for (int b0 = warp * 32; b0 < kLongCap; b0 += kThreads) {   // warp-uniform
        const int L = b0 + lane;
        const bool valid = slot_valid(L);
        const uint32_t key = valid ? ckey[L] : 0u;
        warp_hist_add(hist, (key >> shift) & 1023u, valid && (key & mask) == prefix);
      }
      __syncthreads();
      select_digit(hist, 1024, kk, warp_tot, s_digit, s_above);
      prefix |= s_digit << shift;
      mask |= 1023u << shift;
      kk -= static_cast<int>(s_above);
      __syncthreads();
    }
    compact_candidates(prefix, kk);
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
    // rows being scanned (two per SM) stay resident in L2 between the two passes
    const int smem = 2 * kLongCap * static_cast<int>(sizeof(uint32_t));
    static bool long_attr_set = false;
    if (!long_attr_set) {
      cudaError_t e = cudaFuncSetAttribute(topk_long_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      long_attr_set = true;
    }
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, topk_long_kernel, kThreads, smem);
    const int64_t grid = std::min<int64_t>(p.rows, static_cast<int64_t>(sms) * std::max(per_sm, 1));
    topk_long_kernel<<<static_cast<unsigned>(grid), kThreads, smem, s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace cm
