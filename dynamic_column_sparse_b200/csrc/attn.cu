// attn.cu - attention over a gathered key subset with an online-softmax merge,
// plus the dense passes of the refresh (full attention with row log-sum-exp,
// complement partial; the attention mass and its top-k are in mass.cu).
//
// Persistent CTAs walk (head, 128-query block) tiles. Q arrives once per tile
// by a tiled TMA load; K and V stream in chunks of 128 keys through two-stage
// rings, K one chunk ahead of V: on a sparse step producer warps 9-15 gather
// the selected key rows with 16-byte cp.async (one warp instruction = two
// whole 256-byte key rows), on the dense passes one thread issues tiled TMA
// loads. Warp 8 issues the tcgen05 MMAs: S = Q K^T into one of two TMEM
// buffers, then O += P V with P read from TMEM and V from shared memory.
// Warps 0-7 run the online softmax, two warps per TMEM lane quadrant (32
// query rows), each on one 64-key half of S: they exchange their halves'
// maxima for the row maximum, exponentiate their half into P (bf16 pairs stored into one of
// two TMEM buffers with tcgen05.st) and rescale O in TMEM only when the row
// maximum grows by more than 2^8. S of chunk i+1 is computed while the
// softmax of chunk i runs. Logits are kept in log2 units (scale * log2 e).
#include <algorithm>

#include "kernels.cuh"
#include "ptx.cuh"

namespace cm {
namespace {

constexpr int kThreads = 512;
constexpr int kSoftmaxThreads = 256;   // warps 0-7: two warps per TMEM lane quadrant, one per half of the columns
constexpr int kMmaWarp = 8;
constexpr int kProdWarp0 = 9;          // warps 9-15
constexpr int kProducers = 224;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr uint32_t kTileBytes = 32768;   // one 128 x 128 bf16 operand tile (two 64-column swizzle halves)
constexpr float kRescaleLog2 = 8.0f;     // O and l are rescaled only when the row max grows by more than 2^8

// Shared memory: Q | K[2] | V[2] | barriers | key-index ring [4][128] |
// row-sum exchange [2][2][128] | row-maximum exchange [2][2][128] | key mask
// (complement pass) or merge buffers (delta pass).
struct AttnCfg {
  static constexpr uint32_t kQOff = 0;
  static constexpr uint32_t kKOff = kTileBytes;
  static constexpr uint32_t kVOff = kKOff + 2 * kTileBytes;
  static constexpr uint32_t kBarOff = kVOff + 2 * kTileBytes;
  static constexpr uint32_t kIdxOff = kBarOff + 256;
  static constexpr uint32_t kXsumOff = kIdxOff + 4 * 128 * 4;
  static constexpr uint32_t kXmaxOff = kXsumOff + 2 * 2 * 128 * 4;
  static constexpr uint32_t kMaskOff = kXmaxOff + 2 * 2 * 128 * 4;
};

__device__ __forceinline__ bool wait_warp(uint64_t *bar, uint32_t parity, int *status, volatile int *abort_flag) {
  const bool ok = mbar_wait(bar, parity, status, abort_flag);
  return __all_sync(0xffffffffu, ok);
}


// Persistent: each CTA walks tiles blockIdx.x, blockIdx.x + gridDim.x, ...,
// tile t = head * nb + query block (head-major, so the CTAs running at the
// same time gather from one head's keys and values, which stay in L2 even
// when all heads' do not); every tile has the same number of key chunks,
// so all roles index chunks by one running counter g.
template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using C = AttnCfg;
  constexpr uint32_t kIdescQK = idesc_bf16(128, 128, false, false);
  constexpr uint32_t kIdescPV = idesc_bf16(128, 128, false, true);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align_up<1024>(smem_raw);
  uint8_t *sQ = smem + C::kQOff;
  uint8_t *sK = smem + C::kKOff;
  uint8_t *sV = smem + C::kVOff;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
  uint64_t *q_full = bars + 0;
  uint64_t *q_empty = bars + 1;
  uint64_t *k_full = bars + 2;     // [2]
  uint64_t *v_full = bars + 4;     // [2]
  uint64_t *k_empty = bars + 6;    // [2] released when S = Q K^T of the stage has been computed
  uint64_t *v_empty = bars + 8;    // [2] released when P V of the stage has been computed
  uint64_t *s_full = bars + 10;    // [2]
  uint64_t *s_empty = bars + 12;   // [2]
  uint64_t *o_full = bars + 14;    // the last P V of the tile has landed in O
  uint64_t *o_empty = bars + 15;   // the tile's epilogue has read O
  uint64_t *p_full = bars + 16;    // [2] P of a chunk is in TMEM
  uint64_t *p_empty = bars + 18;   // [2] P V of that chunk has been computed
  uint64_t *pair_bar = bars + 20;  // [4]: the two softmax warps of a lane quadrant exchange row partials
  uint64_t *mask_bar = bars + 25;  // softmax warps: complement mask steps
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 26);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  uint64_t *qt_full = bars + 27;   // [2] Q of a tile is in TMEM buffer tile & 1
  uint64_t *qt_empty = bars + 29;  // [2] the last S = Q K^T of the tile two back has read that buffer
  int *kidx = reinterpret_cast<int *>(smem + C::kIdxOff);        // [4][128] selected keys of chunk g at g & 3
  float *xsum = reinterpret_cast<float *>(smem + C::kXsumOff);   // [2][2][128] partial row sums
  float *xmax = reinterpret_cast<float *>(smem + C::kXmaxOff);   // [2][2][128] partial row maxima by chunk parity
  uint32_t *mask = reinterpret_cast<uint32_t *>(smem + C::kMaskOff);
  float *ebuf = reinterpret_cast<float *>(smem + C::kMaskOff);      // delta pass: [8 warps][32][36] merge buffer

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (*(volatile int *)p.status != kDevOk) return;
  const int T = p.T;
  const int ntiles = p.h * p.nb;
  const int nkeys = MODE == kAttnDelta ? p.k : T;
  const int nchunks = (nkeys + 127) / 128;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, kSoftmaxThreads);   // the softmax warps have copied Q into TMEM
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], MODE == kAttnDelta ? kProducers : 1);
      mbar_init(&v_full[s], MODE == kAttnDelta ? kProducers : 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], kSoftmaxThreads);
      mbar_init(&p_full[s], kSoftmaxThreads);
      mbar_init(&p_empty[s], 1);
    }
    mbar_init(o_full, 1);
    mbar_init(o_empty, kSoftmaxThreads);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&qt_full[s], kSoftmaxThreads);
      mbar_init(&qt_empty[s], 1);
    }
    for (int qd = 0; qd < 4; ++qd) mbar_init(&pair_bar[qd], 64);
    mbar_init(mask_bar, kSoftmaxThreads);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kProdWarp0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // TMEM columns: S[0] at 0, S[1] at 128 (P of a chunk, bf16 pairs, overwrites the first 64 columns of
  // its S buffer), O at 256, Q[0] at 384, Q[1] at 448 (bf16 pairs: the A operand of S = Q K^T)
  const uint32_t tmem = *tmem_slot;

  if (warp >= kProdWarp0) {
    // ------------------------------------------------------------ producers
    // Loads in the order the MMA warp consumes them: per tile Q, K0, K1, V0,
    // K2, V1, .., K(n-1), V(n-2), V(n-1). A K stage frees as soon as its
    // S = Q K^T is done, a V stage only after its P V, so K runs one chunk
    // ahead of V; the last V of a tile goes out before the next tile's loads.
    // g counts chunks over this CTA's tiles.
    const int pw = warp - kProdWarp0;
    const int my_tiles = static_cast<int>(blockIdx.x) < ntiles ? (ntiles - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1 : 0;
    const int total = my_tiles * nchunks;
    // warp pw moves rows 20 pw .. 20 pw + 19 (< 128) of every chunk and
    // stages their selected keys itself (lane l: row 20 pw + l), so the
    // producer warps never wait for one another
    constexpr int kRowsPerWarp = 20;
    const int krow = pw * kRowsPerWarp + lane;
    const bool kload = lane < kRowsPerWarp && krow < 128;
    auto load_keys = [&](int g, int &ka) {
      const int tile = blockIdx.x + (g / nchunks) * gridDim.x, i = g % nchunks;
      const int hh = tile / p.nb, b = tile % p.nb;
      const int32_t *irow = p.idx + (static_cast<size_t>(hh) * p.nb + b) * p.k;
      ka = kload ? __ldg(irow + min(i * 128 + krow, p.k - 1)) : 0;
    };
    // the row pairs (2q, 2q+1), q = 10 pw .. 10 pw + 9 (< 64): lanes 0-15 the
    // even row, 16-31 the odd one, 16 bytes each. The keys are read from
    // shared memory up front, so the copies issue back to back with one
    // address computation each.
    auto gather = [&](const uint16_t *src, uint8_t *dst, const int *ks, int hh) {
      constexpr int kPairs = kRowsPerWarp / 2;
      const int c16 = lane & 15, hi = lane >> 4;
      const uint16_t *lb = src + hh * 128 + c16 * 8;
      const size_t rs = static_cast<size_t>(p.h) * 128;
      const uint32_t d0 = smem_u32(dst) + (c16 >> 3) * 16384;
      const int q0 = pw * kPairs;
      int key[kPairs];
#pragma unroll
      for (int i = 0; i < kPairs; ++i) key[i] = q0 + i < 64 ? ks[2 * (q0 + i) + hi] : 0;
#pragma unroll
      for (int i = 0; i < kPairs; ++i) {
        if (q0 + i < 64) {
          const int r = 2 * (q0 + i) + hi;
          cp_async_16(d0 + sw128_offset(r, c16 & 7), lb + static_cast<size_t>(key[i]) * rs);
        }
      }
    };
    int ka = 0;
    if (MODE == kAttnDelta && total > 0) load_keys(0, ka);
    // K of chunk g (i = its index in the tile), for the tile's head / block
    auto load_k = [&](int g, int i, int hh) -> bool {
      const int s = g & 1;
      if (!wait_warp(&k_empty[s], ((g >> 1) & 1) ^ 1, p.status, abort_flag)) return false;
      if (MODE == kAttnDelta) {
        // stage the chunk's keys in slot g & 3 (read again for V two loads
        // later), range-checked, then fetch the next chunk's while the copies go out
        if (static_cast<unsigned>(ka) >= static_cast<unsigned>(T)) {
          atomicCAS(p.status, kDevOk, kDevBadIndex);
          ka = 0;
        }
        int *ks = kidx + (g & 3) * 128;
        if (kload) ks[krow] = ka;
        __syncwarp();
        if (g + 1 < total) load_keys(g + 1, ka);
        gather(p.k_ptr, sK + s * kTileBytes, ks, hh);
        cp_async_arrive_noinc(&k_full[s]);
      } else if (pw == 0 && lane == 0) {
        mbar_arrive_expect_tx(&k_full[s], kTileBytes);
        tma_load_2d(sK + s * kTileBytes, &tm_k, &k_full[s], hh * 128, i * 128);
        tma_load_2d(sK + s * kTileBytes + 16384, &tm_k, &k_full[s], hh * 128 + 64, i * 128);
      }
      __syncwarp();
      return true;
    };
    auto load_v = [&](int g, int i, int hh) -> bool {
      const int s = g & 1;
      if (!wait_warp(&v_empty[s], ((g >> 1) & 1) ^ 1, p.status, abort_flag)) return false;
      if (MODE == kAttnDelta) {
        gather(p.v_ptr, sV + s * kTileBytes, kidx + (g & 3) * 128, hh);
        cp_async_arrive_noinc(&v_full[s]);
      } else if (pw == 0 && lane == 0) {
        mbar_arrive_expect_tx(&v_full[s], kTileBytes);
        tma_load_2d(sV + s * kTileBytes, &tm_v, &v_full[s], hh * 128, i * 128);
        tma_load_2d(sV + s * kTileBytes + 16384, &tm_v, &v_full[s], hh * 128 + 64, i * 128);
      }
      __syncwarp();
      return true;
    };
    bool ok = true;
    int g0 = 0;
    for (int tl = 0; tl < my_tiles && ok && nchunks > 0; ++tl, g0 += nchunks) {
      const int tile = blockIdx.x + tl * gridDim.x;
      const int hh = tile / p.nb, b = tile % p.nb;
      if (pw == 0) {
        if (!wait_warp(q_empty, (tl & 1) ^ 1, p.status, abort_flag)) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(q_full, kTileBytes);
          tma_load_2d(sQ, &tm_q, q_full, hh * 128, b * 128);
          tma_load_2d(sQ + 16384, &tm_q, q_full, hh * 128 + 64, b * 128);
        }
        __syncwarp();
      }
      if (MODE == kAttnDelta && pw == 1 && lane == 0) {
        // the merge epilogue of this tile reads its rows of the complement accumulator
        const int nrows = min(128, T - b * 128);
        const size_t row0 = (static_cast<size_t>(hh) * T + b * 128) * 128;
        if (p.compact)
          prefetch_l2_bulk(p.o_c + row0, static_cast<uint32_t>(nrows) * 256u);
        else
          prefetch_l2_bulk(p.acc_c + row0, static_cast<uint32_t>(nrows) * 512u);
      }
      for (int i = 0; i <= nchunks; ++i) {
        if (i < nchunks && !load_k(g0 + i, i, hh)) {
          ok = false;
          break;
        }
        if (i >= 1 && !load_v(g0 + i - 1, i - 1, hh)) {
          ok = false;
          break;
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    int tl = 0;
    bool ok = true;
    const uint32_t tO = tmem + 256;
    for (int tile = blockIdx.x; tile < ntiles && ok && nchunks > 0; tile += gridDim.x, ++tl) {
      if (!wait_warp(&qt_full[tl & 1], (tl >> 1) & 1, p.status, abort_flag)) break;
      const uint32_t tQ = tmem + 384 + (tl & 1) * 64;
      for (int i = 0; i <= nchunks && ok; ++i) {
        if (i < nchunks) {
          const int g = tl * nchunks + i, s = g & 1;
          if (!wait_warp(&k_full[s], (g >> 1) & 1, p.status, abort_flag) ||
              !wait_warp(&s_empty[s], ((g >> 1) & 1) ^ 1, p.status, abort_flag)) {
            ok = false;
            break;
          }
          if (MODE == kAttnDelta) fence_async_smem();
          tc_fence_after();
          if (lane == 0) {
            const uint32_t k0 = smem_u32(sK + s * kTileBytes);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
              umma_bf16_ts(tmem + s * 128, tQ + kk * 8, sdesc_sw128(k0 + off, 16, 1024), kIdescQK, kk > 0);
            }
            umma_commit(&s_full[s]);
            umma_commit(&k_empty[s]);
            if (i == nchunks - 1) umma_commit(&qt_empty[tl & 1]);
          }
          __syncwarp();
        }
        if (i >= 1) {
          // P V: A = P from TMEM (buffer g & 1), B = V from shared memory
          const int j = i - 1, g = tl * nchunks + j, s = g & 1;
          // O is free once the previous tile's epilogue has read it (S of this tile went ahead)
          if (j == 0 && !wait_warp(o_empty, (tl & 1) ^ 1, p.status, abort_flag)) {
            ok = false;
            break;
          }
          if (!wait_warp(&p_full[s], (g >> 1) & 1, p.status, abort_flag) ||
              !wait_warp(&v_full[s], (g >> 1) & 1, p.status, abort_flag)) {
            ok = false;
            break;
          }
          if (MODE == kAttnDelta) fence_async_smem();
          tc_fence_after();
          if (lane == 0) {
            const uint32_t v0 = smem_u32(sV + s * kTileBytes);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              umma_bf16_ts(tO, tmem + s * 128 + kk * 8, sdesc_sw128(v0 + kk * 2048, 16384, 1024), kIdescPV,
                           (j | kk) != 0);
            umma_commit(&v_empty[s]);
            umma_commit(&p_empty[s]);
            if (j == nchunks - 1) umma_commit(o_full);
          }
          __syncwarp();
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue (warps 0-7)
    // warp w: TMEM lane quadrant w & 3 (query rows), column half w >> 2 (keys 64h.. of S, dims 64h.. of O)
    const int q = warp & 3, half = warp >> 2;
    const int r = q * 32 + lane;
    const int st = threadIdx.x;  // 0..255
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const float sl2 = p.scale_log2;
    uint32_t pair_phase = 0, mask_phase = 0;
    // both warps of the quadrant have written their partial; bounded wait
    auto pair_sync = [&]() -> bool {
      mbar_arrive(&pair_bar[q]);
      const bool r2 = wait_warp(&pair_bar[q], pair_phase & 1, p.status, abort_flag);
      ++pair_phase;
      return r2;
    };
    auto mask_sync = [&]() -> bool {
      mbar_arrive(mask_bar);
      const bool r2 = wait_warp(mask_bar, mask_phase & 1, p.status, abort_flag);
      ++mask_phase;
      return r2;
    };
    // Q of this CTA's tile tq (arrived by TMA in shared memory) into TMEM buffer tq & 1: this
    // thread's row r, dimensions 64 half .. 64 half + 63 as 32 columns of bf16 pairs; then the
    // shared-memory tile is free for the next tile's Q
    auto copy_q = [&](int tq) -> bool {
      if (!wait_warp(q_full, tq & 1, p.status, abort_flag) ||
          !wait_warp(&qt_empty[tq & 1], ((tq >> 1) & 1) ^ 1, p.status, abort_flag))
        return false;
      tc_fence_after();
      uint32_t wq[32];
      const uint8_t *qh = sQ + half * 16384;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 u = *reinterpret_cast<const uint4 *>(qh + sw128_offset(r, c));
        wq[4 * c] = u.x, wq[4 * c + 1] = u.y, wq[4 * c + 2] = u.z, wq[4 * c + 3] = u.w;
      }
      tmem_st32(tmem + lane_off + 384 + (tq & 1) * 64 + half * 32, reinterpret_cast<const float *>(wq));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&qt_full[tq & 1]);
      mbar_arrive(q_empty);
      return true;
    };
    int tl = 0;
    bool ok = true;
    if (nchunks > 0 && static_cast<int>(blockIdx.x) < ntiles && !copy_q(0)) ok = false;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++tl) {
      const int hh = tile / p.nb, b = tile % p.nb;
      const int gi = b * 128 + r;
      const int ob = tl & 1;
      const uint32_t tO = tmem + lane_off + 256 + half * 64;
      if (MODE == kAttnComplement) {
        // mask of the keys this tile's block selected
        const int nwords = (T + 31) >> 5;
        if (!mask_sync()) break;   // every softmax warp is done with the previous tile's mask
        for (int w = st; w < nwords; w += kSoftmaxThreads) mask[w] = 0u;
        if (!mask_sync()) break;
        const int32_t *irow = p.idx + (static_cast<size_t>(hh) * p.nb + b) * p.k;
        for (int j = st; j < p.k; j += kSoftmaxThreads) {
          const int key = __ldg(irow + j);
          if (static_cast<unsigned>(key) < static_cast<unsigned>(T))
            atomicOr(&mask[key >> 5], 1u << (key & 31));
          else
            atomicCAS(p.status, kDevOk, kDevBadIndex);
        }
        if (!mask_sync()) break;
      }
      // this row's cached complement statistics, needed only by the final merge
      const size_t row = static_cast<size_t>(hh) * T + gi;
      float mc = 0.f, lc = 0.f;
      if (MODE == kAttnDelta && gi < T) {
        // compact cache: l_c e^(m_c) = e^(lse_c), so lse_c takes m_c's place with l_c = 1
        mc = p.compact ? p.lse_c[row] : p.m_c[row];
        lc = p.compact ? 1.f : p.l_c[row];
      }
      float m_used = -INFINITY, l = 0.f;   // m_used in log2 units of the scaled logits
      for (int i = 0; i < nchunks; ++i) {
        const int g = tl * nchunks + i, s = g & 1;
        if (!wait_warp(&s_full[s], (g >> 1) & 1, p.status, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // keys of the chunk that take part, per 32-key group q32 (0..3): bit e = key i*128 + 32 q32 + e
        auto live_bits = [&](int q32) -> uint32_t {
          const int base = i * 128 + q32 * 32;
          const int lim = nkeys - base;
          uint32_t m = lim >= 32 ? 0xffffffffu : (lim <= 0 ? 0u : ((1u << lim) - 1u));
          if (MODE == kAttnComplement && lim > 0) m &= ~mask[base >> 5];
          return m;
        };
        // The row maximum over all 128 keys: each warp takes the maximum of its
        // half and the two warps of the quadrant exchange them through shared
        // memory, so both reach the same maximum and the same rescale decision.
        float mxp[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) mxp[u] = -INFINITY;
        float sv[64];
        tmem_ld32_async(tmem + lane_off + s * 128 + half * 64, sv);
        tmem_ld32_async(tmem + lane_off + s * 128 + half * 64 + 32, sv + 32);
        tmem_wait_ld_regs(sv);
        reg_fence32(sv + 32);
        tc_fence_before();
        mbar_arrive(&s_empty[s]);  // S now lives in registers: the buffer can take S of chunk g + 2
        // keys of this half that take part: bits of live[0] (keys 64h..64h+31) and live[1]
        const uint32_t live[2] = {live_bits(half * 2), live_bits(half * 2 + 1)};
        if ((live[0] & live[1]) != 0xffffffffu) {
#pragma unroll
          for (int e = 0; e < 64; ++e)
            if (!((live[e >> 5] >> (e & 31)) & 1u)) sv[e] = -INFINITY;
        }
#pragma unroll
        for (int e = 0; e < 64; ++e) mxp[e & 3] = fmaxf(mxp[e & 3], sv[e]);
        float mh = fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3]));
        {
          float *xm = xmax + (g & 1) * 256;
          xm[half * 128 + r] = mh;
          if (!pair_sync()) {
            ok = false;
            break;
          }
          mh = fmaxf(mh, xm[(half ^ 1) * 128 + r]);
        }
        const float mx = mh * sl2;
        const float m_new = fmaxf(m_used, mx);
        // lazy rescale: only when the max grows by more than 2^8 over the one in use
        const bool need = m_used != -INFINITY && m_new > m_used + kRescaleLog2;
        if (m_used == -INFINITY) m_used = m_new;
        if (__any_sync(0xffffffffu, need)) {
          // O holds P V of the earlier chunks (i >= 1 here): wait for the last of them, then
          // scale this half in TMEM
          if (!wait_warp(&p_empty[(g - 1) & 1], ((g - 1) >> 1) & 1, p.status, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float alpha = need ? exp2_approx(m_used - m_new) : 1.f;
          if (need) {
            l *= alpha;
            m_used = m_new;
          }
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            float ov[32];
            tmem_ld32(tO + c * 32, ov);
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] *= alpha;
            tmem_st32(tO + c * 32, ov);
          }
          tmem_wait_st();
        }
        // p = 2^(s * scale_log2 - m); masked keys hold -inf and give 0
        const float mneg = (m_used == -INFINITY) ? 0.f : -m_used;
        float lp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          const float x = fmaf(sv[e], sl2, mneg);
          sv[e] = exp2_approx(x);
          lp[e & 3] += sv[e];
        }
        l += (lp[0] + lp[1]) + (lp[2] + lp[3]);
        // P over the first 64 columns of S buffer g & 1 (this row's keys 64h .. 64h+63 as 32
        // columns of bf16 pairs). Both warps of the quadrant have read their half of S (the
        // exchange above), and P V of chunk g - 2, which read the buffer's previous P, was issued
        // before S = Q K^T of chunk g wrote it (tensor-core operations run in issue order).
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) pk[e] = cvt_bf16x2(sv[2 * e], sv[2 * e + 1]);
        tc_fence_after();
        tmem_st32(tmem + lane_off + (g & 1) * 128 + half * 32, reinterpret_cast<const float *>(pk));
        tmem_wait_st();
        tc_fence_before();  // orders the P stores (and a rescale's O stores) before the next P V
        mbar_arrive(&p_full[g & 1]);
      }
      if (!ok) break;
      // the next tile's Q into TMEM now, so its first S = Q K^T overlaps this tile's epilogue
      if (nchunks > 0 && tile + static_cast<int>(gridDim.x) < ntiles && !copy_q(tl + 1)) break;
      // row sum over both halves (buffer by tile parity: the next write to it is two tiles away)
      float *xs = xsum + ob * 256;
      xs[half * 128 + r] = l;
      if (!pair_sync()) break;
      l += xs[(half ^ 1) * 128 + r];
      // Delta pass: the complement rows of this warp's 32 queries (this half's
      // 64 dimensions, pulled into L2 by the producers at the start of the
      // tile) and the output rows move as whole runs through the warp's shared
      // buffer (rows padded to 36 words): fp32 lane = query 4 i + lane / 8,
      // 16-byte piece lane % 8 of a 32-dimension group; bf16 (the compact
      // cache, the output) lane = query 8 i + lane / 4, piece lane % 4. The
      // first group is loaded while P V of the last chunk runs, the second
      // while the first is merged.
      const bool compact = p.compact != 0;
      float *eb = ebuf + warp * (32 * 36);
      const int qbase = b * 128 + q * 32;
      float4 gv[8];
      auto load_group = [&](int c) {
        const int d = half * 64 + c * 32;
        if (!compact) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int gq = qbase + 4 * i + (lane >> 3);
            gv[i] = gq < T ? *reinterpret_cast<const float4 *>(p.acc_c + (static_cast<size_t>(hh) * T + gq) * 128 + d +
                                                               4 * (lane & 7))
                           : make_float4(0.f, 0.f, 0.f, 0.f);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int gq = qbase + 8 * i + (lane >> 2);
            const uint4 u = gq < T ? *reinterpret_cast<const uint4 *>(p.o_c + (static_cast<size_t>(hh) * T + gq) * 128 +
                                                                      d + 8 * (lane & 3))
                                   : make_uint4(0u, 0u, 0u, 0u);
            gv[i] = make_float4(__uint_as_float(u.x), __uint_as_float(u.y), __uint_as_float(u.z), __uint_as_float(u.w));
          }
        }
      };
      if (MODE == kAttnDelta) load_group(0);
      if (nchunks > 0) {
        if (!wait_warp(o_full, tl & 1, p.status, abort_flag)) break;
        tc_fence_after();
      }
      const float m2 = m_used;
      float wc = 0.f, ws = 0.f, inv = 0.f;
      if (MODE == kAttnDelta) {
        const float mc2 = mc * kLog2e;
        const float M = fmaxf(mc2, m2);
        wc = (mc == -INFINITY) ? 0.f : exp2_approx(mc2 - M);
        ws = (m2 == -INFINITY) ? 0.f : exp2_approx(m2 - M);
        const float L = lc * wc + l * ws;
        inv = L > 0.f ? 1.f / L : 0.f;
      } else if (MODE == kAttnDense || compact) {
        inv = l > 0.f ? 1.f / l : 0.f;
      }
      // O of this half in two groups of 32 dimensions
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float ov[32];
        if (nchunks > 0) {
          tmem_ld32(tO + c * 32, ov);
          if (c == 1) {
            tc_fence_before();
            mbar_arrive(o_empty);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = 0.f;
        }
        const int d0 = half * 64 + c * 32;
        if (MODE == kAttnDelta) {
          // the group's complement values into the buffer, then this thread's row out of it
          if (!compact) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              *reinterpret_cast<float4 *>(eb + (4 * i + (lane >> 3)) * 36 + 4 * (lane & 7)) = gv[i];
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              *reinterpret_cast<float4 *>(eb + (8 * i + (lane >> 2)) * 36 + 4 * (lane & 3)) = gv[i];
          }
          __syncwarp();
          if (c == 0) load_group(1);
          uint32_t w[16];
#pragma unroll
          for (int e8 = 0; e8 < 4; ++e8) {
            float av[8];  // complement accumulator (partial) or normalised output (compact), dims d0 + 8 e8 ..
            if (compact) {
              const uint4 u = *reinterpret_cast<const uint4 *>(eb + lane * 36 + 4 * e8);
              const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                av[2 * j] = __uint_as_float(w4[j] << 16);
                av[2 * j + 1] = __uint_as_float(w4[j] & 0xffff0000u);
              }
            } else {
              const float4 a0 = *reinterpret_cast<const float4 *>(eb + lane * 36 + 8 * e8);
              const float4 a1 = *reinterpret_cast<const float4 *>(eb + lane * 36 + 8 * e8 + 4);
              av[0] = a0.x, av[1] = a0.y, av[2] = a0.z, av[3] = a0.w;
              av[4] = a1.x, av[5] = a1.y, av[6] = a1.z, av[7] = a1.w;
            }
            const float *oa = ov + 8 * e8;
#pragma unroll
            for (int j = 0; j < 4; ++j)
              w[4 * e8 + j] = cvt_bf16x2((av[2 * j] * wc + oa[2 * j] * ws) * inv, (av[2 * j + 1] * wc + oa[2 * j + 1] * ws) * inv);
          }
          // the merged row (bf16) back into the buffer, then out as whole runs
          __syncwarp();
#pragma unroll
          for (int v = 0; v < 4; ++v)
            *reinterpret_cast<uint4 *>(eb + lane * 36 + 4 * v) = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int rr = 8 * i + (lane >> 2);
            const int gq = qbase + rr;
            if (gq < T)
              *reinterpret_cast<uint4 *>(p.o + (static_cast<size_t>(gq) * p.h + hh) * 128 + d0 + 8 * (lane & 3)) =
                  *reinterpret_cast<const uint4 *>(eb + rr * 36 + 4 * (lane & 3));
          }
          __syncwarp();  // the buffer takes the next group
        } else if (gi < T) {
          if (MODE == kAttnDense) {
            uint4 *orow = reinterpret_cast<uint4 *>(p.o + (static_cast<size_t>(gi) * p.h + hh) * 128 + d0);
#pragma unroll
            for (int e8 = 0; e8 < 4; ++e8) {
              const float *oa = ov + 8 * e8;
              orow[e8] = make_uint4(cvt_bf16x2(oa[0] * inv, oa[1] * inv), cvt_bf16x2(oa[2] * inv, oa[3] * inv),
                                    cvt_bf16x2(oa[4] * inv, oa[5] * inv), cvt_bf16x2(oa[6] * inv, oa[7] * inv));
            }
          } else if (compact) {
            uint4 *oc = reinterpret_cast<uint4 *>(p.o_c + row * 128 + d0);
#pragma unroll
            for (int e8 = 0; e8 < 4; ++e8) {
              const float *oa = ov + 8 * e8;
              oc[e8] = make_uint4(cvt_bf16x2(oa[0] * inv, oa[1] * inv), cvt_bf16x2(oa[2] * inv, oa[3] * inv),
                                  cvt_bf16x2(oa[4] * inv, oa[5] * inv), cvt_bf16x2(oa[6] * inv, oa[7] * inv));
            }
          } else {
            float4 *ac = reinterpret_cast<float4 *>(p.acc_c + row * 128 + d0);
#pragma unroll
            for (int e4 = 0; e4 < 8; ++e4)
              ac[e4] = make_float4(ov[4 * e4], ov[4 * e4 + 1], ov[4 * e4 + 2], ov[4 * e4 + 3]);
          }
        }
      }
      if (gi < T && half == 0) {
        if (MODE == kAttnDense) {
          p.lse[row] = l > 0.f ? (m2 + log2f(l)) * kLn2 : -INFINITY;
        } else if (MODE == kAttnComplement && compact) {
          p.lse_c[row] = l > 0.f ? (m2 + log2f(l)) * kLn2 : -INFINITY;
        } else if (MODE == kAttnComplement) {
          p.m_c[row] = (m2 == -INFINITY) ? -INFINITY : m2 * kLn2;
          p.l_c[row] = l;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

template <int MODE>
uint32_t attn_smem(int64_t T) {
  const uint32_t mask_bytes = MODE == kAttnComplement ? ((static_cast<uint32_t>(T) + 31) / 32) * 4 : 0;
  const uint32_t merge_bytes = MODE == kAttnDelta ? 8 * 32 * 36 * 4 : 0;
  static_assert(1024 + AttnCfg::kMaskOff + 8 * 32 * 36 * 4 <= 232448, "delta pass over one CTA's shared memory");
  return 1024 + AttnCfg::kMaskOff + mask_bytes + merge_bytes;
}

template <int MODE>
cudaError_t launch_attn_t(const AttnParams &p, const CUtensorMap &q, const CUtensorMap &k, const CUtensorMap &v,
                          cudaStream_t s) {
  const uint32_t smem = attn_smem<MODE>(p.T);
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = static_cast<int64_t>(p.h) * p.nb;
  const int64_t grid = std::min<int64_t>(tiles, sms);
  attn_kernel<MODE><<<static_cast<unsigned>(grid), kThreads, smem, s>>>(q, k, v, p);
  return cudaGetLastError();
}

}  // namespace

uint32_t attn_smem_bytes(int mode, int64_t T) {
  return mode == kAttnComplement ? attn_smem<kAttnComplement>(T) : attn_smem<kAttnDelta>(T);
}

cudaError_t launch_attn(int mode, const AttnParams &p, const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                        const CUtensorMap &tm_v, cudaStream_t s) {
  if (p.h <= 0 || p.nb <= 0) return cudaSuccess;
  switch (mode) {
    case kAttnDelta: return launch_attn_t<kAttnDelta>(p, tm_q, tm_k, tm_v, s);
    case kAttnDense: return launch_attn_t<kAttnDense>(p, tm_q, tm_k, tm_v, s);
    case kAttnComplement: return launch_attn_t<kAttnComplement>(p, tm_q, tm_k, tm_v, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace cm
