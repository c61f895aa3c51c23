// mlp.cu - gathered-column MLP kernels of the sparse delta step and the refresh.
//
// Kernel 1 (mlp_up, the sparse step and the refresh of 64-token blocks):
// tiles (token block b, chunk of 128 selected hidden columns), walked by
// persistent CTAs, two per SM. The 128 selected rows of W1^T are gathered
// into a 128-byte-swizzled shared tile by four producer warps with 16-byte
// cp.async (each warp instruction moves four whole 128-byte row segments); on
// a refresh, where the rows are consecutive, one TMA tile load brings them
// instead. (The refresh of 128-token blocks runs the wide form further down.) The token block of x arrives by a tiled TMA load. One
// thread issues tcgen05 bf16 MMAs accumulating D[col][token] in one of two
// TMEM accumulators. Each epilogue thread owns one hidden column (one TMEM
// lane); the activation cache runs a_cache[b][c][..] and the delta rows are
// moved 64 bytes per run between global memory and a per-warp shared buffer
// that turns them around to and from that layout.
//
// Kernel 2 (mlp_down): one CTA per (token block b, slice of BN model columns).
// K runs over the selected hidden units: the delta rows come from the
// workspace by tiled TMA, the matching W2 rows are gathered by the producer
// warps with cp.async (one warp instruction = whole row segments); both
// operands are MN-major. The epilogue adds the fp32 result into the output
// cache (or overwrites it with result + b2 on a refresh) and writes the bf16
// layer output; each warp turns its 32 x 32 accumulator chunks around in
// shared memory first, so those accesses are whole-line runs.
//
// Each kernel keeps two shared-memory rings: one for the gathered operand
// (filled by the cp.async producer warps) and one for the operand that
// arrives by tiled TMA. The warp roles are listed with `Roles` below. Data
// written by cp.async must pass a generic-to-async proxy fence before the
// tensor core reads it; in mlp_up the TMA warp takes that fence for each
// gathered stage and hands the stage on through a second barrier, because the
// fence stalls whichever warp executes it and the MMA warp is mlp_up's
// critical path (mlp_down's MMA warp takes it itself at no measurable cost).
#include <cuda_fp8.h>

#include <algorithm>

#include "kernels.cuh"
#include "ptx.cuh"

namespace cm {
namespace {

// Warp roles of both kernels: warps 0 .. P-1 gather with cp.async, warp P
// issues the MMAs and owns TMEM, warps P+1 .. P+E run the epilogue (TMEM lane
// quadrant = warp % 4; with E = 8 two warps share a quadrant, one per half of
// the accumulator columns), warp P+E+1 issues the TMA loads.
template <int P, int E>
struct Roles {
  static constexpr int kProdWarps = P;
  static constexpr int kProducers = 32 * P;
  static constexpr int kMmaWarp = P;
  static constexpr int kEpiWarp0 = P + 1;
  static constexpr int kEpiWarps = E;
  static constexpr int kTmaWarp = P + 1 + E;
  static constexpr int kThreads = 32 * (P + 2 + E);
};

constexpr int kBK = 64;  // K elements per pipeline stage = one 128-byte swizzle row

// The order in which a CTA's tiles are walked. Tile t of nb token blocks x
// nparts parts of a block (chunks of its selected columns, or slices of the
// output) is taken a group of `group` blocks at a time, part-major inside the
// group: CTAs running at the same time work on the same part of different
// blocks, so they gather weight rows from the same region of the (ascending)
// index lists, and a group's activation tiles stay in L2 until all of its
// parts are done instead of being read from HBM again for every part. With
// group = nb this is part-major over the whole layer.
struct TileAt {
  int b, part;
};

__device__ __forceinline__ TileAt tile_at(int t, int nb, int nparts, int group) {
  const int per_group = group * nparts;
  const int g = t / per_group, r = t - g * per_group;
  const int b0 = g * group;
  const int gb = min(group, nb - b0);   // blocks in this group (the last may be short)
  return {b0 + r % gb, r / gb};
}

// Blocks walked together: all of them when the layer's activation tiles (x for
// the up-projection) fit in well under half of L2 (the FLUX.1-dev 1280x768 layer), else
// as many as fill about 24 MB (32 blocks of 128 tokens at D = 3072 in bf16).
int up_tile_group(int nb, int64_t tile_bytes) {
  if (static_cast<int64_t>(nb) * tile_bytes <= (48ll << 20)) return nb;
  return std::max<int>(8, static_cast<int>((24ll << 20) / tile_bytes));
}

// The sparse down-projection walks slice-major over all blocks: every CTA
// running at a time gathers W2 rows of the same output slice, which matters
// more for it than keeping the delta tiles of a group in L2 (measured). The
// dense one (a refresh) reads every block's whole activation-cache tile (3 MB at
// H = 12288) once per output slice, so it is walked in groups like the
// up-projection.
int down_tile_group(int nb, bool dense, int64_t tile_bytes) { return dense ? up_tile_group(nb, tile_bytes) : nb; }

// Warp-uniform bounded wait: every lane polls, the warp leaves together.
__device__ __forceinline__ bool wait_warp(uint64_t *bar, uint32_t parity, int *status, volatile int *abort_flag) {
  const bool ok = mbar_wait(bar, parity, status, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

template <int BT>
struct UpCfg : Roles<4, 4> {
  static constexpr int kCtasPerSm = 2;                // two independent pipelines per SM
  static constexpr int kStagesA = BT == 128 ? 3 : 4;  // gathered W1^T rows
  static constexpr int kStagesB = BT == 128 ? 3 : 4;  // x tile
  static constexpr uint32_t kABytes = 128 * 128;      // 128 gathered rows x 64 bf16
  static constexpr uint32_t kBBytes = BT * 128;       // BT tokens x 64 bf16
  static constexpr uint32_t kBOff = kStagesA * kABytes;
  static constexpr uint32_t kPartOff = kBOff + kStagesB * kBBytes;  // [2][128] fp32 partial column scores
  static constexpr uint32_t kBarOff = kPartOff + 2 * 128 * 4;
  static constexpr uint32_t kTbBytes = 32 * 80;  // per epilogue warp: 32 columns x 32 tokens bf16, rows padded to 80 B
  static constexpr uint32_t kEpiOff = kBarOff + 1024;
  static constexpr uint32_t kSmem = 1024 + kEpiOff + kEpiWarps * kTbBytes;
  static_assert(kCtasPerSm * (kSmem + 1024) <= 233472, "two CTAs must fit in one SM's shared memory");
};

// Persistent: CTA c handles tiles c, c + gridDim.x, ..., tile t being chunk
// tile_at(t).part of block tile_at(t).b (grouped, chunk-major in a group: CTAs
// running at the same time gather W1^T rows from the same region, for L2 reuse,
// and a group's x tiles stay in L2). Two TMEM
// accumulators alternate between tiles, so the epilogue of one tile overlaps
// the main loop of the next; ring stages and parities follow one running
// k-step counter across tiles.
//
// F8: the FP8 form of the sparse step. x and W1^T arrive as e4m3 codes; a
// stage still holds 128-byte rows, now of 128 K elements, and the tensor core
// runs kind::f8f6f4 (K = 32 per instruction). The epilogue scales the fp32
// accumulator by s1[c] * sx[t] before the bias, and writes each delta as the
// e4m3 code of delta * g2[c] (the down-projection's operand).
template <int BT, bool DENSE, bool F8 = false>
__global__ void __launch_bounds__(UpCfg<BT>::kThreads, UpCfg<BT>::kCtasPerSm)
    mlp_up_kernel(const __grid_constant__ CUtensorMap tm_w1t, const __grid_constant__ CUtensorMap tm_x,
                  const MlpUpParams p) {
  using C = UpCfg<BT>;
  static_assert(!F8 || (BT == 128 && !DENSE), "the FP8 step runs the sparse form with 128-token blocks");
  constexpr int SA = C::kStagesA, SB = C::kStagesB;
  constexpr int kProducers = C::kProducers, kMmaWarp = C::kMmaWarp, kTmaWarp = C::kTmaWarp;
  constexpr int kEpiThreads = 32 * C::kEpiWarps;
  constexpr int kParts = C::kEpiWarps / 4;  // epilogue warps per TMEM lane quadrant
  constexpr int kHalf = BT / kParts;         // accumulator columns (tokens) of one epilogue warp
  constexpr int kRowIters = 1024 / kProducers;  // gathered rows of a stage per producer thread
  constexpr int kEs = F8 ? 1 : 2;               // bytes per operand element
  constexpr int kKStage = 128 / kEs;            // K elements per stage (one 128-byte swizzle row)
  constexpr uint32_t kIdesc = F8 ? idesc_e4m3(128, BT, false, false) : idesc_bf16(128, BT, false, false);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align_up<1024>(smem_raw);
  uint8_t *sA = smem;
  uint8_t *sB = smem + C::kBOff;
  float *part = reinterpret_cast<float *>(smem + C::kPartOff);
  uint64_t *a_full = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
  uint64_t *a_empty = a_full + SA;
  uint64_t *b_full = a_empty + SA;
  uint64_t *b_empty = b_full + SB;
  uint64_t *acc_full = b_empty + SB;   // [2]
  uint64_t *acc_empty = acc_full + 2;  // [2]
  uint64_t *part_bar = acc_empty + 2;  // refresh: both token halves of every column have their partial score
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(part_bar + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  uint64_t *a_ready = part_bar + 2;    // [SA] sparse step: a gathered stage is ordered for the tensor core

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (*(volatile int *)p.status != kDevOk) return;
  const bool sparse = p.mode == kUpDelta;
  const int ntiles = p.nb * p.nchunks;
  const int my_tiles = static_cast<int>(blockIdx.x) < ntiles
                           ? (ntiles - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                           : 0;
  const int nk = p.D / kKStage;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SA; ++s) {
      mbar_init(&a_full[s], DENSE ? 1 : kProducers);
      mbar_init(&a_empty[s], 1);
    }
    for (int s = 0; s < SB; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], kEpiThreads);
    }
    mbar_init(part_bar, kEpiThreads);
    for (int s = 0; s < SA; ++s) mbar_init(&a_ready[s], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (threadIdx.x == kTmaWarp * 32) {
    prefetch_tmap(&tm_w1t);
    prefetch_tmap(&tm_x);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 2 * BT);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < C::kProdWarps) {
    // gathered W1^T rows: thread pt moves 16-byte chunk (pt & 7) of rows
    // i * (kProducers / 8) + (pt >> 3), i = 0 .. kRowIters - 1
    if (!DENSE) {
      const int pt = threadIdx.x;
      uint32_t dst_off[kRowIters];
#pragma unroll
      for (int i = 0; i < kRowIters; ++i) dst_off[i] = sw128_offset(i * (kProducers / 8) + (pt >> 3), pt & 7);
      // this thread's selected columns of the CTA's tile tl, loaded one tile
      // ahead and range-checked when they are used
      auto load_rows = [&](int tl, int *c) {
        const int tile = blockIdx.x + tl * gridDim.x;
        const TileAt ta = tile_at(tile, p.nb, p.nchunks, p.group);
        const int chunk = ta.part, b = ta.b;
#pragma unroll
        for (int i = 0; i < kRowIters; ++i)
          c[i] = tl < my_tiles ? __ldg(p.idx + static_cast<size_t>(b) * p.k +
                                      min(chunk * 128 + i * (kProducers / 8) + (pt >> 3), p.k - 1))
                               : 0;
      };
      int nxt[kRowIters];
      load_rows(0, nxt);
      const uint32_t a_base = smem_u32(sA);
      int kg = 0;
      bool ok = true;
      const uint8_t *w1b = reinterpret_cast<const uint8_t *>(p.w1t);
      for (int tl = 0; tl < my_tiles && ok; ++tl) {
        const uint8_t *src_row[kRowIters];   // this thread's 16-byte piece of each gathered row
#pragma unroll
        for (int i = 0; i < kRowIters; ++i) {
          int c = nxt[i];
          if (static_cast<unsigned>(c) >= static_cast<unsigned>(p.H)) {  // never address outside the weights
            atomicCAS(p.status, kDevOk, kDevBadIndex);
            c = 0;
          }
          src_row[i] = w1b + static_cast<size_t>(c) * p.D * kEs + (pt & 7) * 16;
        }
        load_rows(tl + 1, nxt);
        for (int kb = 0; kb < nk; ++kb, ++kg) {
          const int s = kg % SA;
          if (!wait_warp(&a_empty[s], ((kg / SA) & 1) ^ 1, p.status, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t stage = a_base + s * C::kABytes;
#pragma unroll
          for (int i = 0; i < kRowIters; ++i) cp_async_16(stage + dst_off[i], src_row[i] + kb * 128);
          cp_async_arrive_noinc(&a_full[s]);
        }
      }
    }
  } else if (warp == kTmaWarp) {
    // x tiles (and, on a refresh, the consecutive W1^T rows) by TMA
    int kg = 0;
    bool ok = true;
    for (int tl = 0; tl < my_tiles && ok; ++tl) {
      const int tile = blockIdx.x + tl * gridDim.x;
      const TileAt ta = tile_at(tile, p.nb, p.nchunks, p.group);
      const int chunk = ta.part, b = ta.b;
      for (int kb = 0; kb < nk; ++kb, ++kg) {
        if (DENSE) {
          const int s = kg % SA;
          if (!wait_warp(&a_empty[s], ((kg / SA) & 1) ^ 1, p.status, abort_flag)) {
            ok = false;
            break;
          }
          if (lane == 0) {
            mbar_arrive_expect_tx(&a_full[s], C::kABytes);
            tma_load_2d(sA + s * C::kABytes, &tm_w1t, &a_full[s], kb * kBK, chunk * 128);
          }
        }
        const int s = kg % SB;
        if (!wait_warp(&b_empty[s], ((kg / SB) & 1) ^ 1, p.status, abort_flag)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&b_full[s], C::kBBytes);
          tma_load_2d(sB + s * C::kBBytes, &tm_x, &b_full[s], kb * kKStage, b * BT);
        }
        __syncwarp();
        if (!DENSE && kg >= 1) {
          // the previous gathered stage has landed: order it for the tensor core here,
          // off the MMA warp
          const int r = kg - 1;
          if (!wait_warp(&a_full[r % SA], (r / SA) & 1, p.status, abort_flag)) {
            ok = false;
            break;
          }
          fence_async_smem();
          if (lane == 0) mbar_arrive(&a_ready[r % SA]);
          __syncwarp();
        }
      }
    }
    if (!DENSE && ok && kg >= 1) {
      const int r = kg - 1;
      if (wait_warp(&a_full[r % SA], (r / SA) & 1, p.status, abort_flag)) {
        fence_async_smem();
        if (lane == 0) mbar_arrive(&a_ready[r % SA]);
      }
    }
  } else if (warp == kMmaWarp) {
    int kg = 0;
    bool ok = true;
    for (int tl = 0; tl < my_tiles && ok; ++tl) {
      const int ab = tl & 1;
      const uint32_t tacc = tmem + ab * BT;
      if (!wait_warp(&acc_empty[ab], ((tl >> 1) & 1) ^ 1, p.status, abort_flag)) break;
      tc_fence_after();
      for (int kb = 0; kb < nk; ++kb, ++kg) {
        const int sa = kg % SA, sb = kg % SB;
        if (!wait_warp(DENSE ? &a_full[sa] : &a_ready[sa], (kg / SA) & 1, p.status, abort_flag) ||
            !wait_warp(&b_full[sb], (kg / SB) & 1, p.status, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a0 = smem_u32(sA + sa * C::kABytes);
          const uint32_t b0 = smem_u32(sB + sb * C::kBBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {   // 32 bytes of K per instruction
            const uint64_t ad = sdesc_sw128(a0 + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(b0 + kk * 32, 16, 1024);
            if (F8)
              umma_e4m3(tacc, ad, bd, kIdesc, (kb | kk) != 0);
            else
              umma_bf16(tacc, ad, bd, kIdesc, (kb | kk) != 0);
          }
          umma_commit(&a_empty[sa]);
          umma_commit(&b_empty[sb]);
        }
        __syncwarp();
      }
      if (ok && lane == 0) umma_commit(&acc_full[ab]);
      __syncwarp();
    }
  } else {
    // epilogue: thread = one selected column (TMEM lane r) and 1 / kParts of
    // the block's tokens, 32 tokens at a time. The cached activations and the
    // delta rows are moved between global memory and the warp's shared buffer
    // as whole 64-byte runs (lane: 16-byte piece lane % 4 of the columns
    // 8 i + lane / 4), and turned around there to and from the one-column-per-
    // thread layout of the accumulator.
    const int ew = warp - C::kEpiWarp0;
    const int q = warp & 3;
    const int th = ew >> 2;
    const int r = q * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const bool first = p.mode == kUpRefreshFirst;
    uint8_t *tb = smem + C::kEpiOff + ew * C::kTbBytes;
    const int ck = lane & 3, cq = lane >> 2;
    for (int tl = 0; tl < my_tiles; ++tl) {
      const int tile = blockIdx.x + tl * gridDim.x;
      const TileAt ta = tile_at(tile, p.nb, p.nchunks, p.group);
      const int chunk = ta.part, b = ta.b;
      const int ab = tl & 1;
      const int j = chunk * 128 + r;
      bool valid_j = sparse ? (j < p.k) : (j < p.H);
      // column, bias and the cached activations are fetched before the accumulator is ready
      int c;
      if (sparse) {
        c = __ldg(p.idx + static_cast<size_t>(b) * p.k + min(j, p.k - 1));
        if (static_cast<unsigned>(c) >= static_cast<unsigned>(p.H)) {
          // never address outside the weights / cache; the column is dropped: no cache
          // write, and its delta row is zero so the down-projection adds nothing for it
          atomicCAS(p.status, kDevOk, kDevBadIndex);
          c = 0;
          valid_j = false;
        }
      } else {
        c = min(j, p.H - 1);
      }
      const float bias = bf16_bits_to_f32(__ldg(p.b1 + c));
      const float s1c = F8 ? __ldg(p.s1 + c) : 1.f;   // FP8: scale of the column's W1^T row
      const float g2c = F8 ? __ldg(p.g2 + c) : 0.f;   // FP8: factor of the column's delta before rounding
      const int nvalid = min(BT, p.T - b * BT);
      const bool need_old = valid_j && !(first && !sparse);
      // the columns whose runs this lane moves: 8 i + cq, i = 0..3
      int ci_of[4];
      uint32_t val_mask = 0, old_mask = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        ci_of[i] = __shfl_sync(0xffffffffu, c, 8 * i + cq);
        val_mask |= __shfl_sync(0xffffffffu, valid_j ? 1u : 0u, 8 * i + cq) << i;
        old_mask |= __shfl_sync(0xffffffffu, need_old ? 1u : 0u, 8 * i + cq) << i;
      }
      const size_t a_off = static_cast<size_t>(b) * p.H * BT + th * kHalf + ck * 8;
      auto arun = [&](int i) { return p.a_cache + a_off + static_cast<size_t>(ci_of[i]) * BT; };
      uint16_t *drun0 = sparse ? p.delta + (static_cast<size_t>(b) * p.k_pad + chunk * 128 + q * 32 + cq) * BT +
                                     th * kHalf + ck * 8
                               : nullptr;
      uint4 pre[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        pre[i] = (old_mask >> i) & 1 ? *reinterpret_cast<const uint4 *>(arun(i)) : make_uint4(0, 0, 0, 0);
      if (!wait_warp(&acc_full[ab], (tl >> 1) & 1, p.status, abort_flag)) break;
      tc_fence_after();
      float score = 0.f;
#pragma unroll 1
      for (int tq = 0; tq < kHalf / 32; ++tq) {
        // old activations of tokens 32 tq .. into the buffer, then this thread's column out of it
#pragma unroll
        for (int i = 0; i < 4; ++i) *reinterpret_cast<uint4 *>(tb + (8 * i + cq) * 80 + ck * 16) = pre[i];
        __syncwarp();
        uint4 oldw[4];
#pragma unroll
        for (int v = 0; v < 4; ++v) oldw[v] = *reinterpret_cast<const uint4 *>(tb + lane * 80 + v * 16);
        float acc[32];
        tmem_ld32(tmem + lane_off + ab * BT + th * kHalf + tq * 32, acc);
        if (tq == kHalf / 32 - 1) {
          tc_fence_before();
          mbar_arrive(&acc_empty[ab]);  // the accumulator can take the next-but-one tile
        }
        const uint16_t *old = reinterpret_cast<const uint16_t *>(oldw);
        // FP8: the scale of token 32 tq + lane, handed to every lane by shuffles
        const int t_lane = th * kHalf + tq * 32 + lane;
        const float sx_lane = F8 && t_lane < nvalid ? __ldg(p.sx + static_cast<size_t>(b) * BT + t_lane) : 0.f;
        uint32_t na[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          uint16_t nab[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int t = th * kHalf + tq * 32 + i + u;
            float pre_act = acc[i + u] + bias;
            if (F8) pre_act = fmaf(acc[i + u], s1c * __shfl_sync(0xffffffffu, sx_lane, i + u), bias);
            const float a = gelu_tanh(pre_act);
            const bool tok = t < nvalid;
            nab[u] = tok ? f32_to_bf16_bits(a) : old[i + u];
            if (!sparse) score += tok ? fabsf(first ? a : a - bf16_bits_to_f32(old[i + u])) : 0.f;
          }
          na[i / 2] = static_cast<uint32_t>(nab[0]) | (static_cast<uint32_t>(nab[1]) << 16);
        }
        // new activations back through the buffer as whole runs
        __syncwarp();
#pragma unroll
        for (int v = 0; v < 4; ++v)
          *reinterpret_cast<uint4 *>(tb + lane * 80 + v * 16) = make_uint4(na[4 * v], na[4 * v + 1], na[4 * v + 2], na[4 * v + 3]);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if ((val_mask >> i) & 1)
            *reinterpret_cast<uint4 *>(arun(i) + tq * 32) = *reinterpret_cast<const uint4 *>(tb + (8 * i + cq) * 80 + ck * 16);
        // the next chunk's old activations are in flight while the delta goes out
        if (tq + 1 < kHalf / 32) {
#pragma unroll
          for (int i = 0; i < 4; ++i)
            pre[i] = (old_mask >> i) & 1 ? *reinterpret_cast<const uint4 *>(arun(i) + (tq + 1) * 32) : make_uint4(0, 0, 0, 0);
        }
        if (F8) {
          // the e4m3 code of (bf16(new) - old) * g2[c] for real tokens of a selected
          // column, else 0; this column's 32 codes go straight out as two 16-byte pieces
          const uint16_t *nw = reinterpret_cast<const uint16_t *>(na);
          uint32_t cw[8];
#pragma unroll
          for (int w = 0; w < 8; ++w) {
            uint32_t word = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = 4 * w + e;
              const bool tok = th * kHalf + tq * 32 + i < nvalid;
              const float d = (bf16_bits_to_f32(nw[i]) - bf16_bits_to_f32(old[i])) * g2c;
              const uint32_t code = (valid_j && tok) ? static_cast<uint32_t>(__nv_cvt_float_to_fp8(d, __NV_SATFINITE, __NV_E4M3)) : 0u;
              word |= code << (8 * e);
            }
            cw[w] = word;
          }
          uint8_t *drow = reinterpret_cast<uint8_t *>(p.delta) +
                          (static_cast<size_t>(b) * p.k_pad + chunk * 128 + r) * BT + th * kHalf + tq * 32;
          reinterpret_cast<uint4 *>(drow)[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
          reinterpret_cast<uint4 *>(drow)[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
        } else if (sparse) {
          // delta = bf16(new) - old for real tokens of a selected column, else 0
          const uint16_t *nw = reinterpret_cast<const uint16_t *>(na);
          uint32_t dl[16];
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            uint16_t dlb[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const bool tok = th * kHalf + tq * 32 + i + u < nvalid;
              dlb[u] = (valid_j && tok) ? f32_to_bf16_bits(bf16_bits_to_f32(nw[i + u]) - bf16_bits_to_f32(old[i + u]))
                                        : static_cast<uint16_t>(0);
            }
            dl[i / 2] = static_cast<uint32_t>(dlb[0]) | (static_cast<uint32_t>(dlb[1]) << 16);
          }
          __syncwarp();
#pragma unroll
          for (int v = 0; v < 4; ++v)
            *reinterpret_cast<uint4 *>(tb + lane * 80 + v * 16) = make_uint4(dl[4 * v], dl[4 * v + 1], dl[4 * v + 2], dl[4 * v + 3]);
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 4; ++i)
            *reinterpret_cast<uint4 *>(drun0 + static_cast<size_t>(8 * i) * BT + tq * 32) =
                *reinterpret_cast<const uint4 *>(tb + (8 * i + cq) * 80 + ck * 16);
        }
        __syncwarp();  // the buffer takes the next chunk's old activations
      }
      if (!sparse && kParts == 1) {
        if (valid_j) p.scores[static_cast<size_t>(b) * p.H + c] = score;
      } else if (!sparse) {
        // the two token halves of a column add up their partial scores in a fixed order
        float *pp = part + (tl & 1) * 128;
        if (th == 1) pp[r] = score;
        mbar_arrive(part_bar);
        if (!wait_warp(part_bar, tl & 1, p.status, abort_flag)) break;
        if (th == 0 && valid_j) p.scores[static_cast<size_t>(b) * p.H + c] = score + pp[r];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, 2 * BT);
}

// Kernel 1 for 128-token blocks, wide form: tiles (token block b, chunk of
// N = 256 hidden columns). The MMA computes D[token][col] with the x tile as
// operand A (M = 128 tokens) and the 256 W1^T rows as operand B (N = 256), so
// each K step reads 48 KB of operands from shared memory for 4.2 MFLOP and
// every x tile serves 256 columns. One CTA per SM: warps 0-7 gather (sparse
// step), warp 8 issues the MMAs into two TMEM accumulators of 256 columns,
// warps 9-12 run the epilogue, warp 13 loads x (and, on a refresh, the
// consecutive W1^T rows) by TMA. The epilogue warp of lane quadrant q owns
// tokens 32q .. 32q + 31; it turns each 32 x 32 accumulator chunk around in a
// padded shared buffer so that a thread holds one column's 32 tokens, and
// moves the activation-cache and delta runs of those tokens (64 bytes per
// column) through a second buffer as whole runs. The refresh uses this form;
// on a sparse step the two-CTA form above measured as fast or faster (FLUX.1-dev
// layer: 137 against 140 us), so the sparse step keeps that one.
template <int N>
struct UpWideCfg : Roles<8, 4> {
  static constexpr int kN = N;                         // selected columns per tile
  static constexpr uint32_t kTmemCols = 512;           // two accumulators of kN columns, allocated as a power of two
  static_assert(2 * N <= 512, "two accumulators must fit in TMEM");
  static constexpr int kStages = 4;
  static constexpr uint32_t kABytes = 128 * 128;       // x: 128 tokens x 64 bf16
  static constexpr uint32_t kBBytes = kN * 128;        // gathered W1^T: kN rows x 64 bf16
  static constexpr uint32_t kBOff = kStages * kABytes;
  static constexpr uint32_t kPartOff = kBOff + kStages * kBBytes;   // refresh: [4][kN] partial column scores
  static constexpr uint32_t kBarOff = kPartOff + 4 * kN * 4;
  static constexpr uint32_t kTrOff = kBarOff + 1024;                // per epilogue warp: 32 x 33 fp32
  static constexpr uint32_t kTbOff = kTrOff + kEpiWarps * 32 * 33 * 4;   // per epilogue warp: 32 x 80 B
  static constexpr uint32_t kSmem = 1024 + kTbOff + kEpiWarps * 32 * 80;
  static_assert(kSmem <= 232448, "over the shared memory of one CTA");
};

template <int N, bool DENSE>
__global__ void __launch_bounds__(UpWideCfg<N>::kThreads, 1)
    mlp_up_wide_kernel(const __grid_constant__ CUtensorMap tm_w1t, const __grid_constant__ CUtensorMap tm_x,
                       const MlpUpParams p) {
  using C = UpWideCfg<N>;
  static_assert(!DENSE || N % 128 == 0, "a refresh loads the consecutive W1^T rows in boxes of 128");
  constexpr int BT = 128, kN = C::kN, S = C::kStages;
  constexpr int kProducers = C::kProducers, kMmaWarp = C::kMmaWarp, kTmaWarp = C::kTmaWarp;
  constexpr int kRowIters = kN * 8 / kProducers;   // gathered 16-byte pieces of a stage per producer thread
  constexpr int kRowStep = kProducers / 8;         // rows covered by one pass of all producer threads
  constexpr uint32_t kIdesc = idesc_bf16(128, kN, false, false);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align_up<1024>(smem_raw);
  uint8_t *sA = smem;
  uint8_t *sB = smem + C::kBOff;
  float *part = reinterpret_cast<float *>(smem + C::kPartOff);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
  uint64_t *empty = full + S;
  uint64_t *acc_full = empty + S;     // [2]
  uint64_t *acc_empty = acc_full + 2; // [2]
  uint64_t *part_bar = acc_empty + 2; // refresh: the four token quarters' partial scores are written / read
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(part_bar + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (*(volatile int *)p.status != kDevOk) return;
  const bool sparse = p.mode == kUpDelta;
  const int kcols = sparse ? p.k : p.H;                 // columns of the block that are computed
  const int nch = (kcols + kN - 1) / kN;
  const int ntiles = p.nb * nch;
  const int my_tiles = static_cast<int>(blockIdx.x) < ntiles
                           ? (ntiles - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                           : 0;
  const int nk = p.D / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], DENSE ? 1 : 1 + kProducers);   // the TMA thread (+ every gathering thread)
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], 32 * C::kEpiWarps);
    }
    mbar_init(part_bar, 32 * C::kEpiWarps);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (threadIdx.x == kTmaWarp * 32) {
    prefetch_tmap(&tm_w1t);
    prefetch_tmap(&tm_x);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < C::kProdWarps) {
    // gathered W1^T rows: thread pt moves 16-byte piece (pt & 7) of rows
    // i * kRowStep + (pt >> 3), i = 0 .. kRowIters - 1
    if (!DENSE) {
      const int pt = threadIdx.x;
      uint32_t dst_off[kRowIters];
#pragma unroll
      for (int i = 0; i < kRowIters; ++i) dst_off[i] = sw128_offset(i * kRowStep + (pt >> 3), pt & 7);
      // this thread's selected columns of the CTA's tile tl, loaded one tile
      // ahead and range-checked when they are used
      auto load_rows = [&](int tl, int *c) {
        const int tile = blockIdx.x + tl * gridDim.x;
        const TileAt ta = tile_at(tile, p.nb, nch, p.group);
        const int chunk = ta.part, b = ta.b;
#pragma unroll
        for (int i = 0; i < kRowIters; ++i)
          c[i] = tl < my_tiles ? __ldg(p.idx + static_cast<size_t>(b) * p.k +
                                      min(chunk * kN + i * kRowStep + (pt >> 3), p.k - 1))
                               : 0;
      };
      int nxt[kRowIters];
      load_rows(0, nxt);
      const uint32_t b_base = smem_u32(sB);
      int kg = 0;
      bool ok = true;
      for (int tl = 0; tl < my_tiles && ok; ++tl) {
        const uint16_t *src_row[kRowIters];
#pragma unroll
        for (int i = 0; i < kRowIters; ++i) {
          int c = nxt[i];
          if (static_cast<unsigned>(c) >= static_cast<unsigned>(p.H)) {  // never address outside the weights
            atomicCAS(p.status, kDevOk, kDevBadIndex);
            c = 0;
          }
          src_row[i] = p.w1t + static_cast<size_t>(c) * p.D + (pt & 7) * 8;
        }
        load_rows(tl + 1, nxt);
        for (int kb = 0; kb < nk; ++kb, ++kg) {
          const int s = kg % S;
          if (!wait_warp(&empty[s], ((kg / S) & 1) ^ 1, p.status, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t stage = b_base + s * C::kBBytes;
#pragma unroll
          for (int i = 0; i < kRowIters; ++i) cp_async_16(stage + dst_off[i], src_row[i] + kb * kBK);
          cp_async_arrive_noinc(&full[s]);
        }
      }
    }
  } else if (warp == kTmaWarp) {
    // x tiles (and, on a refresh, the consecutive W1^T rows) by TMA
    int kg = 0;
    bool ok = true;
    for (int tl = 0; tl < my_tiles && ok; ++tl) {
      const int tile = blockIdx.x + tl * gridDim.x;
      const TileAt ta = tile_at(tile, p.nb, nch, p.group);
      const int chunk = ta.part, b = ta.b;
      for (int kb = 0; kb < nk; ++kb, ++kg) {
        const int s = kg % S;
        if (!wait_warp(&empty[s], ((kg / S) & 1) ^ 1, p.status, abort_flag)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[s], DENSE ? C::kABytes + C::kBBytes : C::kABytes);
          tma_load_2d(sA + s * C::kABytes, &tm_x, &full[s], kb * kBK, b * BT);
          if (DENSE) {
#pragma unroll
            for (int h = 0; h < kN / 128; ++h)
              tma_load_2d(sB + s * C::kBBytes + h * 16384, &tm_w1t, &full[s], kb * kBK, chunk * kN + h * 128);
          }
        }
        __syncwarp();
      }
    }
  } else if (warp == kMmaWarp) {
    int kg = 0;
    bool ok = true;
    for (int tl = 0; tl < my_tiles && ok; ++tl) {
      const int ab = tl & 1;
      const uint32_t tacc = tmem + ab * kN;
      if (!wait_warp(&acc_empty[ab], ((tl >> 1) & 1) ^ 1, p.status, abort_flag)) break;
      tc_fence_after();
      for (int kb = 0; kb < nk; ++kb, ++kg) {
        const int s = kg % S;
        if (!wait_warp(&full[s], (kg / S) & 1, p.status, abort_flag)) {
          ok = false;
          break;
        }
        if (!DENSE) fence_async_smem();
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a0 = smem_u32(sA + s * C::kABytes);
          const uint32_t b0 = smem_u32(sB + s * C::kBBytes);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            umma_bf16(tacc, sdesc_sw128(a0 + kk * 32, 16, 1024), sdesc_sw128(b0 + kk * 32, 16, 1024), kIdesc,
                      (kb | kk) != 0);
          umma_commit(&empty[s]);
        }
        __syncwarp();
      }
      if (ok && lane == 0) umma_commit(&acc_full[ab]);
      __syncwarp();
    }
  } else {
    // epilogue: warp of lane quadrant q = tokens 32q .. 32q + 31, 32 columns at a time
    const int q = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const bool first = p.mode == kUpRefreshFirst;
    float *tr = reinterpret_cast<float *>(smem + C::kTrOff) + (warp - C::kEpiWarp0) * (32 * 33);
    uint8_t *tb = smem + C::kTbOff + (warp - C::kEpiWarp0) * (32 * 80);
    const int ck = lane & 3, cq = lane >> 2;   // run piece and column (8 i + cq) this lane moves
    uint32_t part_phase = 0;
    for (int tl = 0; tl < my_tiles; ++tl) {
      const int tile = blockIdx.x + tl * gridDim.x;
      const TileAt ta = tile_at(tile, p.nb, nch, p.group);
      const int chunk = ta.part, b = ta.b;
      const int ab = tl & 1;
      const int nvalid = min(BT, p.T - b * BT);
      // hidden unit of column j = chunk * kN + 32 cc + lane, for all chunks cc
      // of the tile at once (one load latency), range-checked here
      int c_of[kN / 32];
#pragma unroll
      for (int cc = 0; cc < kN / 32; ++cc) {
        const int j = chunk * kN + cc * 32 + lane;
        if (sparse) {
          c_of[cc] = __ldg(p.idx + static_cast<size_t>(b) * p.k + min(j, p.k - 1));
        } else {
          c_of[cc] = min(j, p.H - 1);
        }
      }
      uint32_t bad = 0;   // bit cc: this lane's column of chunk cc had an index out of range and is dropped
#pragma unroll
      for (int cc = 0; cc < kN / 32; ++cc) {
        if (static_cast<unsigned>(c_of[cc]) >= static_cast<unsigned>(p.H)) {  // never address outside the cache
          atomicCAS(p.status, kDevOk, kDevBadIndex);
          c_of[cc] = 0;
          bad |= 1u << cc;
        }
      }
      // old activations of tokens 32q .. 32q + 31 for the columns 8 i + cq of chunk cc, and the bias
      const size_t a_off = static_cast<size_t>(b) * p.H * BT + q * 32 + ck * 8;
      auto load_old = [&](int cc, uint4 (&pre)[4], float &bias) {
        const int c = c_of[cc];
        const bool need_old = chunk * kN + cc * 32 + lane < kcols && !((bad >> cc) & 1u) && !(first && !sparse);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int ci = __shfl_sync(0xffffffffu, c, 8 * i + cq);
          const bool ni = __shfl_sync(0xffffffffu, need_old, 8 * i + cq);
          pre[i] = ni ? *reinterpret_cast<const uint4 *>(p.a_cache + a_off + static_cast<size_t>(ci) * BT)
                      : make_uint4(0, 0, 0, 0);
        }
        bias = bf16_bits_to_f32(__ldg(p.b1 + c));
      };
      uint4 pre[4];
      float bias;
      load_old(0, pre, bias);
      if (!wait_warp(&acc_full[ab], (tl >> 1) & 1, p.status, abort_flag)) break;
      tc_fence_after();
#pragma unroll 1
      for (int cc = 0; cc < kN / 32; ++cc) {
        const int c = c_of[cc];
        const bool valid_j = chunk * kN + cc * 32 + lane < kcols && !((bad >> cc) & 1u);
        // old activations into the run buffer, then this thread's column out of it;
        // the next chunk's are requested right away
#pragma unroll
        for (int i = 0; i < 4; ++i) *reinterpret_cast<uint4 *>(tb + (8 * i + cq) * 80 + ck * 16) = pre[i];
        const float bias_c = bias;
        if (cc + 1 < kN / 32) load_old(cc + 1, pre, bias);
        __syncwarp();
        uint4 oldw[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) oldw[u] = *reinterpret_cast<const uint4 *>(tb + lane * 80 + u * 16);
        // accumulator chunk: lane = token, 32 columns; turned around so that lane = column
        {
          float acc[32];
          tmem_ld32(tmem + lane_off + ab * kN + cc * 32, acc);
          if (cc == kN / 32 - 1) {
            tc_fence_before();
            mbar_arrive(&acc_empty[ab]);  // the accumulator can take the next-but-one tile
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) tr[lane * 33 + i] = acc[i];
        }
        __syncwarp();
        float v[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) v[t] = tr[t * 33 + lane];
        const uint16_t *old = reinterpret_cast<const uint16_t *>(oldw);
        float score = 0.f;
        uint32_t na[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          uint16_t nab[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const float a = gelu_tanh(v[i + u] + bias_c);
            const bool tok = q * 32 + i + u < nvalid;
            nab[u] = tok ? f32_to_bf16_bits(a) : old[i + u];
            if (!sparse) score += tok ? fabsf(first ? a : a - bf16_bits_to_f32(old[i + u])) : 0.f;
          }
          na[i / 2] = static_cast<uint32_t>(nab[0]) | (static_cast<uint32_t>(nab[1]) << 16);
        }
        // new activations back out as whole runs
        __syncwarp();
#pragma unroll
        for (int u = 0; u < 4; ++u)
          *reinterpret_cast<uint4 *>(tb + lane * 80 + u * 16) = make_uint4(na[4 * u], na[4 * u + 1], na[4 * u + 2], na[4 * u + 3]);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int ci = __shfl_sync(0xffffffffu, c, 8 * i + cq);
          if (__shfl_sync(0xffffffffu, valid_j, 8 * i + cq))
            *reinterpret_cast<uint4 *>(p.a_cache + a_off + static_cast<size_t>(ci) * BT) =
                *reinterpret_cast<const uint4 *>(tb + (8 * i + cq) * 80 + ck * 16);
        }
        if (sparse) {
          // delta = bf16(new) - old for real tokens of a selected column, else 0;
          // rows up to the padded width are written, none beyond it
          const uint16_t *nw = reinterpret_cast<const uint16_t *>(na);
          uint32_t dl[16];
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            uint16_t dlb[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const bool tok = q * 32 + i + u < nvalid;
              dlb[u] = (valid_j && tok) ? f32_to_bf16_bits(bf16_bits_to_f32(nw[i + u]) - bf16_bits_to_f32(old[i + u]))
                                        : static_cast<uint16_t>(0);
            }
            dl[i / 2] = static_cast<uint32_t>(dlb[0]) | (static_cast<uint32_t>(dlb[1]) << 16);
          }
          __syncwarp();
#pragma unroll
          for (int u = 0; u < 4; ++u)
            *reinterpret_cast<uint4 *>(tb + lane * 80 + u * 16) = make_uint4(dl[4 * u], dl[4 * u + 1], dl[4 * u + 2], dl[4 * u + 3]);
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int jr = chunk * kN + cc * 32 + 8 * i + cq;
            if (jr < p.k_pad)
              *reinterpret_cast<uint4 *>(p.delta + (static_cast<size_t>(b) * p.k_pad + jr) * BT + q * 32 + ck * 8) =
                  *reinterpret_cast<const uint4 *>(tb + (8 * i + cq) * 80 + ck * 16);
          }
        } else {
          part[q * kN + cc * 32 + lane] = score;
        }
        __syncwarp();  // the buffers take the next chunk
      }
      if (!sparse) {
        // column score = the four token quarters' partial sums, added in a fixed order
        mbar_arrive(part_bar);
        if (!wait_warp(part_bar, part_phase & 1, p.status, abort_flag)) break;
        ++part_phase;
        for (int col = (warp - C::kEpiWarp0) * 32 + lane; col < kN; col += 32 * C::kEpiWarps) {
          const int j = chunk * kN + col;
          if (j < kcols)
            p.scores[static_cast<size_t>(b) * p.H + j] =
                ((part[col] + part[kN + col]) + part[2 * kN + col]) + part[3 * kN + col];
        }
        mbar_arrive(part_bar);   // the partials have been read: the next tile may overwrite them
        if (!wait_warp(part_bar, part_phase & 1, p.status, abort_flag)) break;
        ++part_phase;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, C::kTmemCols);
}

template <int BN>
struct DownCfg : Roles<8, 4> {   // eight gathering warps: the W2 stream is bound by cp.async issue per warp
  static constexpr int kCtasPerSm = 1;
  static constexpr int kAccs = 2;                        // TMEM accumulators (kAccs * BN columns)
  static constexpr int kStagesA = 3;                     // delta tile
  static constexpr int kStagesB = BN == 256 ? 5 : 8;     // gathered W2 rows
  static constexpr uint32_t kABytes = 128 * 128;         // 64 K-rows x 128 tokens (two 64-token atoms)
  static constexpr uint32_t kBBytes = (BN / 64) * 8192;  // 64 K-rows x BN columns
  static constexpr uint32_t kBOff = kStagesA * kABytes;
  static constexpr uint32_t kBarOff = kBOff + kStagesB * kBBytes;
  static constexpr uint32_t kEpiOff = kBarOff + 1024;   // per epilogue warp: 32 x 33 fp32 transpose buffer
  static constexpr uint32_t kSmem = 1024 + kEpiOff + kEpiWarps * 32 * 33 * 4;
  static_assert(kSmem <= 232448, "over the shared memory of one CTA");
};

// Persistent: CTA c handles tiles c, c + gridDim.x, ...; the two TMEM
// accumulators alternate between tiles so the epilogue of one tile overlaps
// the main loop of the next. Ring stages and their parities follow one
// running k-step counter across tiles.
//
// F8: the FP8 form of the sparse step. The delta codes and the gathered W2
// rows are e4m3: a stage holds 128 K-rows (selected columns) of 128-byte
// rows, the delta tile (128 tokens) arrives by one TMA load, the W2 row
// segments (BN bytes) form BN / 128 slabs of 128 columns, the tensor core runs
// kind::f8f6f4 (K = 32 per instruction) and the epilogue scales the result by
// the deltas' scale before adding it to the output cache.
template <int BT, int BN, bool DENSE, bool F8 = false>
__global__ void __launch_bounds__(DownCfg<BN>::kThreads, DownCfg<BN>::kCtasPerSm)
    mlp_down_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_w2,
                    const MlpDownParams p) {
  using C = DownCfg<BN>;
  static_assert(!F8 || (BT == 128 && BN == 256 && !DENSE), "the FP8 step runs the sparse form, 128 x 256 tiles");
  constexpr int SA = C::kStagesA, SB = C::kStagesB;
  constexpr int kProducers = C::kProducers, kMmaWarp = C::kMmaWarp, kTmaWarp = C::kTmaWarp, kThreads = C::kThreads;
  constexpr int kEs = F8 ? 1 : 2;                     // bytes per operand element
  constexpr int kKStage = 128 / kEs;                  // K rows (selected columns) per stage
  constexpr int kRowsPerWarp = kKStage / C::kProdWarps;   // gathered W2 rows of a stage per producer warp
  constexpr uint32_t kIdesc = F8 ? idesc_e4m3(128, BN, true, true) : idesc_bf16(128, BN, true, true);
  constexpr uint32_t kATx = F8 ? 16384 : (BT / 64) * 8192;
  constexpr int kChunksPerRow = BN * kEs / 16;        // 16-byte chunks of one gathered W2 row segment
  constexpr int kRowsPerInstr = 32 / kChunksPerRow;   // rows one warp instruction covers
  constexpr uint32_t kSlabBytes = kKStage * 128;      // one 128-byte-wide column slab of a B stage
  constexpr uint32_t kKStep = (F8 ? 32 : 16) * 128;   // bytes of the 128-byte K rows one MMA consumes
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align_up<1024>(smem_raw);
  uint8_t *sA = smem;
  uint8_t *sB = smem + C::kBOff;
  uint64_t *a_full = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
  uint64_t *a_empty = a_full + SA;
  uint64_t *b_full = a_empty + SA;
  uint64_t *b_empty = b_full + SB;
  uint64_t *acc_full = b_empty + SB;   // [2]
  uint64_t *acc_empty = acc_full + 2;  // [2]
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (*(volatile int *)p.status != kDevOk) return;
  const int ntiles = p.nb * p.n_slices;
  const int kext = DENSE ? p.krows : p.k;
  const int nk = (kext + kKStage - 1) / kKStage;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SA; ++s) {
      mbar_init(&a_full[s], 1);
      mbar_init(&a_empty[s], 1);
    }
    for (int s = 0; s < SB; ++s) {
      mbar_init(&b_full[s], DENSE ? 1 : kProducers);
      mbar_init(&b_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], 128);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (threadIdx.x == kTmaWarp * 32) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_w2);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, C::kAccs * BN);
    tmem_relinquish();
  }
  if (BT == 64) {
    // tokens 64..127 of every A stage stay zero: the MMA always runs M = 128
    for (int s = 0; s < SA; ++s) {
      uint4 *z = reinterpret_cast<uint4 *>(sA + s * C::kABytes + 8192);
      for (int i = threadIdx.x; i < 8192 / 16; i += kThreads) z[i] = make_uint4(0, 0, 0, 0);
    }
    fence_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // grouped, slice-major in a group (tile_at): CTAs running at the same time
  // share an N slice and sweep their (ascending) W2 rows in the same order (L2
  // reuse), and a group's delta tiles stay in L2 while its slices are done
  if (warp < C::kProdWarps) {
    // gathered W2 rows: warp pw moves rows pw*R .. pw*R+R-1 (R = kRowsPerWarp) of each 64-row stage
    if (!DENSE) {
      const int pw = warp;
      const int csub = lane % kChunksPerRow;           // chunk of the row segment this lane moves
      const int rsub = lane / kChunksPerRow;           // row within one instruction
      const uint32_t b_base = smem_u32(sB);
      const int my_tiles = static_cast<int>(blockIdx.x) < ntiles
                               ? (ntiles - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                               : 0;
      const int total = my_tiles * nk;
      // Stage kg runs over this CTA's tiles; lanes < R hold the index of row
      // pw*R + lane. Each index is loaded four stages before its copies are
      // issued, into a register nothing reads until then (the loop body is
      // unrolled four times, so no move waits on a pending load); its range
      // is checked only when it is used.
      // the tile's block and slice are worked out once per tile, not per stage
      int ltile = blockIdx.x, lkb = 0;                 // stage whose index is loaded next
      const int32_t *lrow = p.idx + static_cast<size_t>(tile_at(ltile, p.nb, p.n_slices, p.group).b) * p.k;
      auto load_idx = [&]() -> int {
        int c = 0;
        if (lane < kRowsPerWarp && ltile < ntiles) c = __ldg(lrow + min(lkb * kKStage + pw * kRowsPerWarp + lane, p.k - 1));
        if (++lkb == nk) {
          lkb = 0;
          ltile += gridDim.x;
          if (ltile < ntiles) lrow = p.idx + static_cast<size_t>(tile_at(ltile, p.nb, p.n_slices, p.group).b) * p.k;
        }
        return c;
      };
      int tile = blockIdx.x, kb = 0;                   // stage whose copies are issued next
      int n0 = tile_at(tile, p.nb, p.n_slices, p.group).part * BN;
      auto issue = [&](int kg, int c) -> bool {
        const int s = kg % SB;
        if (static_cast<unsigned>(c) >= static_cast<unsigned>(p.H)) {
          atomicCAS(p.status, kDevOk, kDevBadIndex);
          c = 0;
        }
        if (!wait_warp(&b_empty[s], ((kg / SB) & 1) ^ 1, p.status, abort_flag)) return false;
        const uint32_t stage = b_base + s * C::kBBytes;
#pragma unroll
        for (int i = 0; i < kRowsPerWarp / kRowsPerInstr; ++i) {
          const int rr = i * kRowsPerInstr + rsub;   // row within this warp's rows
          const int r = pw * kRowsPerWarp + rr;      // row of the stage
          const int cr = __shfl_sync(0xffffffffu, c, rr);
          const int slab = csub >> 3, cc = csub & 7;
          cp_async_16(stage + slab * kSlabBytes + sw128_offset(r, cc),
                      reinterpret_cast<const uint8_t *>(p.w2) + (static_cast<size_t>(cr) * p.D + n0) * kEs + csub * 16);
        }
        cp_async_arrive_noinc(&b_full[s]);
        if (++kb == nk) {
          kb = 0;
          tile += gridDim.x;
          if (tile < ntiles) n0 = tile_at(tile, p.nb, p.n_slices, p.group).part * BN;
        }
        return true;
      };
      int c0 = load_idx(), c1 = load_idx(), c2 = load_idx(), c3 = load_idx();
      for (int kg = 0; kg < total; kg += 4) {
        if (!issue(kg, c0)) break;
        c0 = load_idx();
        if (kg + 1 >= total || !issue(kg + 1, c1)) break;
        c1 = load_idx();
        if (kg + 2 >= total || !issue(kg + 2, c2)) break;
        c2 = load_idx();
        if (kg + 3 >= total || !issue(kg + 3, c3)) break;
        c3 = load_idx();
      }
    }
  } else if (warp == kTmaWarp) {
    // delta / activation tiles (and, on a refresh, the consecutive W2 rows) by TMA
    int kg = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
      const TileAt ta = tile_at(tile, p.nb, p.n_slices, p.group);
      const int b = ta.b, n0 = ta.part * BN;
      for (int kb = 0; kb < nk; ++kb, ++kg) {
        if (DENSE) {
          const int s = kg % SB;
          if (!wait_warp(&b_empty[s], ((kg / SB) & 1) ^ 1, p.status, abort_flag)) {
            ok = false;
            break;
          }
          if (lane == 0) {
            mbar_arrive_expect_tx(&b_full[s], C::kBBytes);
#pragma unroll
            for (int ns = 0; ns < BN / 64; ++ns)
              tma_load_2d(sB + s * C::kBBytes + ns * 8192, &tm_w2, &b_full[s], n0 + ns * 64, kb * kBK);
          }
        }
        const int s = kg % SA;
        if (!wait_warp(&a_empty[s], ((kg / SA) & 1) ^ 1, p.status, abort_flag)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&a_full[s], kATx);
          if (F8) {
            tma_load_3d(sA + s * C::kABytes, &tm_a, &a_full[s], 0, kb * kKStage, b);
          } else {
#pragma unroll
            for (int mt = 0; mt < BT / 64; ++mt)
              tma_load_3d(sA + s * C::kABytes + mt * 8192, &tm_a, &a_full[s], mt * 64, kb * kBK, b);
          }
        }
        __syncwarp();
      }
    }
  } else if (warp == kMmaWarp) {
    int kg = 0, tl = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++tl) {
      const int ab = tl % C::kAccs;
      const uint32_t tacc = tmem + ab * BN;
      if (!wait_warp(&acc_empty[ab], ((tl / C::kAccs) & 1) ^ 1, p.status, abort_flag)) break;
      tc_fence_after();
      for (int kb = 0; kb < nk; ++kb, ++kg) {
        const int sa = kg % SA, sb = kg % SB;
        if (!wait_warp(&a_full[sa], (kg / SA) & 1, p.status, abort_flag) ||
            !wait_warp(&b_full[sb], (kg / SB) & 1, p.status, abort_flag)) {
          ok = false;
          break;
        }
        if (!DENSE) fence_async_smem();
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a0 = smem_u32(sA + sa * C::kABytes);
          const uint32_t b0 = smem_u32(sB + sb * C::kBBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            // MN-major: A atoms of 128 bytes of tokens (two 64-token atoms 8 KB apart for bf16, one
            // 128-token atom for e4m3), B slabs kSlabBytes apart, 8-row groups 1 KB apart
            const uint64_t ad = sdesc_sw128(a0 + kk * kKStep, 8192, 1024);
            const uint64_t bd = sdesc_sw128(b0 + kk * kKStep, kSlabBytes, 1024);
            if (F8)
              umma_e4m3(tacc, ad, bd, kIdesc, (kb | kk) != 0);
            else
              umma_bf16(tacc, ad, bd, kIdesc, (kb | kk) != 0);
          }
          umma_commit(&a_empty[sa]);
          umma_commit(&b_empty[sb]);
        }
        __syncwarp();
      }
      if (ok && lane == 0) umma_commit(&acc_full[ab]);
      __syncwarp();
    }
  } else {
    // epilogue: warp w reads TMEM lane quadrant q = w % 4 (tokens 32q ..
    // 32q + 31, one per thread) 32 columns at a time and turns the chunk
    // around in its shared buffer (rows padded to 33 words, so both the
    // row-wise writes and the column-wise reads are free of bank conflicts);
    // then eight lanes cover one token's 32 columns, and every access to the
    // output cache and the layer output is a whole 128-byte (64-byte) run.
    static_assert(C::kEpiWarps == 4, "one epilogue warp per TMEM lane quadrant");
    const int q = warp & 3;
    float *ebuf = reinterpret_cast<float *>(smem + C::kEpiOff) + (warp - C::kEpiWarp0) * (32 * 33);
    const int rsub = lane >> 3, c4 = (lane & 7) * 4;   // row within a group of four, first column
    const bool accumulate = p.mode == kDownAccumulate;
    int tl = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++tl) {
      const TileAt ta = tile_at(tile, p.nb, p.n_slices, p.group);
      const int b = ta.b, n0 = ta.part * BN;
      const int ab = tl % C::kAccs;
      if (!wait_warp(&acc_full[ab], (tl / C::kAccs) & 1, p.status, abort_flag)) break;
      tc_fence_after();
#pragma unroll 1
      for (int nc = 0; nc < BN / 32; ++nc) {
        float acc[32];
        tmem_ld32(tmem + ab * BN + (static_cast<uint32_t>(q * 32) << 16) + nc * 32, acc);
        if (nc == BN / 32 - 1) {
          tc_fence_before();
          mbar_arrive(&acc_empty[ab]);  // the accumulator can take the next-but-one tile
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) ebuf[lane * 33 + i] = acc[i];
        __syncwarp();
        const int n = n0 + nc * 32 + c4;
        float4 old[8];
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const int r = q * 32 + 4 * g + rsub;               // token within the block
          const int64_t grow = static_cast<int64_t>(b) * BT + r;
          if (accumulate && r < BT && grow < p.T)
            old[g] = *reinterpret_cast<const float4 *>(p.y_cache + grow * p.D + n);
        }
        float4 bias = make_float4(0.f, 0.f, 0.f, 0.f);
        if (!accumulate)
          bias = make_float4(bf16_bits_to_f32(__ldg(p.b2 + n)), bf16_bits_to_f32(__ldg(p.b2 + n + 1)),
                             bf16_bits_to_f32(__ldg(p.b2 + n + 2)), bf16_bits_to_f32(__ldg(p.b2 + n + 3)));
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const int rr = 4 * g + rsub;                       // row of the warp's quadrant
          const int r = q * 32 + rr;
          const int64_t grow = static_cast<int64_t>(b) * BT + r;
          if (r < BT && grow < p.T) {
            const float *e = ebuf + rr * 33 + c4;
            const float4 base = accumulate ? old[g] : bias;
            const float sd = F8 ? p.s_delta : 1.f;
            const float4 y = F8 ? make_float4(fmaf(e[0], sd, base.x), fmaf(e[1], sd, base.y), fmaf(e[2], sd, base.z),
                                              fmaf(e[3], sd, base.w))
                                : make_float4(base.x + e[0], base.y + e[1], base.z + e[2], base.w + e[3]);
            *reinterpret_cast<float4 *>(p.y_cache + grow * p.D + n) = y;
            if (p.out != nullptr)
              *reinterpret_cast<uint2 *>(p.out + grow * p.D + n) = make_uint2(cvt_bf16x2(y.x, y.y), cvt_bf16x2(y.z, y.w));
          }
        }
        __syncwarp();  // the buffer is rewritten by the next chunk
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, C::kAccs * BN);
}

// out = bf16(y) when a sparse step selects nothing
__global__ void y_to_out_kernel(const float4 *__restrict__ y, uint2 *__restrict__ out, int64_t n4) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 v = y[i];
    out[i] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
  }
}

template <typename K>
cudaError_t set_smem(K kernel, uint32_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
}

template <int BT, bool DENSE>
cudaError_t launch_up_t(const MlpUpParams &p, const CUtensorMap &w, const CUtensorMap &x, cudaStream_t s) {
  using C = UpCfg<BT>;
  cudaError_t e = set_smem(mlp_up_kernel<BT, DENSE>, C::kSmem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t grid = std::min<int64_t>(static_cast<int64_t>(p.nb) * p.nchunks, static_cast<int64_t>(sms) * C::kCtasPerSm);
  mlp_up_kernel<BT, DENSE><<<static_cast<unsigned>(grid), C::kThreads, C::kSmem, s>>>(w, x, p);
  return cudaGetLastError();
}

template <int N, bool DENSE>
cudaError_t launch_up_wide(const MlpUpParams &p, const CUtensorMap &w, const CUtensorMap &x, cudaStream_t s) {
  using C = UpWideCfg<N>;
  cudaError_t e = set_smem(mlp_up_wide_kernel<N, DENSE>, C::kSmem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int kcols = p.mode == kUpDelta ? p.k : p.H;
  const int64_t tiles = static_cast<int64_t>(p.nb) * ((kcols + C::kN - 1) / C::kN);
  const int64_t grid = std::min<int64_t>(tiles, sms);
  mlp_up_wide_kernel<N, DENSE><<<static_cast<unsigned>(grid), C::kThreads, C::kSmem, s>>>(w, x, p);
  return cudaGetLastError();
}

template <int BT, int BN, bool DENSE>
cudaError_t launch_down_t(const MlpDownParams &p, const CUtensorMap &a, const CUtensorMap &w, cudaStream_t s) {
  using C = DownCfg<BN>;
  cudaError_t e = set_smem(mlp_down_kernel<BT, BN, DENSE>, C::kSmem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t grid = std::min<int64_t>(static_cast<int64_t>(p.nb) * p.n_slices, static_cast<int64_t>(sms) * C::kCtasPerSm);
  mlp_down_kernel<BT, BN, DENSE><<<static_cast<unsigned>(grid), C::kThreads, C::kSmem, s>>>(a, w, p);
  return cudaGetLastError();
}

template <int BT, bool DENSE>
cudaError_t launch_down_bn(const MlpDownParams &p, const CUtensorMap &a, const CUtensorMap &w, cudaStream_t s) {
  switch (p.bn) {
    case 256: return launch_down_t<BT, 256, DENSE>(p, a, w, s);
    case 128: return launch_down_t<BT, 128, DENSE>(p, a, w, s);
    case 64: return launch_down_t<BT, 64, DENSE>(p, a, w, s);
    default: return cudaErrorInvalidValue;
  }
}

// out = bf16(y_cache) when a sparse step selects nothing
cudaError_t y_to_out(const MlpDownParams &p, cudaStream_t s) {
  if (p.out == nullptr) return cudaSuccess;
  const int64_t n4 = static_cast<int64_t>(p.T) * p.D / 4;
  y_to_out_kernel<<<static_cast<unsigned>(std::min<int64_t>((n4 + 255) / 256, 148 * 16)), 256, 0, s>>>(
      reinterpret_cast<const float4 *>(p.y_cache), reinterpret_cast<uint2 *>(p.out), n4);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_mlp_up_fp8(const MlpUpParams &p0, const CUtensorMap &tm_x, cudaStream_t s) {
  MlpUpParams p = p0;
  p.group = up_tile_group(p.nb, static_cast<int64_t>(p.Bt) * p.D);   // e4m3 x tiles
  if (p.nb <= 0 || p.nchunks <= 0) return cudaSuccess;
  if (p.Bt != 128 || p.mode != kUpDelta) return cudaErrorInvalidValue;
  using C = UpCfg<128>;
  cudaError_t e = set_smem(mlp_up_kernel<128, false, true>, C::kSmem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t grid = std::min<int64_t>(static_cast<int64_t>(p.nb) * p.nchunks, static_cast<int64_t>(sms) * C::kCtasPerSm);
  // the W1^T tile map serves the refresh only; a sparse step gathers the rows itself
  mlp_up_kernel<128, false, true><<<static_cast<unsigned>(grid), C::kThreads, C::kSmem, s>>>(tm_x, tm_x, p);
  return cudaGetLastError();
}

cudaError_t launch_mlp_down_fp8(const MlpDownParams &p0, const CUtensorMap &tm_a, cudaStream_t s) {
  MlpDownParams p = p0;
  p.group = down_tile_group(p.nb, false, 0);
  if (p.nb <= 0) return cudaSuccess;
  if (p.k <= 0) return y_to_out(p, s);
  if (p.Bt != 128 || p.bn != 256 || p.mode != kDownAccumulate) return cudaErrorInvalidValue;
  using C = DownCfg<256>;
  cudaError_t e = set_smem(mlp_down_kernel<128, 256, false, true>, C::kSmem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t grid = std::min<int64_t>(static_cast<int64_t>(p.nb) * p.n_slices, static_cast<int64_t>(sms) * C::kCtasPerSm);
  // the W2 tile map serves the refresh only; a sparse step gathers the rows itself
  mlp_down_kernel<128, 256, false, true><<<static_cast<unsigned>(grid), C::kThreads, C::kSmem, s>>>(tm_a, tm_a, p);
  return cudaGetLastError();
}

cudaError_t launch_mlp_up(const MlpUpParams &p0, const CUtensorMap &tm_w1t, const CUtensorMap &tm_x, cudaStream_t s) {
  MlpUpParams p = p0;
  p.group = up_tile_group(p.nb, static_cast<int64_t>(p.Bt) * p.D * 2);   // bf16 x tiles
  if (p.nb <= 0 || p.nchunks <= 0) return cudaSuccess;
  const bool dense = p.mode != kUpDelta;
  if (p.Bt == 128) return dense ? launch_up_wide<256, true>(p, tm_w1t, tm_x, s) : launch_up_t<128, false>(p, tm_w1t, tm_x, s);
  if (p.Bt == 64) return dense ? launch_up_t<64, true>(p, tm_w1t, tm_x, s) : launch_up_t<64, false>(p, tm_w1t, tm_x, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_mlp_down(const MlpDownParams &p0, const CUtensorMap &tm_a, const CUtensorMap &tm_w2, bool dense,
                            cudaStream_t s) {
  MlpDownParams p = p0;
  p.group = down_tile_group(p.nb, dense, static_cast<int64_t>(p.krows) * p.Bt * 2);   // bf16 activation-cache tiles
  if (p.nb <= 0) return cudaSuccess;
  const int kext = dense ? p.krows : p.k;
  if (kext <= 0) return y_to_out(p, s);
  if (p.Bt == 128) return dense ? launch_down_bn<128, true>(p, tm_a, tm_w2, s) : launch_down_bn<128, false>(p, tm_a, tm_w2, s);
  if (p.Bt == 64) return dense ? launch_down_bn<64, true>(p, tm_a, tm_w2, s) : launch_down_bn<64, false>(p, tm_a, tm_w2, s);
  return cudaErrorInvalidValue;
}

}  // namespace cm
