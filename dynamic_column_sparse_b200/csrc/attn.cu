// attn.cu - attention over a gathered key subset with an online-softmax merge,
// plus the dense passes of the refresh (full attention with row log-sum-exp,
// attention mass per query block, complement partial).
//
// One CTA per (head, 128-query block). Q arrives once by a tiled TMA load; K
// and V stream in chunks of 128 keys through a two-stage ring: on a sparse
// step the producer warps 5-7 gather the selected key rows with 16-byte
// cp.async (one warp instruction = two whole 256-byte key rows), on the dense
// passes one thread issues tiled TMA loads. Warp 4 issues the tcgen05 MMAs:
// S = Q K^T into one of two TMEM buffers, then O_tmp = P V into a third.
// Warps 0-3 run the online softmax, one query row per thread: they
// read S from TMEM, write P (bf16) into a 128-byte-swizzled shared tile that is
// the A operand of the next P V, and fold each O_tmp into a register
// accumulator rescaled by the running max. S of chunk i+1 is computed while the
// softmax of chunk i runs. Logits are kept in log2 units (scale * log2 e).
#include <algorithm>

#include "kernels.cuh"
#include "ptx.cuh"

namespace cm {
namespace {

constexpr int kThreads = 256;
constexpr int kMmaWarp = 4;
constexpr int kProdWarp0 = 5;
constexpr int kProducers = 96;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

constexpr uint32_t kQOff = 0;             // Q: two 64-column halves of [128 rows][128 B]
constexpr uint32_t kKOff = 32768;         // K: 2 stages x 32 KB
constexpr uint32_t kVOff = 98304;         // V: 2 stages x 32 KB
constexpr uint32_t kPOff = 163840;        // P: two 64-key halves of [128 rows][128 B]
constexpr uint32_t kBarOff = 196608;
constexpr uint32_t kMaskOff = kBarOff + 256;
constexpr uint32_t kTileBytes = 32768;

__device__ __forceinline__ bool wait_warp(uint64_t *bar, uint32_t parity, int *status, volatile int *abort_flag) {
  const bool ok = mbar_wait(bar, parity, status, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  constexpr uint32_t kIdescQK = idesc_bf16(128, 128, false, false);
  constexpr uint32_t kIdescPV = idesc_bf16(128, 128, false, true);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align_up<1024>(smem_raw);
  uint8_t *sQ = smem + kQOff;
  uint8_t *sK = smem + kKOff;
  uint8_t *sV = smem + kVOff;
  uint8_t *sP = smem + kPOff;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kBarOff);
  uint64_t *q_full = bars + 0;
  uint64_t *k_full = bars + 1;    // [2]
  uint64_t *v_full = bars + 3;    // [2]
  uint64_t *kv_empty = bars + 5;  // [2]
  uint64_t *s_full = bars + 7;    // [2]
  uint64_t *s_free = bars + 9;    // [2]
  uint64_t *p_full = bars + 11;
  uint64_t *o_full = bars + 12;
  uint64_t *o_free = bars + 13;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 14);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  uint32_t *mask = reinterpret_cast<uint32_t *>(smem + kMaskOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (*(volatile int *)p.status != kDevOk) return;
  const int hh = blockIdx.x % p.h;
  const int b = blockIdx.x / p.h;
  const int T = p.T;
  const int nkeys = MODE == kAttnDelta ? p.k : T;
  const int nchunks = (nkeys + 127) / 128;
  const int32_t *irow = p.idx + (static_cast<size_t>(hh) * p.nb + b) * p.k;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], MODE == kAttnDelta ? kProducers : 1);
      mbar_init(&v_full[s], MODE == kAttnDelta ? kProducers : 1);
      mbar_init(&kv_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 128);
    }
    mbar_init(p_full, 128);
    mbar_init(o_full, 1);
    mbar_init(o_free, 128);
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
  if (MODE == kAttnComplement) {
    const int nwords = (T + 31) >> 5;
    for (int w = threadIdx.x; w < nwords; w += kThreads) mask[w] = 0u;
    __syncthreads();
    for (int j = threadIdx.x; j < p.k; j += kThreads) {
      const int key = __ldg(irow + j);
      if (static_cast<unsigned>(key) < static_cast<unsigned>(T))
        atomicOr(&mask[key >> 5], 1u << (key & 31));
      else
        atomicCAS(p.status, kDevOk, kDevBadIndex);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= kProdWarp0) {
    const int pw = warp - kProdWarp0;
    if (pw == 0 && lane == 0 && nchunks > 0) {
      mbar_arrive_expect_tx(q_full, kTileBytes);
      tma_load_2d(sQ, &tm_q, q_full, hh * 128, b * 128);
      tma_load_2d(sQ + 16384, &tm_q, q_full, hh * 128 + 64, b * 128);
    }
    for (int i = 0; i < nchunks; ++i) {
      const int s = i & 1;
      if (!wait_warp(&kv_empty[s], ((i >> 1) & 1) ^ 1, p.status, abort_flag)) break;
      uint8_t *dk = sK + s * kTileBytes;
      uint8_t *dv = sV + s * kTileBytes;
      if (MODE == kAttnDelta) {
        // warp pw moves key rows 2q and 2q+1 for q = pw, pw+3, ..: lanes 0-15 one row, 16-31 the other
        const int c16 = lane & 15;
        const uint32_t off_half = (c16 >> 3) * 16384;
        const uint32_t k0 = smem_u32(dk), v0 = smem_u32(dv);
        for (int qp = pw; qp < 64; qp += 3) {
          const int r = 2 * qp + (lane >> 4);
          int key = __ldg(irow + min(i * 128 + r, p.k - 1));
          if (static_cast<unsigned>(key) >= static_cast<unsigned>(T)) {
            atomicCAS(p.status, kDevOk, kDevBadIndex);
            key = 0;
          }
          const size_t g = (static_cast<size_t>(key) * p.h + hh) * 128 + c16 * 8;
          const uint32_t o = off_half + sw128_offset(r, c16 & 7);
          cp_async_16(k0 + o, p.k_ptr + g);
          cp_async_16(v0 + o, p.v_ptr + g);
        }
        cp_async_arrive_noinc(&k_full[s]);
        cp_async_arrive_noinc(&v_full[s]);
      } else if (pw == 0 && lane == 0) {
        mbar_arrive_expect_tx(&k_full[s], kTileBytes);
        tma_load_2d(dk, &tm_k, &k_full[s], hh * 128, i * 128);
        tma_load_2d(dk + 16384, &tm_k, &k_full[s], hh * 128 + 64, i * 128);
        mbar_arrive_expect_tx(&v_full[s], kTileBytes);
        tma_load_2d(dv, &tm_v, &v_full[s], hh * 128, i * 128);
        tma_load_2d(dv + 16384, &tm_v, &v_full[s], hh * 128 + 64, i * 128);
      }
      __syncwarp();
    }
  } else if (warp == kMmaWarp) {
    if (nchunks > 0 && wait_warp(q_full, 0, p.status, abort_flag)) {
      tc_fence_after();
      const uint32_t q0 = smem_u32(sQ), p0 = smem_u32(sP);
      for (int i = 0; i <= nchunks; ++i) {
        if (i < nchunks) {
          const int s = i & 1;
          if (!wait_warp(&k_full[s], (i >> 1) & 1, p.status, abort_flag)) break;
          if (!wait_warp(&s_free[s], ((i >> 1) & 1) ^ 1, p.status, abort_flag)) break;
          if (MODE == kAttnDelta) fence_async_smem();
          tc_fence_after();
          if (lane == 0) {
            const uint32_t k0 = smem_u32(sK + s * kTileBytes);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
              umma_bf16(tmem + s * 128, sdesc_sw128(q0 + off, 16, 1024), sdesc_sw128(k0 + off, 16, 1024), kIdescQK,
                        kk > 0);
            }
            umma_commit(&s_full[s]);
          }
          __syncwarp();
        }
        if (i >= 1) {
          const int j = i - 1, s = j & 1;
          if (!wait_warp(p_full, j & 1, p.status, abort_flag)) break;
          if (!wait_warp(&v_full[s], (j >> 1) & 1, p.status, abort_flag)) break;
          if (!wait_warp(o_free, (j & 1) ^ 1, p.status, abort_flag)) break;
          fence_async_smem();
          tc_fence_after();
          if (lane == 0) {
            const uint32_t v0 = smem_u32(sV + s * kTileBytes);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              umma_bf16(tmem + 256, sdesc_sw128(p0 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                        sdesc_sw128(v0 + kk * 2048, 16384, 1024), kIdescPV, kk > 0);
            }
            umma_commit(o_full);
            umma_commit(&kv_empty[s]);
          }
          __syncwarp();
        }
      }
    }
  } else {
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int gi = b * 128 + r;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const float sl2 = p.scale_log2;
    float o_acc[128];
#pragma unroll
    for (int e = 0; e < 128; ++e) o_acc[e] = 0.f;
    float m2 = -INFINITY, l = 0.f;
    bool ok = true;
    for (int i = 0; i < nchunks && ok; ++i) {
      const int sb = i & 1;
      if (!wait_warp(&s_full[sb], (i >> 1) & 1, p.status, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // bit e of live[c]: key slot i*128 + c*32 + e takes part in this pass
      uint32_t live[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int base = i * 128 + c * 32;
        const int lim = (MODE == kAttnDelta ? p.k : T) - base;
        uint32_t m = lim >= 32 ? 0xffffffffu : (lim <= 0 ? 0u : ((1u << lim) - 1u));
        if (MODE == kAttnComplement && lim > 0) m &= ~mask[base >> 5];
        live[c] = m;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float v[32];
        tmem_ld32(tmem + lane_off + sb * 128 + c * 32, v);
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if ((live[c] >> e) & 1u) mx = fmaxf(mx, v[e] * sl2);
      }
      const float m_new = fmaxf(m2, mx);
      const float alpha = (m2 == -INFINITY) ? 0.f : exp2_approx(m2 - m_new);
      if (i >= 1) {
        if (!wait_warp(o_full, (i - 1) & 1, p.status, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float v[32];
          tmem_ld32(tmem + lane_off + 256 + c * 32, v);
#pragma unroll
          for (int e = 0; e < 32; ++e) o_acc[c * 32 + e] += v[e];
        }
        tc_fence_before();
        mbar_arrive(o_free);
      }
#pragma unroll
      for (int e = 0; e < 128; ++e) o_acc[e] *= alpha;
      l *= alpha;
      m2 = m_new;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float v[32];
        tmem_ld32(tmem + lane_off + sb * 128 + c * 32, v);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float pe[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const bool valid = (live[c] >> (e + u)) & 1u;
            pe[u] = (valid && m2 != -INFINITY) ? exp2_approx(v[e + u] * sl2 - m2) : 0.f;
            l += pe[u];
          }
          pk[e / 2] = pack_bf16x2(pe[0], pe[1]);
        }
        uint8_t *prow = sP + (c >> 1) * 16384 + r * 128;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int cc = (c & 1) * 4 + u;
          *reinterpret_cast<uint4 *>(prow + ((cc ^ (r & 7)) << 4)) =
              make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(&s_free[sb]);
      fence_async_smem();
      mbar_arrive(p_full);
    }
    if (ok && nchunks > 0) {
      if (wait_warp(o_full, (nchunks - 1) & 1, p.status, abort_flag)) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float v[32];
          tmem_ld32(tmem + lane_off + 256 + c * 32, v);
#pragma unroll
          for (int e = 0; e < 32; ++e) o_acc[c * 32 + e] += v[e];
        }
      } else {
        ok = false;
      }
    }
    if (ok && gi < T) {
      const size_t row = static_cast<size_t>(hh) * T + gi;
      if (MODE == kAttnDelta) {
        const float mc = p.m_c[row], lc = p.l_c[row];
        const float mc2 = mc * kLog2e;
        const float M = fmaxf(mc2, m2);
        const float wc = (mc == -INFINITY) ? 0.f : exp2_approx(mc2 - M);
        const float ws = (m2 == -INFINITY) ? 0.f : exp2_approx(m2 - M);
        const float L = lc * wc + l * ws;
        const float inv = L > 0.f ? 1.f / L : 0.f;
        const float4 *ac = reinterpret_cast<const float4 *>(p.acc_c + row * 128);
        uint4 *orow = reinterpret_cast<uint4 *>(p.o + (static_cast<size_t>(gi) * p.h + hh) * 128);
#pragma unroll
        for (int e8 = 0; e8 < 16; ++e8) {
          const float4 a0 = ac[2 * e8], a1 = ac[2 * e8 + 1];
          const float *oa = o_acc + 8 * e8;
          orow[e8] = make_uint4(pack_bf16x2((a0.x * wc + oa[0] * ws) * inv, (a0.y * wc + oa[1] * ws) * inv),
                                pack_bf16x2((a0.z * wc + oa[2] * ws) * inv, (a0.w * wc + oa[3] * ws) * inv),
                                pack_bf16x2((a1.x * wc + oa[4] * ws) * inv, (a1.y * wc + oa[5] * ws) * inv),
                                pack_bf16x2((a1.z * wc + oa[6] * ws) * inv, (a1.w * wc + oa[7] * ws) * inv));
        }
      } else if (MODE == kAttnDense) {
        const float inv = l > 0.f ? 1.f / l : 0.f;
        uint4 *orow = reinterpret_cast<uint4 *>(p.o + (static_cast<size_t>(gi) * p.h + hh) * 128);
#pragma unroll
        for (int e8 = 0; e8 < 16; ++e8) {
          const float *oa = o_acc + 8 * e8;
          orow[e8] = make_uint4(pack_bf16x2(oa[0] * inv, oa[1] * inv), pack_bf16x2(oa[2] * inv, oa[3] * inv),
                                pack_bf16x2(oa[4] * inv, oa[5] * inv), pack_bf16x2(oa[6] * inv, oa[7] * inv));
        }
        p.lse[row] = l > 0.f ? (m2 + log2f(l)) * kLn2 : -INFINITY;
      } else {
        p.m_c[row] = (m2 == -INFINITY) ? -INFINITY : m2 * kLn2;
        p.l_c[row] = l;
        float4 *ac = reinterpret_cast<float4 *>(p.acc_c + row * 128);
#pragma unroll
        for (int e4 = 0; e4 < 32; ++e4)
          ac[e4] = make_float4(o_acc[4 * e4], o_acc[4 * e4 + 1], o_acc[4 * e4 + 2], o_acc[4 * e4 + 3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

// Attention mass of each key for one query block: D = K Q^T in TMEM (lane =
// key, column = query), then each thread sums exp2(s - lse) over the block's
// queries for its key.
constexpr uint32_t kMQOff = 0;
constexpr uint32_t kMKOff = 32768;        // 2 stages x 32 KB
constexpr uint32_t kMBarOff = 98304;
constexpr uint32_t kMLseOff = kMBarOff + 256;
constexpr uint32_t kMSmem = 1024 + kMLseOff + 512 + 64;
constexpr int kMassThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 column sums

__global__ void __launch_bounds__(kMassThreads, 1)
    attn_mass_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const MassParams p) {
  constexpr uint32_t kIdesc = idesc_bf16(128, 128, false, false);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align_up<1024>(smem_raw);
  uint8_t *sQ = smem + kMQOff;
  uint8_t *sK = smem + kMKOff;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kMBarOff);
  uint64_t *q_full = bars + 0;
  uint64_t *k_full = bars + 1;   // [2]
  uint64_t *k_empty = bars + 3;  // [2]
  uint64_t *d_full = bars + 5;   // [2]
  uint64_t *d_free = bars + 7;   // [2]
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 9);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  float *lse2 = reinterpret_cast<float *>(smem + kMLseOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (*(volatile int *)p.status != kDevOk) return;
  const int hh = blockIdx.x % p.h;
  const int b = blockIdx.x / p.h;
  const int T = p.T;
  const int nchunks = (T + 127) / 128;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&d_full[s], 1);
      mbar_init(&d_free[s], 128);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  if (threadIdx.x < 128) {
    const int gq = b * 128 + threadIdx.x;
    lse2[threadIdx.x] = gq < T ? p.lse[static_cast<size_t>(hh) * T + gq] * kLog2e : INFINITY;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, kTileBytes);
      tma_load_2d(sQ, &tm_q, q_full, hh * 128, b * 128);
      tma_load_2d(sQ + 16384, &tm_q, q_full, hh * 128 + 64, b * 128);
    }
    for (int i = 0; i < nchunks; ++i) {
      const int s = i & 1;
      if (!wait_warp(&k_empty[s], ((i >> 1) & 1) ^ 1, p.status, abort_flag)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&k_full[s], kTileBytes);
        tma_load_2d(sK + s * kTileBytes, &tm_k, &k_full[s], hh * 128, i * 128);
        tma_load_2d(sK + s * kTileBytes + 16384, &tm_k, &k_full[s], hh * 128 + 64, i * 128);
      }
      __syncwarp();
    }
  } else if (warp == 1) {
    if (wait_warp(q_full, 0, p.status, abort_flag)) {
      tc_fence_after();
      const uint32_t q0 = smem_u32(sQ);
      for (int i = 0; i < nchunks; ++i) {
        const int s = i & 1;
        if (!wait_warp(&k_full[s], (i >> 1) & 1, p.status, abort_flag)) break;
        if (!wait_warp(&d_free[s], ((i >> 1) & 1) ^ 1, p.status, abort_flag)) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t k0 = smem_u32(sK + s * kTileBytes);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            umma_bf16(tmem + s * 128, sdesc_sw128(k0 + off, 16, 1024), sdesc_sw128(q0 + off, 16, 1024), kIdesc, kk > 0);
          }
          umma_commit(&k_empty[s]);
          umma_commit(&d_full[s]);
        }
        __syncwarp();
      }
    }
  } else {
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    float *mrow = p.mass + (static_cast<size_t>(hh) * p.nb + b) * T;
    for (int i = 0; i < nchunks; ++i) {
      const int s = i & 1;
      if (!wait_warp(&d_full[s], (i >> 1) & 1, p.status, abort_flag)) break;
      tc_fence_after();
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float v[32];
        tmem_ld32(tmem + lane_off + s * 128 + c * 32, v);
#pragma unroll
        for (int e = 0; e < 32; ++e) sum += exp2_approx(v[e] * p.scale_log2 - lse2[c * 32 + e]);
      }
      tc_fence_before();
      mbar_arrive(&d_free[s]);
      const int key = i * 128 + r;
      if (key < T) mrow[key] = sum;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 256);
}

template <int MODE>
cudaError_t launch_attn_t(const AttnParams &p, const CUtensorMap &q, const CUtensorMap &k, const CUtensorMap &v,
                          cudaStream_t s) {
  const uint32_t mask_bytes = MODE == kAttnComplement ? ((static_cast<uint32_t>(p.T) + 31) / 32) * 4 : 0;
  const uint32_t smem = 1024 + kMaskOff + mask_bytes;
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t grid = static_cast<int64_t>(p.h) * p.nb;
  attn_kernel<MODE><<<static_cast<unsigned>(grid), kThreads, smem, s>>>(q, k, v, p);
  return cudaGetLastError();
}

}  // namespace

uint32_t attn_smem_bytes(int mode, int64_t T) {
  const uint32_t mask_bytes = mode == kAttnComplement ? ((static_cast<uint32_t>(T) + 31) / 32) * 4 : 0;
  return 1024 + kMaskOff + mask_bytes;
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

cudaError_t launch_attn_mass(const MassParams &p, const CUtensorMap &tm_q, const CUtensorMap &tm_k, cudaStream_t s) {
  if (p.h <= 0 || p.nb <= 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(attn_mass_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kMSmem));
  if (e != cudaSuccess) return e;
  const int64_t grid = static_cast<int64_t>(p.h) * p.nb;
  attn_mass_kernel<<<static_cast<unsigned>(grid), kMassThreads, kMSmem, s>>>(tm_q, tm_k, p);
  return cudaGetLastError();
}

}  // namespace cm
