// kernels.cuh - parameter blocks and host launchers of the library's kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace cm {

// ------------------------------------------------------------------ top-k

struct TopkParams {
  const float *scores;
  int64_t rows, n, ld_scores;
  int32_t k;
  int32_t *idx;
  int64_t ld_idx;
  int *status;
};
cudaError_t launch_topk(const TopkParams &p, cudaStream_t s);

// ------------------------------------------------------------------ cache column gather / scatter

cudaError_t launch_gather_cols(const uint16_t *a_cache, int64_t nb, int64_t H, int Bt, const int32_t *idx, int k,
                               uint16_t *packed, int *status, cudaStream_t s);
cudaError_t launch_scatter_cols(const uint16_t *packed, int64_t nb, int64_t H, int Bt, const int32_t *idx, int k,
                                uint16_t *a_cache, int *status, cudaStream_t s);

// ------------------------------------------------------------------ MLP

enum MlpUpMode : int { kUpDelta = 0, kUpRefresh = 1, kUpRefreshFirst = 2 };

// Kernel 1: a = gelu(x W1[:, S] + b1[S]) over gathered hidden columns, with
// the delta / cache-writeback (sparse step) or score / cache-rebuild (refresh)
// epilogue. One CTA per (token block, chunk of 128 selected columns).
struct MlpUpParams {
  int T, D, H, k, Bt, nb, nchunks, k_pad, mode;
  const uint16_t *w1t;    // [H][D] (rows gathered on a sparse step); e4m3 codes [H][D] in the FP8 step
  const int32_t *idx;     // [nb][k] (sparse step)
  const uint16_t *b1;     // [H]
  uint16_t *a_cache;      // [nb][H][Bt]
  uint16_t *delta;        // [nb][k_pad][Bt] (sparse step); e4m3 codes in the FP8 step
  float *scores;          // [nb][H] (refresh)
  int *status;
  // FP8 step only: x ~ sx[t] * x8[t][:], W1^T ~ s1[c] * w1t8[c][:], the delta
  // of column c is multiplied by g2[c] before it is rounded to e4m3
  const float *sx, *s1, *g2;
  int group;              // token blocks walked together (set by the launcher)
};
// tm_w1t: tile map over W1^T [H][D] (box 64 x 128), read on a refresh only.
cudaError_t launch_mlp_up(const MlpUpParams &p, const CUtensorMap &tm_w1t, const CUtensorMap &tm_x, cudaStream_t s);
// The sparse step with e4m3 operands (Bt = 128): tm_x is a byte map over the
// codes x8 [T][D] (box 128 x 128); the deltas are written as e4m3 codes.
cudaError_t launch_mlp_up_fp8(const MlpUpParams &p, const CUtensorMap &tm_x, cudaStream_t s);

enum MlpDownMode : int { kDownAccumulate = 0, kDownOverwrite = 1 };

// Kernel 2: Y[b, n-slice] (+)= A[b] W2[S_b, n-slice] where A is the delta
// workspace (sparse step, rows gathered from W2) or the rebuilt activation
// cache (refresh, all rows). One CTA per (token block, slice of BN columns).
struct MlpDownParams {
  int T, D, Bt, nb, krows, k, n_slices, bn, mode;
  const uint16_t *w2;     // [H][D] (rows gathered on a sparse step); e4m3 codes [H][D] in the FP8 step
  int H;
  const int32_t *idx;     // [nb][k] (sparse step)
  const uint16_t *b2;     // [D] (refresh)
  float *y_cache;         // [T][D]
  uint16_t *out;          // [T][D] or nullptr
  int *status;
  float s_delta;          // FP8 step only: the scale of the delta codes
  int group;              // token blocks walked together (set by the launcher)
};
// tm_a: 3-D map over A [nb][rows][Bt]; tm_w2: tile map over W2 [H][D] (box 64 x 64), read on a refresh only.
cudaError_t launch_mlp_down(const MlpDownParams &p, const CUtensorMap &tm_a, const CUtensorMap &tm_w2, bool dense,
                            cudaStream_t s);
// The sparse step with e4m3 operands (Bt = 128, D a multiple of 256): tm_a is
// a byte map over the delta codes [nb][k_pad][128] (box 128 x 128 x 1).
cudaError_t launch_mlp_down_fp8(const MlpDownParams &p, const CUtensorMap &tm_a, cudaStream_t s);

// ------------------------------------------------------------------ FP8 quantisation

// codes[r][:] = e4m3(x[r][:] / scales[r]), scales[r] = max |x[r][:]| / 448 (1 for an all-zero row).
cudaError_t launch_quantize_e4m3_rows(const uint16_t *x, int64_t rows, int64_t cols, uint8_t *codes, float *scales,
                                      int *status, cudaStream_t s);

// ------------------------------------------------------------------ attention

enum AttnMode : int { kAttnDelta = 0, kAttnDense = 1, kAttnComplement = 2 };

struct AttnParams {
  int T, h, nb, k;
  float scale_log2;       // logit scale * log2(e)
  const uint16_t *k_ptr, *v_ptr;  // [T][h][128] (key rows gathered on a sparse step)
  const int32_t *idx;     // [h][nb][k]
  float *m_c, *l_c, *acc_c;  // [h][T], [h][T], [h][T][128] (partial-form complement cache)
  uint16_t *o;            // [T][h][128]
  float *lse;             // [h][T] (dense)
  int *status;
  int compact;            // complement cache as lse_c [h][T] fp32 and o_c [h][T][128] bf16
  float *lse_c;
  uint16_t *o_c;
};
// tm_q: tile map over Q [T][h*128] (box 64 x 128). tm_k / tm_v: tile maps
// over K, V [T][h*128] for the dense and complement passes (a sparse step
// gathers the selected rows with cp.async and does not use them).
cudaError_t launch_attn(int mode, const AttnParams &p, const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                        const CUtensorMap &tm_v, cudaStream_t s);

// Attention mass of every key per query block, mass[h][b][j] = sum over the
// block's queries i of exp2(s_ij * scale_log2 - lse_i * log2 e), and the top k
// keys of each mass row written to idx[h][b][0..k) (ascending, ties to the
// lower index), in one kernel.
struct MassParams {
  int T, h, nb, k;
  float scale_log2;
  const float *lse;       // [h][T] (natural log)
  float *mass;            // [h][nb][T], or nullptr: rows live in row_buf only
  float *row_buf;         // [mass_row_buffers(h * nb, T)][mass_row_floats(T)], 128-byte aligned, when mass is nullptr
  int32_t *idx;           // [h][nb][k]
  int *status;
};
// Row buffers the kernel uses for `tiles` tiles of rows of T on the current device (when the caller
// keeps no mass tensor): one or two per persistent CTA.
int64_t mass_row_buffers(int64_t tiles, int64_t T);
int64_t mass_row_floats(int64_t T);
cudaError_t launch_attn_mass_select(const MassParams &p, const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                                    cudaStream_t s);

// One CTA waiting on a barrier nothing signals (bounded: records a timeout).
cudaError_t launch_selftest_wait(int *status, cudaStream_t s);

}  // namespace cm
