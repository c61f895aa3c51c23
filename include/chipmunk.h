/*
 * chipmunk.h - C ABI of the column-sparse cross-step delta library (B200, sm_100a).
 *
 * The library implements the hot path of Chipmunk-style training-free
 * acceleration of diffusion transformers ("Chipmunk: Training-Free Acceleration
 * of Diffusion Transformers with Dynamic Column-Sparse Deltas", Together AI
 * blog post, 4/21/2025). A layer keeps a cache of its MLP activations and
 * outputs and of a partial attention state; on a sparse step only a selected
 * subset of intermediate columns (MLP hidden units, attention keys) is
 * recomputed per block of 128 tokens and the change is applied to the cache
 * (post, "Activation Deltas Across Diffusion Steps are Very Sparse": the dense
 * step written as "subtract the previous step's output vectors from the
 * cache, add the new ones", restricted to a subset).
 *
 * Conventions for every entry point
 * ---------------------------------
 * - All tensor pointers are DEVICE pointers into memory the caller owns and
 *   keeps alive until the work on `stream` has finished. The library
 *   allocates no device memory on any call below; scratch memory is passed in
 *   as `ws` / `ws_bytes` (query the size with chipmunk_workspace_bytes).
 * - Tensors are dense and row-major in the layouts stated per argument.
 *   Every base pointer must be 16-byte aligned.
 * - bf16 means IEEE bfloat16 bit patterns (uint16_t storage); fp32 is float.
 * - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default
 *   stream) and the call returns without waiting. Nothing synchronises except
 *   chipmunk_read_device_status.
 * - Arguments are checked on the host before anything is enqueued; a failed
 *   check returns a non-zero status, enqueues nothing and records a message
 *   for chipmunk_last_error(). A failed launch returns CHIPMUNK_ERR_CUDA.
 *   Kernels never trap: a bounded wait that runs out sets the device status
 *   word, which chipmunk_read_device_status reports.
 * - Calls on the same stream are ordered; calls that share output buffers
 *   must not run concurrently on different streams.
 */
#ifndef CHIPMUNK_H
#define CHIPMUNK_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CHIPMUNK_API __attribute__((visibility("default")))
#else
#define CHIPMUNK_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t chipmunk_status;
#define CHIPMUNK_OK               0
#define CHIPMUNK_ERR_INVALID_ARG  1 /* null pointer, bad enum, k out of range */
#define CHIPMUNK_ERR_SHAPE        2 /* a size outside the supported set       */
#define CHIPMUNK_ERR_ALIGNMENT    3 /* a base pointer not 16-byte aligned      */
#define CHIPMUNK_ERR_CUDA         4 /* a CUDA runtime/driver call failed       */
#define CHIPMUNK_ERR_DEVICE       5 /* a kernel set the device status word     */
#define CHIPMUNK_ERR_UNSUPPORTED  6 /* no sm_100 device, or option not built   */
#define CHIPMUNK_ERR_WORKSPACE    7 /* ws missing or smaller than required     */

/* Device status word values (chipmunk_read_device_status). */
#define CHIPMUNK_DEV_OK            0
#define CHIPMUNK_DEV_WAIT_TIMEOUT  1 /* a pipeline wait exceeded its bound       */
#define CHIPMUNK_DEV_BAD_INDEX     2 /* a selected index was outside its range   */

typedef void *chipmunk_stream; /* cudaStream_t */

/*
 * MLP layer state and inputs. The MLP is  y = gelu(x W1 + b1) W2 + b2
 * (post, "MLP" equation; GELU in its tanh form; the bias b2 is one extra
 * static vector and lives only in the output cache).
 *
 *   T       tokens (rows of x), >= 1
 *   D       model width, multiple of 64, 64..16384
 *   H       hidden width (columns of W1), >= 1, multiple of 8
 *   Bt      token block: 64 or 128; nb = ceil(T / Bt) blocks, the last may be short
 *   k       selected hidden columns per block, 0 <= k <= H
 *   x       [T][D]      bf16   current input
 *   w1t     [H][D]      bf16   W1 transposed: hidden column c of W1 is row c
 *   b1      [H]         bf16
 *   w2      [H][D]      bf16   hidden unit c writes row c
 *   b2      [D]         bf16   (read by the dense refresh only)
 *   idx     [nb][k]     int32  selected hidden columns of each block, strictly
 *                              ascending, each in [0, H)
 *   a_cache [nb][H][Bt] bf16   cached activations, block-column-major: the Bt
 *                              values of column c of block b are contiguous
 *                              (slots of a short last block past T are unused)
 *   y_cache [T][D]      fp32   cached MLP output
 *   out     [T][D]      bf16   layer output bf16(y_cache) after the step; may be NULL
 */
typedef struct chipmunk_mlp_args {
  int64_t T, D, H;
  int32_t Bt, k;
  const void *x, *w1t, *b1, *w2, *b2;
  int32_t *idx;
  void *a_cache;
  float *y_cache;
  void *out;
} chipmunk_mlp_args;

/*
 * Attention layer state and inputs, per head: O = softmax(scale Q K^T) V
 * (post, "Attention" equation; the 1/sqrt(d) logit scale is passed in).
 *
 *   T       tokens (queries = keys), >= 1
 *   h       heads, >= 1
 *   d       head dimension: 128
 *   Bt      query block: 128; nb = ceil(T / 128)
 *   k       selected keys per (head, query block), 0 <= k <= T
 *   scale   logit scale
 *   q, kk, v [T][h][d]  bf16
 *   idx     [h][nb][k]  int32  selected keys, strictly ascending, each in [0, T)
 *   m_c,l_c [h][T]      fp32   cached partial over the complementary keys:
 *   acc_c   [h][T][d]   fp32   m = max logit, l = sum exp(s - m),
 *                              acc = sum exp(s - m) v; an empty complement is
 *                              m = -inf, l = 0, acc = 0
 *                              (cache_format CHIPMUNK_ATTN_CACHE_PARTIAL)
 *   o       [T][h][d]   bf16   output
 *   cache_format               CHIPMUNK_ATTN_CACHE_PARTIAL (0): the complement
 *                              is cached as m_c, l_c, acc_c above; lse_c and
 *                              o_c are not used (may be NULL).
 *                              CHIPMUNK_ATTN_CACHE_COMPACT (1): it is cached as
 *   lse_c   [h][T]      fp32   lse = m + ln l (natural log, of the scaled
 *                              logits; -inf for an empty complement) and
 *   o_c     [h][T][d]   bf16   o = acc / l (0 for an empty complement); m_c,
 *                              l_c, acc_c are not used (may be NULL). Same
 *                              state in half the bytes of acc: o_c is rounded
 *                              to bf16. (The post caches the partial state;
 *                              this log-sum-exp encoding of it is the
 *                              library's own.)
 */
#define CHIPMUNK_ATTN_CACHE_PARTIAL 0
#define CHIPMUNK_ATTN_CACHE_COMPACT 1
typedef struct chipmunk_attn_args {
  int64_t T;
  int32_t h, d, Bt, k;
  float scale;
  const void *q, *kk, *v;
  int32_t *idx;
  float *m_c, *l_c, *acc_c;
  void *o;
  int32_t cache_format;
  float *lse_c;
  void *o_c;
} chipmunk_attn_args;

#define CHIPMUNK_REFRESH_MLP  0
#define CHIPMUNK_REFRESH_ATTN 1

/*
 * Dense refresh of one layer (the dense steps of the schedule; the post's
 * HunyuanVideo footnote runs 6 of 50 steps at lower sparsity).
 *   kind == CHIPMUNK_REFRESH_MLP: reads mlp.{x,w1t,b1,w2,b2}, the old
 *     mlp.a_cache; writes scores [nb][H] (fp32, per block and column the sum
 *     over the block's rows of |a - a_cache_old|, or of |a| when first_step
 *     is non-zero), mlp.idx (top mlp.k columns of each score row),
 *     mlp.a_cache = bf16(a), mlp.y_cache = a W2 + b2 and mlp.out (if not NULL).
 *   kind == CHIPMUNK_REFRESH_ATTN: reads attn.{q,kk,v}; writes attn.o (dense
 *     attention), attn.idx (top attn.k keys of each row of the attention
 *     mass: per head and query block the column sums of the softmax
 *     probabilities, fp32; the top-k is taken inside the kernel that computes
 *     the mass), the complement cache of every query over the keys its block
 *     did not select, in attn.cache_format: attn.{m_c,l_c,acc_c} or
 *     attn.{lse_c,o_c}; and, if scores is not NULL, the mass itself to
 *     scores [h][nb][T]. With scores NULL the mass rows live only in the
 *     workspace's row buffers (the post's "fast sparsity identification":
 *     the 4-byte-per-key mass need not travel to HBM and back).
 * scores: 16-byte aligned; required for the MLP, optional for attention.
 */
typedef struct chipmunk_refresh_args {
  int32_t kind;
  int32_t first_step;
  chipmunk_mlp_args mlp;
  chipmunk_attn_args attn;
  float *scores;
} chipmunk_refresh_args;

#define CHIPMUNK_OP_TOPK         0
#define CHIPMUNK_OP_MLP_DELTA    1
#define CHIPMUNK_OP_ATTN_DELTA   2
#define CHIPMUNK_OP_REFRESH      3
#define CHIPMUNK_OP_MLP_DELTA_FP8 4

/*
 * Top-k column selection (post: Chipmunk "dynamically chooses which ones to
 * recompute in each step"; its kernel notes name fast custom sparsity
 * identification). For each of `rows` rows of `n` fp32 scores, writes the k
 * largest as strictly ascending column indices. Scores compare by value with
 * -0 == +0; equal scores go to the lower index, so the result is unique.
 * NaN orders by its bits (+NaN above +inf). 0 <= k <= n, n <= 2^30.
 *   scores  [rows][ld_scores] fp32 (ld_scores >= n)
 *   idx     [rows][ld_idx]    int32 output (ld_idx >= k)
 * Needs no workspace (ws may be NULL).
 */
CHIPMUNK_API chipmunk_status chipmunk_topk_cols(const float *scores, int64_t rows, int64_t n, int64_t ld_scores,
                                   int32_t k, int32_t *idx, int64_t ld_idx,
                                   void *ws, size_t ws_bytes, chipmunk_stream stream);

/*
 * Sparse MLP step against the cache (post, "Activation Deltas Across
 * Diffusion Steps are Very Sparse"). For each block b and selected column c:
 *   a = gelu(x[b] W1[:,c] + b1[c]);  delta = bf16(a) - a_cache[b][c];
 *   y_cache[b] += sum_c delta * W2[c,:];  a_cache[b][c] = bf16(a);
 * then out = bf16(y_cache) if out is not NULL. Unselected columns and the
 * rest of the cache are left untouched. The activation is rounded before the
 * delta is taken, so y_cache stays equal to a_cache W2 + b2 up to fp32
 * accumulation. Workspace: chipmunk_workspace_bytes(CHIPMUNK_OP_MLP_DELTA, a)
 * bytes (nb * round_up(k,128) * Bt bf16 deltas).
 */
CHIPMUNK_API chipmunk_status chipmunk_mlp_delta(const chipmunk_mlp_args *a, void *ws, size_t ws_bytes,
                                   chipmunk_stream stream);

/*
 * The two kernels of chipmunk_mlp_delta as separate calls, same arguments and
 * workspace: _up recomputes the selected activations, writes their deltas to
 * the workspace and the new values into a_cache; _down adds delta * W2[S,:]
 * into y_cache and writes out. Calling _up then _down on one stream is
 * chipmunk_mlp_delta.
 */
CHIPMUNK_API chipmunk_status chipmunk_mlp_delta_up(const chipmunk_mlp_args *a, void *ws, size_t ws_bytes, chipmunk_stream stream);
CHIPMUNK_API chipmunk_status chipmunk_mlp_delta_down(const chipmunk_mlp_args *a, void *ws, size_t ws_bytes,
                                        chipmunk_stream stream);

/*
 * chipmunk_mlp_delta_noalloc - the sparse MLP step for callers that cannot
 * allocate device memory. No counterpart in the blog post, which describes the
 * method, not how its scratch memory is obtained.
 *
 * Some callers can't call cudaMalloc: a host framework that owns all device
 * memory and gives its plugins no allocator, or a latency-bound loop where an
 * allocation would synchronise the device. This call computes exactly what
 * chipmunk_mlp_delta computes, with the same arguments, but takes its delta
 * scratch from a fixed array inside the library instead of from the caller:
 *   - The array holds CHIPMUNK_NOALLOC_SCRATCH_BYTES (64 MiB). It is reserved
 *     on a device when the part of the library that holds it is loaded there:
 *     under CUDA's default lazy module loading, at this entry point's first
 *     call on that device (no other entry point loads it); with
 *     CUDA_MODULE_LOADING=EAGER, when the device's context is created. From
 *     then on that device keeps it until the process exits. If the device has
 *     no 64 MiB left at that moment, the first call returns CHIPMUNK_ERR_CUDA
 *     and enqueues nothing.
 *   - Calls that need more (nb * round_up(k, 128) * Bt * 2 bytes; the
 *     FLUX.1-dev layer at 70% sparsity needs 32.3 MB) return
 *     CHIPMUNK_ERR_WORKSPACE and enqueue nothing.
 *   - The first call on a device looks up the array's device address (a
 *     one-time set-up per device, done with that device current); make that
 *     first call before any stream capture.
 *   - It allocates nothing: no cudaMalloc, no cudaFree, no allocating library.
 *   - All calls share the one array and it keeps the last call's contents.
 *     Nothing in it needs to start at zero (each call writes every scratch
 *     byte it reads before reading it), but calls whose work overlaps on the
 *     GPU (different streams, or different host threads without ordering)
 *     race on it and must be serialised by the caller.
 */
#define CHIPMUNK_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
CHIPMUNK_API chipmunk_status chipmunk_mlp_delta_noalloc(const chipmunk_mlp_args *a, chipmunk_stream stream);

/*
 * FP8 form of the sparse MLP step (the post reports the method on an FP8
 * FLUX.1-dev, sparsified, 1.1x over the fastest open-source implementation;
 * the scaling scheme below is this library's). The gathered GEMMs run on e4m3
 * operands (tcgen05 kind::f8f6f4, fp32 accumulation):
 *   x[t][:]  ~ sx[t] * x8[t][:]          (per-token scale)
 *   W1^T[c][:] ~ s1[c] * w1t8[c][:]      (per-hidden-unit scale)
 *   W2[c][:] ~ s2[c] * w2_8[c][:]        (per-hidden-unit scale)
 * For each block b and selected column c:
 *   a = gelu(s1[c] sx[t] (x8[t] . w1t8[c]) + b1[c]);  delta = bf16(a) - a_cache[b][c];
 *   code = e4m3(delta * g2[c])  with g2[c] = s2[c] / s_delta (rounded to nearest
 *          even, saturated at +-448);
 *   y_cache[t] += s_delta * sum_c code * w2_8[c];  a_cache[b][c] = bf16(a);
 * then out = bf16(y_cache) if out is not NULL. s_delta is a static scale of
 * the deltas chosen by the caller (deltas beyond 448 s_delta / s2[c]
 * saturate). Use chipmunk_quantize_e4m3_rows for the codes and scales.
 *   T, H    as for chipmunk_mlp_args; Bt must be 128; D a multiple of 256
 *   x8      [T][D] e4m3 codes (bytes);  sx [T] fp32
 *   w1t8    [H][D] e4m3;  s1 [H] fp32;  b1 [H] bf16
 *   w2_8    [H][D] e4m3;  g2 [H] fp32;  s_delta > 0
 *   idx, a_cache, y_cache, out: as for chipmunk_mlp_args
 * Workspace: chipmunk_workspace_bytes(CHIPMUNK_OP_MLP_DELTA_FP8, a) bytes
 * (nb * round_up(k,128) * 128 delta codes).
 */
typedef struct chipmunk_mlp_fp8_args {
  int64_t T, D, H;
  int32_t Bt, k;
  const void *x8;
  const float *sx;
  const void *w1t8;
  const float *s1;
  const void *b1;
  const void *w2_8;
  const float *g2;
  float s_delta;
  int32_t *idx;
  void *a_cache;
  float *y_cache;
  void *out;
} chipmunk_mlp_fp8_args;

CHIPMUNK_API chipmunk_status chipmunk_mlp_delta_fp8(const chipmunk_mlp_fp8_args *a, void *ws, size_t ws_bytes,
                                                    chipmunk_stream stream);

/*
 * Rows of bf16 values to e4m3 codes with one scale per row (the operands of
 * chipmunk_mlp_delta_fp8: activations per token, weights per hidden unit).
 * For each row r: amax = max |x[r][:]|, inv = 448 / amax and scale = amax / 448
 * (fp32 divisions rounded to nearest; both 1 for an all-zero row), codes[r][i]
 * = e4m3(x[r][i] * inv) (fp32 product, rounded to nearest even, saturated at
 * +-448), scales[r] = scale, so that x ~ scale * code. Values must be finite.
 *   x [rows][cols] bf16, codes [rows][cols] bytes, scales [rows] fp32;
 *   cols a multiple of 16.
 */
CHIPMUNK_API chipmunk_status chipmunk_quantize_e4m3_rows(const void *x, int64_t rows, int64_t cols, void *codes,
                                                         float *scales, chipmunk_stream stream);

/*
 * Sparse attention step (post: attention output as a sum of scaled rows of V,
 * of which only a subset is replaced each step). For each head and 128-query
 * block the selected keys idx[h][b] are attended with the current q, kk, v by
 * online softmax and merged with the cached complement partial:
 *   M = max(m_c, m_s);  o = (acc_c e^(m_c-M) + acc_s e^(m_s-M)) / (l_c e^(m_c-M) + l_s e^(m_s-M)).
 * With the compact cache (cache_format 1) the complement enters as
 * l_c e^(m_c) = e^(lse_c) and acc_c e^(m_c) = o_c e^(lse_c):
 *   M = max(lse_c, m_s);  o = (o_c e^(lse_c-M) + acc_s e^(m_s-M)) / (e^(lse_c-M) + l_s e^(m_s-M)).
 * Rows where nothing contributes (l = 0 on both sides) get 0. The cache is
 * read only. Needs no workspace.
 */
CHIPMUNK_API chipmunk_status chipmunk_attn_delta(const chipmunk_attn_args *a, void *ws, size_t ws_bytes,
                                    chipmunk_stream stream);

/*
 * Dense refresh (see chipmunk_refresh_args). Workspace:
 * chipmunk_workspace_bytes(CHIPMUNK_OP_REFRESH, a) bytes, 16-byte aligned
 * (MLP: none; attention: the row log-sum-exp, h * T fp32 rounded up to 256
 * bytes, then, when a->scores is NULL, the mass kernel's row buffers from the
 * next 128-byte boundary: one or two rows of round_up(T, 32) fp32 per
 * persistent CTA, sized for the current device, so query the size on the
 * device that runs the call). Too small a
 * workspace is rejected with CHIPMUNK_ERR_WORKSPACE before anything runs.
 */
CHIPMUNK_API chipmunk_status chipmunk_dense_refresh(const chipmunk_refresh_args *a, void *ws, size_t ws_bytes,
                                       chipmunk_stream stream);

/*
 * Standalone cache column gather and scatter (post's kernel notes: cache
 * writeback of the recomputed columns). With the block-column-major cache
 * layout every selected column of a block is one contiguous run of Bt bf16.
 *   gather:  packed[b][j][:] = a_cache[b][idx[b][j]][:]
 *   scatter: a_cache[b][idx[b][j]][:] = packed[b][j][:]
 *   a_cache [nb][H][Bt] bf16, packed [nb][k][Bt] bf16, idx [nb][k] int32 in [0, H).
 * Bt is 64 or 128. Scatter requires the indices of a block to be distinct.
 */
CHIPMUNK_API chipmunk_status chipmunk_gather_cols(const void *a_cache, int64_t nb, int64_t H, int32_t Bt,
                                     const int32_t *idx, int32_t k, void *packed, chipmunk_stream stream);
CHIPMUNK_API chipmunk_status chipmunk_scatter_cols(const void *packed, int64_t nb, int64_t H, int32_t Bt,
                                      const int32_t *idx, int32_t k, void *a_cache, chipmunk_stream stream);

/*
 * Workspace bytes an operation needs for the given arguments (a pointer to
 * the op's argument struct; for CHIPMUNK_OP_TOPK pass NULL). 0 = none.
 */
CHIPMUNK_API size_t chipmunk_workspace_bytes(int32_t op, const void *args);

/* Name of a status code (static string). */
CHIPMUNK_API const char *chipmunk_status_string(chipmunk_status status);

/* Message of the last failed call on this host thread (static storage). */
CHIPMUNK_API const char *chipmunk_last_error(void);

/*
 * Waits for `stream`, copies the device status word of the current device
 * to *host_out and clears it. Returns CHIPMUNK_ERR_DEVICE if it was set.
 */
CHIPMUNK_API chipmunk_status chipmunk_read_device_status(int32_t *host_out, chipmunk_stream stream);

/*
 * Diagnostic for failure detection (no counterpart in the post): launches one
 * CTA that waits, with the same bounded wait every kernel uses, on a barrier
 * nothing signals. The wait gives up after about 2 s and records
 * CHIPMUNK_DEV_WAIT_TIMEOUT in the device status word; the kernel then
 * returns normally (no trap, no fault) and the context stays usable. Read
 * and clear the word with chipmunk_read_device_status. Kernels launched
 * while the word is set return at entry without doing work.
 */
CHIPMUNK_API chipmunk_status chipmunk_selftest_bounded_wait(chipmunk_stream stream);

/* Library version, e.g. "0.1.0". */
CHIPMUNK_API const char *chipmunk_version(void);

#ifdef __cplusplus
}
#endif
#endif /* CHIPMUNK_H */
