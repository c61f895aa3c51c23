// chipmunk_oracle.cpp - the oracle of the column-sparse cross-step delta method,
// in plain C++ and fp64.
//
// TEST INFRASTRUCTURE ONLY. This is a slow, direct CPU restatement of what the
// method computes, used to check the CUDA library. Only the tests, the smoke
// check in __graft_entry__ and the CPU-baseline / reference legs of bench.py
// may load it (through oracle/cpp.py). It shares no code, header or constant
// with the CUDA path and includes nothing from the package.
//
// Source: "Chipmunk: Training-Free Acceleration of Diffusion Transformers with
// Dynamic Column-Sparse Deltas" (Together AI blog post, 4/21/2025), sections
// "Slow-Changing, Sparse Activations" and "Activation Deltas Across Diffusion
// Steps are Very Sparse": the attention and MLP equations and the cache-delta
// identity that follows them.
//
// Conventions. Every array is dense and row-major; values are double unless
// stated. MLP: x [T][D], W1 [D][H], b1 [H], W2 [H][D], b2 [D], activations
// [T][H], outputs [T][D]. Attention, per head: q, k, v [h][T][d]; a softmax
// partial state is (m, l, acc): m the row maximum of the logits, l the sum of
// exp(s - m), acc the sum of exp(s - m) v ([h][T][d]). Tokens form blocks of
// Bt consecutive rows, the last one possibly short. Selections are int32,
// ascending: [nb][k] (MLP) or [h][nb][k] (attention). Sums run over ascending
// indices, one term at a time. Readings where the post is silent are the same
// as the numpy oracle's (GELU in its tanh form, 1/sqrt(d) logit scale passed
// in, column L1 score of the activation change, attention mass score, top-k
// with ties to the lower index).
//
// Independent work items (token blocks, (head, block) tiles, score rows) run
// on std::thread workers; each item writes only its own outputs, so the result
// does not depend on the number of threads.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <functional>
#include <limits>
#include <thread>
#include <vector>

namespace {

const double kNegInf = -std::numeric_limits<double>::infinity();

int g_threads = 0;  // 0: one per hardware thread

int worker_count() {
  if (g_threads > 0) return g_threads;
  unsigned n = std::thread::hardware_concurrency();
  return n == 0 ? 1 : static_cast<int>(n);
}

// Runs fn(i) for i = 0 .. n-1 on the worker threads.
void parallel_for(int64_t n, const std::function<void(int64_t)> &fn) {
  const int nt = static_cast<int>(std::min<int64_t>(worker_count(), n));
  if (nt <= 1) {
    for (int64_t i = 0; i < n; ++i) fn(i);
    return;
  }
  std::atomic<int64_t> next(0);
  std::vector<std::thread> pool;
  for (int t = 0; t < nt; ++t)
    pool.emplace_back([&]() {
      for (int64_t i = next.fetch_add(1); i < n; i = next.fetch_add(1)) fn(i);
    });
  for (auto &th : pool) th.join();
}

// ------------------------------------------------------------------ blocks

int64_t block_count(int64_t T, int64_t Bt) { return (T + Bt - 1) / Bt; }

// First row and end row of token block b; the last block ends at T.
void block_range(int64_t b, int64_t T, int64_t Bt, int64_t *r0, int64_t *r1) {
  *r0 = b * Bt;
  *r1 = std::min((b + 1) * Bt, T);
}

// ------------------------------------------------------------------ storage

double bf16_to_double(uint16_t bits) {
  const uint32_t u = static_cast<uint32_t>(bits) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return static_cast<double>(f);
}

// double -> float (the C++ conversion rounds to nearest even) -> bf16, rounding
// the float's 32 bits to their upper 16, to nearest with ties to even.
uint16_t double_to_bf16(double x) {
  const float f = static_cast<float>(x);
  if (std::isnan(f)) return 0x7FC0;
  uint32_t u;
  std::memcpy(&u, &f, 4);
  const uint32_t lsb = (u >> 16) & 1u;
  return static_cast<uint16_t>((static_cast<uint64_t>(u) + 0x7FFFu + lsb) >> 16);
}

// e4m3 (OCP FP8 E4M3: 1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no
// infinities, S.1111.111 is NaN, the largest finite value 448 = 1.75 * 2^8,
// subnormals m / 8 * 2^-6) from a float: rounded to nearest, ties to the even
// code, magnitudes above 448 saturated to 448.
uint8_t e4m3_encode(float x) {
  if (std::isnan(x)) return 0x7F;
  const uint8_t sign = std::signbit(x) ? 0x80 : 0x00;
  const double a = std::fabs(static_cast<double>(x));
  if (a >= 448.0) return sign | 0x7E;
  if (a < std::ldexp(1.0, -6)) {
    // subnormal range: steps of 2^-9; 8 steps is the smallest normal, code 0x08
    const double m = std::nearbyint(a * 512.0);
    return sign | static_cast<uint8_t>(m);
  }
  int e2;
  std::frexp(a, &e2);                  // a = f * 2^e2, f in [0.5, 1)
  int e = e2 - 1;                      // a in [2^e, 2^(e+1))
  double r = std::nearbyint(std::ldexp(a, 3 - e));   // in [8, 16]
  if (r == 16.0) {
    r = 8.0;
    ++e;
  }
  const int be = e + 7;
  const int m = static_cast<int>(r) - 8;
  if (be > 15 || (be == 15 && m == 7)) return sign | 0x7E;
  return sign | static_cast<uint8_t>((be << 3) | m);
}

double e4m3_decode(uint8_t c) {
  const double sign = (c & 0x80) ? -1.0 : 1.0;
  const int be = (c >> 3) & 15, m = c & 7;
  if (be == 15 && m == 7) return std::numeric_limits<double>::quiet_NaN();
  if (be == 0) return sign * std::ldexp(m / 8.0, -6);
  return sign * std::ldexp(1.0 + m / 8.0, be - 7);
}

// ------------------------------------------------------------------ MLP pieces

// GELU, tanh form (Hendrycks and Gimpel): the post's MLP non-linearity.
double gelu(double u) {
  const double c = std::sqrt(2.0 / M_PI);
  return 0.5 * u * (1.0 + std::tanh(c * (u + 0.044715 * u * u * u)));
}

// Rows are worked on side by side in groups of at most kRows; a group's
// running sums sit in a small local array.
constexpr int64_t kRows = 16;

// The two contractions below keep their running sums in small local arrays
// whose fixed-length inner loops the compiler unrolls into vector registers;
// its loop vectorizer, which reorganises these nests badly, is turned off for
// them. Neither changes any sum: each is formed term by term in ascending order.
#define ORACLE_CONTRACTION __attribute__((optimize("no-tree-loop-vectorize")))

// Pre-activation of hidden unit c for the nr <= kRows rows of a group:
// u[r] = sum over d (ascending) of x[r][d] W1[d][c], then + b1[c]. w1t is W1
// transposed ([H][D]: the input weights of hidden unit c are row c); xt is the
// group's inputs transposed ([D][kRows], rows past nr are zero).
ORACLE_CONTRACTION void preactivation(const double *xt, int64_t nr, const double *w1t, const double *b1, int64_t D,
                                      int64_t c, double *u) {
  const double *w = w1t + c * D;
  double acc[kRows] = {};
  for (int64_t d = 0; d < D; ++d) {
    const double *xd = xt + d * kRows;
#pragma GCC unroll 16
    for (int64_t r = 0; r < kRows; ++r) acc[r] += xd[r] * w[d];
  }
  for (int64_t r = 0; r < nr; ++r) u[r] = acc[r] + b1[c];
}

// sums[r][n] = sum over j (ascending) of coef[r][j] rows[j][n] for the nr <=
// kRows rows of a group, n = 0 .. D-1: coef is [nr][ncoef] (row stride ldc),
// rows[j] points at a row of D values, sums [nr][D] (row stride lds) must hold
// zeros on entry. Sixteen sums at a time run over 128 terms in a local array
// and are stored back in between (a double stored and reloaded is exact), so
// the weight rows of those terms are reused from cache by all rows.
ORACLE_CONTRACTION void weighted_row_sums(const double *coef, int64_t ldc, int64_t nr, const double *const *rows,
                                          int64_t ncoef, int64_t D, double *sums, int64_t lds) {
  const int64_t kTerms = 128;
  for (int64_t j0 = 0; j0 < ncoef; j0 += kTerms) {
    const int64_t j1 = std::min(j0 + kTerms, ncoef);
    for (int64_t n0 = 0; n0 < D; n0 += 16) {
      const int64_t nn = std::min<int64_t>(16, D - n0);
      for (int64_t r = 0; r < nr; ++r) {
        double *o = sums + r * lds + n0;
        if (nn == 16) {
          double acc[16];
#pragma GCC unroll 16
          for (int64_t e = 0; e < 16; ++e) acc[e] = o[e];
          for (int64_t j = j0; j < j1; ++j) {
            const double cj = coef[r * ldc + j];
            const double *w = rows[j] + n0;
#pragma GCC unroll 16
            for (int64_t e = 0; e < 16; ++e) acc[e] += cj * w[e];
          }
#pragma GCC unroll 16
          for (int64_t e = 0; e < 16; ++e) o[e] = acc[e];
        } else {
          for (int64_t j = j0; j < j1; ++j)
            for (int64_t e = 0; e < nn; ++e) o[e] += coef[r * ldc + j] * rows[j][n0 + e];
        }
      }
    }
  }
}

// x rows r0 .. r1-1 (at most kRows) transposed into xt [D][kRows], zero past r1.
void transpose_rows(const double *x, int64_t r0, int64_t r1, int64_t D, double *xt) {
  for (int64_t i = 0; i < D * kRows; ++i) xt[i] = 0.0;
  for (int64_t r = r0; r < r1; ++r)
    for (int64_t d = 0; d < D; ++d) xt[d * kRows + (r - r0)] = x[r * D + d];
}

// ------------------------------------------------------------------ selection

// fp32 value -> uint32 key whose unsigned order is the numeric order: negative
// values have all bits flipped, others get the sign bit set; -0 is first
// mapped to +0 so the two compare equal. A NaN lands by its bits.
uint32_t ordered_key(float f) {
  uint32_t b;
  std::memcpy(&b, &f, 4);
  if (b == 0x80000000u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// The k largest fp32 scores of one row, ties to the lower index, as ascending
// indices: a stable sort of the indices by key, descending, then the first k
// sorted by index.
void topk_row(const float *row, int64_t n, int64_t k, int32_t *out) {
  std::vector<int64_t> order(n);
  for (int64_t i = 0; i < n; ++i) order[i] = i;
  std::vector<uint32_t> key(n);
  for (int64_t i = 0; i < n; ++i) key[i] = ordered_key(row[i]);
  std::stable_sort(order.begin(), order.end(), [&](int64_t a, int64_t b) { return key[a] > key[b]; });
  std::sort(order.begin(), order.begin() + k);
  for (int64_t i = 0; i < k; ++i) out[i] = static_cast<int32_t>(order[i]);
}

// ------------------------------------------------------------------ attention pieces

// Softmax partial state of the n query rows q [n][d] over the keys keys[0..m-1]
// (rows of kmat / vmat [T][d]): m = max of the logits scale * q k^T, l = sum of
// exp(s - m), acc = sum of exp(s - m) v. No keys: (-inf, 0, 0). The keys are
// first copied out transposed ([d][m]) so that one query's logits are summed
// side by side; every logit is the plain ascending-index dot product.
void partial_over(const double *q, int64_t n, const double *kmat, const double *vmat, const int64_t *keys, int64_t m,
                  int64_t d, double scale, double *m_out, double *l_out, double *acc_out) {
  std::vector<double> kt(d * m), s(m);
  for (int64_t j = 0; j < m; ++j)
    for (int64_t e = 0; e < d; ++e) kt[e * m + j] = kmat[keys[j] * d + e];
  for (int64_t i = 0; i < n; ++i) {
    double *acc = acc_out + i * d;
    for (int64_t e = 0; e < d; ++e) acc[e] = 0.0;
    if (m == 0) {
      m_out[i] = kNegInf;
      l_out[i] = 0.0;
      continue;
    }
    for (int64_t j = 0; j < m; ++j) s[j] = 0.0;
    for (int64_t e = 0; e < d; ++e) {
      const double qe = q[i * d + e];
      const double *ke = kt.data() + e * m;
      for (int64_t j = 0; j < m; ++j) s[j] += qe * ke[j];
    }
    double mx = kNegInf;
    for (int64_t j = 0; j < m; ++j) {
      s[j] *= scale;
      mx = std::max(mx, s[j]);
    }
    double l = 0.0;
    for (int64_t j = 0; j < m; ++j) {
      const double p = std::exp(s[j] - mx);
      l += p;
      const double *vr = vmat + keys[j] * d;
      for (int64_t e = 0; e < d; ++e) acc[e] += p * vr[e];
    }
    m_out[i] = mx;
    l_out[i] = l;
  }
}

// Online-softmax merge of two partial states of one row over disjoint key sets.
void merge_row(double m1, double l1, const double *a1, double m2, double l2, const double *a2, int64_t d, double *M,
               double *L, double *A) {
  const double mm = std::max(m1, m2);
  const double w1 = (m1 == kNegInf) ? 0.0 : std::exp(m1 - mm);
  const double w2 = (m2 == kNegInf) ? 0.0 : std::exp(m2 - mm);
  *M = mm;
  *L = l1 * w1 + l2 * w2;
  for (int64_t e = 0; e < d; ++e) A[e] = a1[e] * w1 + a2[e] * w2;
}

// Normalised output acc / l of a partial state (0 where no key contributed).
void finish_row(double l, const double *acc, int64_t d, double *out) {
  for (int64_t e = 0; e < d; ++e) out[e] = l > 0 ? acc[e] / l : 0.0;
}

// Attention mass of each key for the query rows q [n][d]: the column sums of
// the row softmax over all T keys, sum over i of softmax_i(j). The keys are
// copied out transposed as in partial_over.
void mass_rows(const double *q, int64_t n, const double *kmat, int64_t T, int64_t d, double scale, double *out) {
  std::vector<double> kt(d * T), s(T);
  for (int64_t j = 0; j < T; ++j)
    for (int64_t e = 0; e < d; ++e) kt[e * T + j] = kmat[j * d + e];
  for (int64_t j = 0; j < T; ++j) out[j] = 0.0;
  for (int64_t i = 0; i < n; ++i) {
    for (int64_t j = 0; j < T; ++j) s[j] = 0.0;
    for (int64_t e = 0; e < d; ++e) {
      const double qe = q[i * d + e];
      const double *ke = kt.data() + e * T;
      for (int64_t j = 0; j < T; ++j) s[j] += qe * ke[j];
    }
    double mx = kNegInf;
    for (int64_t j = 0; j < T; ++j) {
      s[j] *= scale;
      mx = std::max(mx, s[j]);
    }
    double l = 0.0;
    for (int64_t j = 0; j < T; ++j) {
      s[j] = std::exp(s[j] - mx);
      l += s[j];
    }
    for (int64_t j = 0; j < T; ++j) out[j] += s[j] / l;
  }
}

}  // namespace

extern "C" {

void or_set_threads(int n) { g_threads = n; }
int or_threads(void) { return worker_count(); }

// ------------------------------------------------------------------ storage

void or_bf16_decode(const uint16_t *bits, int64_t n, double *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = bf16_to_double(bits[i]);
}

void or_bf16_round(const double *x, int64_t n, uint16_t *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = double_to_bf16(x[i]);
}

// Selected count for a kept fraction in per mille, rounded down.
int64_t or_k_from_density(int64_t n, int64_t permille) { return (n * permille) / 1000; }

int64_t or_block_count(int64_t T, int64_t Bt) { return block_count(T, Bt); }

void or_block_range(int64_t b, int64_t T, int64_t Bt, int64_t *r0, int64_t *r1) { block_range(b, T, Bt, r0, r1); }

// ------------------------------------------------------------------ MLP

void or_gelu_tanh(const double *u, int64_t n, double *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = gelu(u[i]);
}

// gelu(x W1 + b1) W2 + b2 (post: "MLP" equation; the bias is one more static
// vector), with W1 given transposed (w1t [H][D]). Writes the activations
// a [T][H] and the output y [T][D]. Rows are worked on in groups of kRows, one
// group per work item; each output is the plain ascending-index sum.
void or_dense_mlp(const double *x, const double *w1t, const double *b1, const double *W2, const double *b2, int64_t T,
                  int64_t D, int64_t H, double *a, double *y) {
  std::vector<const double *> w2rows(H);
  for (int64_t c = 0; c < H; ++c) w2rows[c] = W2 + c * D;
  parallel_for(block_count(T, kRows), [&](int64_t g) {
    int64_t r0, r1;
    block_range(g, T, kRows, &r0, &r1);
    const int64_t nr = r1 - r0;
    std::vector<double> xt(D * kRows), u(kRows);
    transpose_rows(x, r0, r1, D, xt.data());
    for (int64_t c = 0; c < H; ++c) {
      preactivation(xt.data(), nr, w1t, b1, D, c, u.data());
      for (int64_t r = 0; r < nr; ++r) a[(r0 + r) * H + c] = gelu(u[r]);
    }
    // y[r] = sum over hidden units c (ascending) of a[r][c] W2[c], then + b2
    for (int64_t r = r0; r < r1; ++r)
      for (int64_t n = 0; n < D; ++n) y[r * D + n] = 0.0;
    weighted_row_sums(a + r0 * H, H, nr, w2rows.data(), H, D, y + r0 * D, D);
    for (int64_t r = r0; r < r1; ++r)
      for (int64_t n = 0; n < D; ++n) y[r * D + n] += b2[n];
  });
}

// One sparse step of the MLP against its cache. The output is a sum of rows of
// W2 weighted by the activations. For each token block b and selected hidden
// column c of idx[b] the activation is recomputed, the old vector
// A_cache[r][c] W2[c] is subtracted from the cached output and the new one
// added (post: the dense step rewritten as "subtract the old output vectors,
// add the new ones", restricted to the recomputed subset); unselected columns
// keep their cached value. Writes A_new [T][H] and Y_new [T][D] (the layer
// output).
void or_mlp_delta(const double *x, const double *w1t, const double *b1, const double *W2, const int32_t *idx,
                  int64_t k, const double *A_cache, const double *Y_cache, int64_t T, int64_t D, int64_t H, int64_t Bt,
                  double *A_new, double *Y_new) {
  std::memcpy(A_new, A_cache, sizeof(double) * T * H);
  std::memcpy(Y_new, Y_cache, sizeof(double) * T * D);
  if (k == 0) return;
  parallel_for(block_count(T, Bt), [&](int64_t b) {
    int64_t blk0, blk1;
    block_range(b, T, Bt, &blk0, &blk1);
    const int32_t *S = idx + b * k;
    std::vector<const double *> w2rows(k);
    for (int64_t j = 0; j < k; ++j) w2rows[j] = W2 + static_cast<int64_t>(S[j]) * D;
    std::vector<double> xt(D * kRows), u(kRows), delta(kRows * k), change(kRows * D);
    // the block's rows, kRows at a time
    for (int64_t r0 = blk0; r0 < blk1; r0 += kRows) {
      const int64_t r1 = std::min(r0 + kRows, blk1), nr = r1 - r0;
      transpose_rows(x, r0, r1, D, xt.data());
      for (int64_t j = 0; j < k; ++j) {
        const int64_t c = S[j];
        preactivation(xt.data(), nr, w1t, b1, D, c, u.data());
        for (int64_t r = 0; r < nr; ++r) {
          const double an = gelu(u[r]);
          delta[r * k + j] = an - A_cache[(r0 + r) * H + c];
          A_new[(r0 + r) * H + c] = an;
        }
      }
      // change[r] = sum over the selected columns (ascending) of delta[r][c] W2[c], then Y += change
      std::fill(change.begin(), change.end(), 0.0);
      weighted_row_sums(delta.data(), k, nr, w2rows.data(), k, D, change.data(), D);
      for (int64_t r = 0; r < nr; ++r) {
        double *yr = Y_new + (r0 + r) * D;
        for (int64_t n = 0; n < D; ++n) yr[n] += change[r * D + n];
      }
    }
  });
}

// Per block and hidden column: the sum over the block's rows of |a - A_cache|,
// or of |a| on a first step, which has no cache (post: "Activations are
// sparse": the largest activations carry the output). out [nb][H].
void or_mlp_scores(const double *a, const double *A_cache, int64_t T, int64_t H, int64_t Bt, int first_step,
                   double *out) {
  const int64_t nb = block_count(T, Bt);
  for (int64_t b = 0; b < nb; ++b) {
    int64_t r0, r1;
    block_range(b, T, Bt, &r0, &r1);
    for (int64_t c = 0; c < H; ++c) {
      double s = 0.0;
      for (int64_t r = r0; r < r1; ++r) s += std::fabs(first_step ? a[r * H + c] : a[r * H + c] - A_cache[r * H + c]);
      out[b * H + c] = s;
    }
  }
}

// ------------------------------------------------------------------ selection

void or_ordered_key(const float *s, int64_t n, uint32_t *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = ordered_key(s[i]);
}

// k largest fp32 scores of each row, ties to the lower index, ascending indices. out [rows][k].
void or_topk_cols(const float *scores, int64_t rows, int64_t n, int64_t k, int32_t *out) {
  parallel_for(rows, [&](int64_t r) { topk_row(scores + r * n, n, k, out + r * k); });
}

// Dense step: activations and output, scores against the old cache (|a| on a
// first step), the top-k of the fp32-rounded scores per block. Writes a, y,
// scores [nb][H] (double) and idx [nb][k].
void or_mlp_refresh(const double *x, const double *w1t, const double *b1, const double *W2, const double *b2,
                    const double *A_old, int64_t T, int64_t D, int64_t H, int64_t Bt, int64_t k, int first_step,
                    double *a, double *y, double *scores, int32_t *idx) {
  or_dense_mlp(x, w1t, b1, W2, b2, T, D, H, a, y);
  or_mlp_scores(a, A_old, T, H, Bt, first_step, scores);
  const int64_t nb = block_count(T, Bt);
  std::vector<float> s32(nb * H);
  for (int64_t i = 0; i < nb * H; ++i) s32[i] = static_cast<float>(scores[i]);
  or_topk_cols(s32.data(), nb, H, k, idx);
}

// ------------------------------------------------------------------ FP8 form of the MLP step

void or_e4m3_encode(const float *x, int64_t n, uint8_t *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_encode(x[i]);
}

void or_e4m3_decode(const uint8_t *c, int64_t n, double *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_decode(c[i]);
}

// Rows of fp32 values (bf16 ones in practice) to e4m3 codes with one scale
// per row: amax = max |x|, inv = 448 / amax and scale = amax / 448 (float
// divisions; both 1 when amax is 0), code = e4m3(x * inv) (a float product),
// so that x ~ scale * code.
void or_quantize_rows_e4m3(const float *x, int64_t rows, int64_t cols, uint8_t *codes, float *scales) {
  for (int64_t r = 0; r < rows; ++r) {
    float amax = 0.f;
    for (int64_t i = 0; i < cols; ++i) amax = std::max(amax, std::fabs(x[r * cols + i]));
    const float inv = amax > 0.f ? 448.f / amax : 1.f;
    scales[r] = amax > 0.f ? amax / 448.f : 1.f;
    for (int64_t i = 0; i < cols; ++i) {
      const float prod = x[r * cols + i] * inv;
      codes[r * cols + i] = e4m3_encode(prod);
    }
  }
}

// The FP8 form of one sparse MLP step (the library's own scaling scheme for
// the post's FP8 FLUX result). Operands are e4m3 codes with scales: x[t] ~
// sx[t] x8[t], W1^T[c] ~ s1[c] w1t8[c], W2[c] ~ s2[c] w2_8[c]. For each block
// and selected column c: a = gelu(s1[c] sx[t] (x8[t] . w1t8[c]) + b1[c]); the
// delta against the cache is taken from a rounded to bf16 (as it is stored),
// multiplied by g2[c] = s2[c] / s_delta as floats and rounded to an e4m3 code;
// the cached output gains s_delta * sum_c code * w2_8[c]. A_new takes a.
void or_mlp_delta_fp8(const uint8_t *x8, const float *sx, const uint8_t *w1t8, const float *s1, const double *b1,
                      const uint8_t *w2_8, const float *g2, float s_delta, const int32_t *idx, int64_t k,
                      const double *A_cache, const double *Y_cache, int64_t T, int64_t D, int64_t H, int64_t Bt,
                      double *A_new, double *Y_new) {
  std::memcpy(A_new, A_cache, sizeof(double) * T * H);
  std::memcpy(Y_new, Y_cache, sizeof(double) * T * D);
  if (k == 0) return;
  std::vector<double> xd(T * D), w1d(H * D), w2d(H * D);
  for (int64_t i = 0; i < T * D; ++i) xd[i] = e4m3_decode(x8[i]);
  for (int64_t i = 0; i < H * D; ++i) w1d[i] = e4m3_decode(w1t8[i]);
  for (int64_t i = 0; i < H * D; ++i) w2d[i] = e4m3_decode(w2_8[i]);
  parallel_for(block_count(T, Bt), [&](int64_t b) {
    int64_t blk0, blk1;
    block_range(b, T, Bt, &blk0, &blk1);
    const int32_t *S = idx + b * k;
    std::vector<const double *> w2rows(k);
    for (int64_t j = 0; j < k; ++j) w2rows[j] = w2d.data() + static_cast<int64_t>(S[j]) * D;
    std::vector<double> xt(D * kRows), u(kRows), code(kRows * k), change(kRows * D);
    const std::vector<double> no_bias(H, 0.0);
    for (int64_t r0 = blk0; r0 < blk1; r0 += kRows) {
      const int64_t r1 = std::min(r0 + kRows, blk1), nr = r1 - r0;
      transpose_rows(xd.data(), r0, r1, D, xt.data());
      for (int64_t j = 0; j < k; ++j) {
        const int64_t c = S[j];
        preactivation(xt.data(), nr, w1d.data(), no_bias.data(), D, c, u.data());   // x8[t] . w1t8[c]
        for (int64_t r = 0; r < nr; ++r) {
          const double an = gelu(u[r] * s1[c] * sx[r0 + r] + b1[c]);
          const double stored = bf16_to_double(double_to_bf16(an));
          const float d = static_cast<float>(stored - A_cache[(r0 + r) * H + c]);
          code[r * k + j] = e4m3_decode(e4m3_encode(d * g2[c]));
          A_new[(r0 + r) * H + c] = an;
        }
      }
      std::fill(change.begin(), change.end(), 0.0);
      weighted_row_sums(code.data(), k, nr, w2rows.data(), k, D, change.data(), D);
      for (int64_t r = 0; r < nr; ++r) {
        double *yr = Y_new + (r0 + r) * D;
        for (int64_t n = 0; n < D; ++n) yr[n] += static_cast<double>(s_delta) * change[r * D + n];
      }
    }
  });
}

// ------------------------------------------------------------------ attention

// Partial state of the query rows q [n][d] over all m keys k, v [m][d].
void or_attn_partial(const double *q, int64_t n, const double *k, const double *v, int64_t m, int64_t d, double scale,
                     double *m_out, double *l_out, double *acc_out) {
  std::vector<int64_t> keys(m);
  for (int64_t j = 0; j < m; ++j) keys[j] = j;
  partial_over(q, n, k, v, keys.data(), m, d, scale, m_out, l_out, acc_out);
}

void or_merge_partials(const double *m1, const double *l1, const double *a1, const double *m2, const double *l2,
                       const double *a2, int64_t n, int64_t d, double *M, double *L, double *A) {
  for (int64_t i = 0; i < n; ++i) merge_row(m1[i], l1[i], a1 + i * d, m2[i], l2[i], a2 + i * d, d, M + i, L + i, A + i * d);
}

void or_finish(const double *l, const double *acc, int64_t n, int64_t d, double *out) {
  for (int64_t i = 0; i < n; ++i) finish_row(l[i], acc + i * d, d, out + i * d);
}

// Sparse attention step: for each head and query block the selected keys are
// attended with the current q, k, v and merged with the cached partial over
// the complementary keys (post: attention output as a sum of scaled rows of V,
// of which only a subset is replaced each step). out [h][T][d]. With tiles
// non-null only the ntiles (head, query block) pairs listed there
// (tiles[2i], tiles[2i+1]) are computed and the rest of out is left as it is.
void or_attn_delta(const double *q, const double *k, const double *v, const int32_t *idx, int64_t kk,
                   const double *m_c, const double *l_c, const double *acc_c, int64_t h, int64_t T, int64_t d,
                   double scale, int64_t Bt, double *out, const int64_t *tiles, int64_t ntiles) {
  const int64_t nb = block_count(T, Bt);
  parallel_for(tiles ? ntiles : h * nb, [&](int64_t item) {
    const int64_t hh = tiles ? tiles[2 * item] : item / nb, b = tiles ? tiles[2 * item + 1] : item % nb;
    int64_t r0, r1;
    block_range(b, T, Bt, &r0, &r1);
    const int64_t nr = r1 - r0;
    std::vector<int64_t> keys(kk);
    for (int64_t j = 0; j < kk; ++j) keys[j] = idx[(hh * nb + b) * kk + j];
    std::vector<double> ms(nr), ls(nr), as(nr * d), M(nr), L(nr), A(nr * d);
    const double *qh = q + (hh * T + r0) * d;
    partial_over(qh, nr, k + hh * T * d, v + hh * T * d, keys.data(), kk, d, scale, ms.data(), ls.data(), as.data());
    for (int64_t i = 0; i < nr; ++i) {
      const int64_t row = hh * T + r0 + i;
      merge_row(m_c[row], l_c[row], acc_c + row * d, ms[i], ls[i], as.data() + i * d, d, &M[i], &L[i], &A[i * d]);
      finish_row(L[i], &A[i * d], d, out + row * d);
    }
  });
}

// The same partial state in log-sum-exp form: lse = m + ln l and the
// normalised output o = acc / l; an empty partial (l = 0) gives (-inf, 0).
// Since e^lse = l e^m and o e^lse = acc e^m, a merge needs nothing else (a
// denser encoding of the post's cached partial; the encoding is this
// library's).
void or_compact_partial(const double *m, const double *l, const double *acc, int64_t n, int64_t d, double *lse,
                        double *o) {
  for (int64_t i = 0; i < n; ++i) {
    lse[i] = l[i] > 0 ? m[i] + std::log(l[i]) : kNegInf;
    for (int64_t e = 0; e < d; ++e) o[i * d + e] = l[i] > 0 ? acc[i * d + e] / l[i] : 0.0;
  }
}

// Sparse attention step against a complement cached as (lse_c, o_c): the
// cache enters the merge as the partial (lse_c, 1, o_c).
void or_attn_delta_compact(const double *q, const double *k, const double *v, const int32_t *idx, int64_t kk,
                           const double *lse_c, const double *o_c, int64_t h, int64_t T, int64_t d, double scale,
                           int64_t Bt, double *out) {
  const int64_t nb = block_count(T, Bt);
  parallel_for(h * nb, [&](int64_t tile) {
    const int64_t hh = tile / nb, b = tile % nb;
    int64_t r0, r1;
    block_range(b, T, Bt, &r0, &r1);
    const int64_t nr = r1 - r0;
    std::vector<int64_t> keys(kk);
    for (int64_t j = 0; j < kk; ++j) keys[j] = idx[(hh * nb + b) * kk + j];
    std::vector<double> ms(nr), ls(nr), as(nr * d), A(nr * d);
    partial_over(q + (hh * T + r0) * d, nr, k + hh * T * d, v + hh * T * d, keys.data(), kk, d, scale, ms.data(),
                 ls.data(), as.data());
    for (int64_t i = 0; i < nr; ++i) {
      const int64_t row = hh * T + r0 + i;
      double M, L;
      merge_row(lse_c[row], 1.0, o_c + row * d, ms[i], ls[i], as.data() + i * d, d, &M, &L, &A[i * d]);
      finish_row(L, &A[i * d], d, out + row * d);
    }
  });
}

// softmax(scale q k^T) v per head (post: "Attention" equation) and the row
// log-sum-exp. O [h][T][d], lse [h][T].
void or_dense_attention(const double *q, const double *k, const double *v, int64_t h, int64_t T, int64_t d,
                        double scale, double *O, double *lse) {
  const int64_t G = 64;
  const int64_t ng = block_count(T, G);
  parallel_for(h * ng, [&](int64_t item) {
    const int64_t hh = item / ng, g = item % ng;
    int64_t r0, r1;
    block_range(g, T, G, &r0, &r1);
    const int64_t nr = r1 - r0;
    std::vector<double> m(nr), l(nr), acc(nr * d);
    or_attn_partial(q + (hh * T + r0) * d, nr, k + hh * T * d, v + hh * T * d, T, d, scale, m.data(), l.data(),
                    acc.data());
    for (int64_t i = 0; i < nr; ++i) {
      const int64_t row = hh * T + r0 + i;
      for (int64_t e = 0; e < d; ++e) O[row * d + e] = acc[i * d + e] / l[i];
      lse[row] = m[i] + std::log(l[i]);
    }
  });
}

// Attention mass of each key for one query block q_rows [n][d] over keys k [m][d].
void or_attn_mass_rows(const double *q_rows, int64_t n, const double *k, int64_t m, int64_t d, double scale,
                       double *out) {
  mass_rows(q_rows, n, k, m, d, scale, out);
}

// mass[h][b][j] = sum over the rows i of block b of softmax_i(j). out [h][nb][T].
void or_attn_mass(const double *q, const double *k, int64_t h, int64_t T, int64_t d, double scale, int64_t Bt,
                  double *out) {
  const int64_t nb = block_count(T, Bt);
  parallel_for(h * nb, [&](int64_t tile) {
    const int64_t hh = tile / nb, b = tile % nb;
    int64_t r0, r1;
    block_range(b, T, Bt, &r0, &r1);
    mass_rows(q + (hh * T + r0) * d, r1 - r0, k + hh * T * d, T, d, scale, out + (hh * nb + b) * T);
  });
}

// Partial state of every query over the keys its block did NOT select,
// computed directly over the complement (not as dense minus selected).
// m_c, l_c [h][T], acc_c [h][T][d].
void or_complement_partial(const double *q, const double *k, const double *v, const int32_t *idx, int64_t kk,
                           int64_t h, int64_t T, int64_t d, double scale, int64_t Bt, double *m_c, double *l_c,
                           double *acc_c) {
  const int64_t nb = block_count(T, Bt);
  parallel_for(h * nb, [&](int64_t tile) {
    const int64_t hh = tile / nb, b = tile % nb;
    int64_t r0, r1;
    block_range(b, T, Bt, &r0, &r1);
    std::vector<char> selected(T, 0);
    for (int64_t j = 0; j < kk; ++j) selected[idx[(hh * nb + b) * kk + j]] = 1;
    std::vector<int64_t> keys;
    for (int64_t j = 0; j < T; ++j)
      if (!selected[j]) keys.push_back(j);
    const int64_t row = hh * T + r0;
    partial_over(q + row * d, r1 - r0, k + hh * T * d, v + hh * T * d, keys.data(), static_cast<int64_t>(keys.size()),
                 d, scale, m_c + row, l_c + row, acc_c + row * d);
  });
}

// Dense step: output and lse, mass scores, the top-k of the fp32-rounded mass
// per (head, block), and the complement cache for that selection.
void or_attn_refresh(const double *q, const double *k, const double *v, int64_t h, int64_t T, int64_t d, double scale,
                     int64_t Bt, int64_t kk, double *O, double *lse, double *mass, int32_t *idx, double *m_c,
                     double *l_c, double *acc_c) {
  or_dense_attention(q, k, v, h, T, d, scale, O, lse);
  or_attn_mass(q, k, h, T, d, scale, Bt, mass);
  const int64_t rows = h * block_count(T, Bt);
  std::vector<float> m32(rows * T);
  for (int64_t i = 0; i < rows * T; ++i) m32[i] = static_cast<float>(mass[i]);
  or_topk_cols(m32.data(), rows, T, kk, idx);
  or_complement_partial(q, k, v, idx, kk, h, T, d, scale, Bt, m_c, l_c, acc_c);
}

}  // extern "C"
