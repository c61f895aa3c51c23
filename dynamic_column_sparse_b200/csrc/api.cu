// api.cu - the C ABI (include/chipmunk.h): argument checks, TMA tensor maps,
// launch sequences and the device status word.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/chipmunk.h"
#include "abi_internal.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace cm {
uint32_t attn_smem_bytes(int mode, int64_t T);
}

namespace {

// Written by kernels when a bounded wait gives up; read and cleared by
// chipmunk_read_device_status. One instance per device.
__device__ int g_status = 0;

thread_local std::string g_last_error;

chipmunk_status fail(chipmunk_status st, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
chipmunk_status fail(chipmunk_status st, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

chipmunk_status cuda_fail(cudaError_t e, const char *what) {
  return fail(CHIPMUNK_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int *g_status_ptr[kMaxDevices] = {};
bool g_device_ok[kMaxDevices] = {};
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Per-device set-up: checks for an sm_100 device and resolves the status word.
chipmunk_status device_setup(int **status_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(CHIPMUNK_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_device_ok[dev]) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0)
      return fail(CHIPMUNK_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a only", dev, major,
                  minor);
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_status);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status word)");
    g_status_ptr[dev] = static_cast<int *>(p);
    if (g_encode == nullptr) {
      void *fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
      if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr)
        return fail(CHIPMUNK_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    g_device_ok[dev] = true;
  }
  *status_out = g_status_ptr[dev];
  return CHIPMUNK_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Tensor map of rank 2 or 3 with 128-byte swizzle (bf16 elements, or bytes when
// `bytes` is set). dims/box innermost first.
chipmunk_status make_map(CUtensorMap *m, const void *base, int rank, const uint64_t *dims, const uint64_t *strides_bytes,
                         const uint32_t *box, const char *what, bool bytes = false) {
  cuuint64_t gd[3], gs[2];
  cuuint32_t bx[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
  }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
  CUresult r = g_encode(m, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank,
                        const_cast<void *>(base), gd, gs, bx, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CHIPMUNK_ERR_CUDA, "cuTensorMapEncodeTiled(%s) failed with %d", what, int(r));
  return CHIPMUNK_OK;
}

// rows x cols bf16 matrix, row-major, box = box_cols x box_rows
chipmunk_status map2d(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                      uint32_t box_rows, const char *what) {
  const uint64_t dims[2] = {cols, rows};
  const uint64_t strides[1] = {cols * 2};
  const uint32_t box[2] = {box_cols, box_rows};
  return make_map(m, base, 2, dims, strides, box, what);
}

// [nb][rows][Bt] bf16, box 64 tokens x 64 rows x 1 block
chipmunk_status map_blocks(CUtensorMap *m, const void *base, uint64_t nb, uint64_t rows, uint32_t Bt,
                           const char *what) {
  const uint64_t dims[3] = {Bt, rows, nb};
  const uint64_t strides[2] = {uint64_t(Bt) * 2, rows * Bt * 2};
  const uint32_t box[3] = {64, 64, 1};
  return make_map(m, base, 3, dims, strides, box, what);
}

#define CM_CHECK(expr)                         \
  do {                                         \
    chipmunk_status _st = (expr);              \
    if (_st != CHIPMUNK_OK) return _st;        \
  } while (0)

#define CM_CUDA(expr, what)                    \
  do {                                         \
    cudaError_t _e = (expr);                   \
    if (_e != cudaSuccess) return cuda_fail(_e, what); \
  } while (0)

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

int down_bn(int64_t D) { return D % 256 == 0 ? 256 : (D % 128 == 0 ? 128 : 64); }

chipmunk_status check_mlp(const chipmunk_mlp_args *a, bool refresh) {
  if (a == nullptr) return fail(CHIPMUNK_ERR_INVALID_ARG, "args is NULL");
  if (a->T < 1 || a->T > (int64_t(1) << 30)) return fail(CHIPMUNK_ERR_SHAPE, "T=%lld out of range", (long long)a->T);
  if (a->D < 64 || a->D > 16384 || a->D % 64 != 0)
    return fail(CHIPMUNK_ERR_SHAPE, "D=%lld must be a multiple of 64 in [64, 16384]", (long long)a->D);
  if (a->H < 1 || a->H > (int64_t(1) << 24)) return fail(CHIPMUNK_ERR_SHAPE, "H=%lld out of range", (long long)a->H);
  if (a->Bt != 64 && a->Bt != 128) return fail(CHIPMUNK_ERR_SHAPE, "Bt=%d must be 64 or 128", a->Bt);
  if (a->k < 0 || a->k > a->H) return fail(CHIPMUNK_ERR_INVALID_ARG, "k=%d outside [0, H=%lld]", a->k, (long long)a->H);
  const void *req[] = {a->x, a->w1t, a->b1, a->w2, a->a_cache, a->y_cache, a->idx};
  const char *names[] = {"x", "w1t", "b1", "w2", "a_cache", "y_cache", "idx"};
  for (int i = 0; i < 7; ++i) {
    if (req[i] == nullptr && !(i == 6 && !refresh && a->k == 0))
      return fail(CHIPMUNK_ERR_INVALID_ARG, "%s is NULL", names[i]);
    if (req[i] != nullptr && !aligned16(req[i])) return fail(CHIPMUNK_ERR_ALIGNMENT, "%s is not 16-byte aligned", names[i]);
  }
  if (refresh && a->b2 == nullptr) return fail(CHIPMUNK_ERR_INVALID_ARG, "b2 is NULL");
  if (a->b2 != nullptr && !aligned16(a->b2)) return fail(CHIPMUNK_ERR_ALIGNMENT, "b2 is not 16-byte aligned");
  if (a->out != nullptr && !aligned16(a->out)) return fail(CHIPMUNK_ERR_ALIGNMENT, "out is not 16-byte aligned");
  return CHIPMUNK_OK;
}

chipmunk_status check_attn(const chipmunk_attn_args *a, bool refresh) {
  if (a == nullptr) return fail(CHIPMUNK_ERR_INVALID_ARG, "args is NULL");
  if (a->T < 1 || a->T > (int64_t(1) << 30)) return fail(CHIPMUNK_ERR_SHAPE, "T=%lld out of range", (long long)a->T);
  if (a->h < 1 || a->h > 1024) return fail(CHIPMUNK_ERR_SHAPE, "h=%d out of range", a->h);
  if (a->d != 128) return fail(CHIPMUNK_ERR_SHAPE, "head dim d=%d: only 128 is built", a->d);
  if (a->Bt != 128) return fail(CHIPMUNK_ERR_SHAPE, "query block Bt=%d: only 128 is built", a->Bt);
  if (a->k < 0 || a->k > a->T) return fail(CHIPMUNK_ERR_INVALID_ARG, "k=%d outside [0, T]", a->k);
  if (!std::isfinite(a->scale)) return fail(CHIPMUNK_ERR_INVALID_ARG, "scale is not finite");
  if (refresh && cm::attn_smem_bytes(cm::kAttnComplement, a->T) > 227 * 1024)
    return fail(CHIPMUNK_ERR_SHAPE, "T=%lld too long for the complement pass", (long long)a->T);
  if (a->cache_format != CHIPMUNK_ATTN_CACHE_PARTIAL && a->cache_format != CHIPMUNK_ATTN_CACHE_COMPACT)
    return fail(CHIPMUNK_ERR_INVALID_ARG, "cache_format=%d unknown", a->cache_format);
  const bool compact = a->cache_format == CHIPMUNK_ATTN_CACHE_COMPACT;
  const void *req[] = {a->q, a->kk, a->v, a->o, a->idx, compact ? static_cast<const void *>(a->lse_c) : a->m_c,
                       compact ? a->o_c : static_cast<const void *>(a->l_c), compact ? nullptr : a->acc_c};
  const char *names[] = {"q", "kk", "v", "o", "idx", compact ? "lse_c" : "m_c", compact ? "o_c" : "l_c", "acc_c"};
  const int nreq = compact ? 7 : 8;
  for (int i = 0; i < nreq; ++i) {
    if (req[i] == nullptr && !(i == 4 && !refresh && a->k == 0))
      return fail(CHIPMUNK_ERR_INVALID_ARG, "%s is NULL", names[i]);
    if (req[i] != nullptr && !aligned16(req[i])) return fail(CHIPMUNK_ERR_ALIGNMENT, "%s is not 16-byte aligned", names[i]);
  }
  return CHIPMUNK_OK;
}

// Attention refresh scratch: the row log-sum-exp [h][T] fp32, then (when the
// caller keeps no mass tensor) one mass row buffer per persistent CTA of the
// fused mass/top-k kernel.
size_t attn_refresh_lse_bytes(const chipmunk_attn_args *a) {
  return (size_t(a->h) * size_t(a->T) * sizeof(float) + 255) & ~size_t(255);
}

size_t attn_refresh_ws(const chipmunk_refresh_args *r) {
  const chipmunk_attn_args *a = &r->attn;
  if (a->T < 1 || a->h < 1) return 0;
  size_t bytes = attn_refresh_lse_bytes(a);
  if (r->scores == nullptr) {
    const int64_t tiles = int64_t(a->h) * ceil_div(a->T, 128);
    // + 128: the row buffers start at the first 128-byte boundary after the log-sum-exp
    bytes += 128 + size_t(cm::mass_row_buffers(tiles, a->T)) * size_t(cm::mass_row_floats(a->T)) * sizeof(float);
  }
  return bytes;
}

size_t mlp_delta_ws(const chipmunk_mlp_args *a) {
  if (a->k <= 0) return 0;
  const int64_t nb = ceil_div(a->T, a->Bt);
  return size_t(nb) * size_t(ceil_div(a->k, 128) * 128) * size_t(a->Bt) * 2;
}

chipmunk_status topk_impl(const float *scores, int64_t rows, int64_t n, int64_t ld_scores, int32_t k, int32_t *idx,
                          int64_t ld_idx, int *status, cudaStream_t s) {
  cm::TopkParams p{scores, rows, n, ld_scores, k, idx, ld_idx, status};
  CM_CUDA(cm::launch_topk(p, s), "top-k launch");
  return CHIPMUNK_OK;
}

// Checks shared by the sparse MLP entry points; resolves the device set-up.
chipmunk_status mlp_delta_prologue(const chipmunk_mlp_args *a, void *ws, size_t ws_bytes, int **status) {
  CM_CHECK(check_mlp(a, false));
  const size_t need = mlp_delta_ws(a);
  if (need > 0 && (ws == nullptr || ws_bytes < need))
    return fail(CHIPMUNK_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws_bytes);
  if (need > 0 && !aligned16(ws)) return fail(CHIPMUNK_ERR_ALIGNMENT, "ws is not 16-byte aligned");
  return device_setup(status);
}

chipmunk_status mlp_up_impl(const chipmunk_mlp_args *a, void *ws, int *status, cudaStream_t s) {
  if (a->k == 0) return CHIPMUNK_OK;
  const int64_t nb = ceil_div(a->T, a->Bt);
  const int64_t nchunks = ceil_div(a->k, 128);
  CUtensorMap tm_w1t, tm_x;
  CM_CHECK(map2d(&tm_w1t, a->w1t, a->H, a->D, 64, 128, "w1t"));
  CM_CHECK(map2d(&tm_x, a->x, a->T, a->D, 64, a->Bt, "x"));
  cm::MlpUpParams up{int(a->T), int(a->D), int(a->H), a->k, a->Bt, int(nb), int(nchunks), int(nchunks * 128),
                     cm::kUpDelta, static_cast<const uint16_t *>(a->w1t), a->idx,
                     static_cast<const uint16_t *>(a->b1), static_cast<uint16_t *>(a->a_cache),
                     static_cast<uint16_t *>(ws), nullptr, status};
  CM_CUDA(cm::launch_mlp_up(up, tm_w1t, tm_x, s), "MLP up-projection launch");
  return CHIPMUNK_OK;
}

chipmunk_status mlp_down_impl(const chipmunk_mlp_args *a, void *ws, int *status, cudaStream_t s) {
  const int64_t nb = ceil_div(a->T, a->Bt);
  const int64_t k_pad = ceil_div(a->k, 128) * 128;
  const int bn = down_bn(a->D);
  cm::MlpDownParams dp{int(a->T), int(a->D), a->Bt, int(nb), int(k_pad), a->k, int(a->D / bn), bn,
                       cm::kDownAccumulate, static_cast<const uint16_t *>(a->w2), int(a->H), a->idx,
                       static_cast<const uint16_t *>(a->b2), a->y_cache, static_cast<uint16_t *>(a->out), status};
  CUtensorMap tm_d, tm_w2;
  if (a->k > 0) {
    CM_CHECK(map_blocks(&tm_d, ws, nb, k_pad, a->Bt, "delta workspace"));
    CM_CHECK(map2d(&tm_w2, a->w2, a->H, a->D, 64, 64, "w2"));
  }
  CM_CUDA(cm::launch_mlp_down(dp, tm_d, tm_w2, false, s), "MLP down-projection launch");
  return CHIPMUNK_OK;
}

chipmunk_status check_mlp_fp8(const chipmunk_mlp_fp8_args *a) {
  if (a == nullptr) return fail(CHIPMUNK_ERR_INVALID_ARG, "args is NULL");
  if (a->T < 1 || a->T > (int64_t(1) << 30)) return fail(CHIPMUNK_ERR_SHAPE, "T=%lld out of range", (long long)a->T);
  if (a->D < 256 || a->D > 16384 || a->D % 256 != 0)
    return fail(CHIPMUNK_ERR_SHAPE, "D=%lld must be a multiple of 256 in [256, 16384] for the FP8 step", (long long)a->D);
  if (a->H < 1 || a->H > (int64_t(1) << 24)) return fail(CHIPMUNK_ERR_SHAPE, "H=%lld out of range", (long long)a->H);
  if (a->Bt != 128) return fail(CHIPMUNK_ERR_SHAPE, "Bt=%d: the FP8 step is built for 128", a->Bt);
  if (a->k < 0 || a->k > a->H) return fail(CHIPMUNK_ERR_INVALID_ARG, "k=%d outside [0, H=%lld]", a->k, (long long)a->H);
  if (!(a->s_delta > 0.f) || !std::isfinite(a->s_delta)) return fail(CHIPMUNK_ERR_INVALID_ARG, "s_delta must be > 0");
  const void *req[] = {a->x8, a->sx, a->w1t8, a->s1, a->b1, a->w2_8, a->g2, a->a_cache, a->y_cache, a->idx};
  const char *names[] = {"x8", "sx", "w1t8", "s1", "b1", "w2_8", "g2", "a_cache", "y_cache", "idx"};
  for (int i = 0; i < 10; ++i) {
    if (req[i] == nullptr && !(i == 9 && a->k == 0)) return fail(CHIPMUNK_ERR_INVALID_ARG, "%s is NULL", names[i]);
    if (req[i] != nullptr && !aligned16(req[i])) return fail(CHIPMUNK_ERR_ALIGNMENT, "%s is not 16-byte aligned", names[i]);
  }
  if (a->out != nullptr && !aligned16(a->out)) return fail(CHIPMUNK_ERR_ALIGNMENT, "out is not 16-byte aligned");
  return CHIPMUNK_OK;
}

size_t mlp_delta_fp8_ws(const chipmunk_mlp_fp8_args *a) {
  if (a->k <= 0) return 0;
  return size_t(ceil_div(a->T, 128)) * size_t(ceil_div(a->k, 128) * 128) * 128;
}

}  // namespace

namespace cm {

chipmunk_status record_error(chipmunk_status st, const char *msg) { return fail(st, "%s", msg); }

chipmunk_status mlp_delta_fixed_scratch(const chipmunk_mlp_args *a, size_t scratch_bytes,
                                        chipmunk_status (*get_scratch)(void **), cudaStream_t s) {
  CM_CHECK(check_mlp(a, false));
  const size_t need = mlp_delta_ws(a);
  if (need > scratch_bytes)
    return fail(CHIPMUNK_ERR_WORKSPACE,
                "chipmunk_mlp_delta_noalloc needs %zu bytes of scratch, more than its fixed %zu; "
                "use chipmunk_mlp_delta with a caller workspace",
                need, scratch_bytes);
  int *status = nullptr;
  CM_CHECK(device_setup(&status));
  void *ws = nullptr;
  CM_CHECK(get_scratch(&ws));
  CM_CHECK(mlp_up_impl(a, ws, status, s));
  return mlp_down_impl(a, ws, status, s);
}

}  // namespace cm

extern "C" {

const char *chipmunk_version(void) { return "0.1.0"; }

const char *chipmunk_last_error(void) { return g_last_error.c_str(); }

const char *chipmunk_status_string(chipmunk_status st) {
  switch (st) {
    case CHIPMUNK_OK: return "ok";
    case CHIPMUNK_ERR_INVALID_ARG: return "invalid argument";
    case CHIPMUNK_ERR_SHAPE: return "unsupported shape";
    case CHIPMUNK_ERR_ALIGNMENT: return "misaligned pointer";
    case CHIPMUNK_ERR_CUDA: return "CUDA error";
    case CHIPMUNK_ERR_DEVICE: return "device status word set";
    case CHIPMUNK_ERR_UNSUPPORTED: return "unsupported device or option";
    case CHIPMUNK_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

size_t chipmunk_workspace_bytes(int32_t op, const void *args) {
  switch (op) {
    case CHIPMUNK_OP_MLP_DELTA:
      return args ? mlp_delta_ws(static_cast<const chipmunk_mlp_args *>(args)) : 0;
    case CHIPMUNK_OP_MLP_DELTA_FP8:
      return args ? mlp_delta_fp8_ws(static_cast<const chipmunk_mlp_fp8_args *>(args)) : 0;
    case CHIPMUNK_OP_REFRESH: {
      if (!args) return 0;
      const chipmunk_refresh_args *r = static_cast<const chipmunk_refresh_args *>(args);
      if (r->kind == CHIPMUNK_REFRESH_ATTN) return attn_refresh_ws(r);
      return 0;
    }
    default: return 0;
  }
}

chipmunk_status chipmunk_topk_cols(const float *scores, int64_t rows, int64_t n, int64_t ld_scores, int32_t k,
                                   int32_t *idx, int64_t ld_idx, void *ws, size_t ws_bytes, chipmunk_stream stream) {
  (void)ws;
  (void)ws_bytes;
  if (rows < 0 || n < 1 || n > (int64_t(1) << 30)) return fail(CHIPMUNK_ERR_SHAPE, "rows/n out of range");
  if (k < 0 || k > n) return fail(CHIPMUNK_ERR_INVALID_ARG, "k=%d outside [0, n=%lld]", k, (long long)n);
  if (ld_scores < n || ld_idx < k) return fail(CHIPMUNK_ERR_SHAPE, "leading dimension smaller than the row");
  if (rows == 0 || k == 0) return CHIPMUNK_OK;
  if (scores == nullptr || idx == nullptr) return fail(CHIPMUNK_ERR_INVALID_ARG, "scores or idx is NULL");
  if (!aligned16(scores) || !aligned16(idx)) return fail(CHIPMUNK_ERR_ALIGNMENT, "scores or idx not 16-byte aligned");
  int *status = nullptr;
  CM_CHECK(device_setup(&status));
  return topk_impl(scores, rows, n, ld_scores, k, idx, ld_idx, status, static_cast<cudaStream_t>(stream));
}

chipmunk_status chipmunk_mlp_delta(const chipmunk_mlp_args *a, void *ws, size_t ws_bytes, chipmunk_stream stream) {
  int *status = nullptr;
  CM_CHECK(mlp_delta_prologue(a, ws, ws_bytes, &status));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  CM_CHECK(mlp_up_impl(a, ws, status, s));
  return mlp_down_impl(a, ws, status, s);
}

chipmunk_status chipmunk_mlp_delta_up(const chipmunk_mlp_args *a, void *ws, size_t ws_bytes, chipmunk_stream stream) {
  int *status = nullptr;
  CM_CHECK(mlp_delta_prologue(a, ws, ws_bytes, &status));
  return mlp_up_impl(a, ws, status, static_cast<cudaStream_t>(stream));
}

chipmunk_status chipmunk_mlp_delta_down(const chipmunk_mlp_args *a, void *ws, size_t ws_bytes,
                                        chipmunk_stream stream) {
  int *status = nullptr;
  CM_CHECK(mlp_delta_prologue(a, ws, ws_bytes, &status));
  return mlp_down_impl(a, ws, status, static_cast<cudaStream_t>(stream));
}

chipmunk_status chipmunk_mlp_delta_fp8(const chipmunk_mlp_fp8_args *a, void *ws, size_t ws_bytes,
                                       chipmunk_stream stream) {
  CM_CHECK(check_mlp_fp8(a));
  const size_t need = mlp_delta_fp8_ws(a);
  if (need > 0 && (ws == nullptr || ws_bytes < need))
    return fail(CHIPMUNK_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws_bytes);
  if (need > 0 && !aligned16(ws)) return fail(CHIPMUNK_ERR_ALIGNMENT, "ws is not 16-byte aligned");
  int *status = nullptr;
  CM_CHECK(device_setup(&status));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t nb = ceil_div(a->T, 128);
  const int64_t nchunks = ceil_div(a->k, 128);
  const int64_t k_pad = nchunks * 128;
  if (a->k > 0) {
    CUtensorMap tm_x;
    {
      const uint64_t dims[2] = {uint64_t(a->D), uint64_t(a->T)};
      const uint64_t strides[1] = {uint64_t(a->D)};
      const uint32_t box[2] = {128, 128};
      CM_CHECK(make_map(&tm_x, a->x8, 2, dims, strides, box, "x8", true));
    }
    cm::MlpUpParams up{int(a->T), int(a->D), int(a->H), a->k, 128, int(nb), int(nchunks), int(k_pad), cm::kUpDelta,
                       static_cast<const uint16_t *>(a->w1t8), a->idx, static_cast<const uint16_t *>(a->b1),
                       static_cast<uint16_t *>(a->a_cache), static_cast<uint16_t *>(ws), nullptr, status,
                       a->sx, a->s1, a->g2};
    CM_CUDA(cm::launch_mlp_up_fp8(up, tm_x, s), "FP8 MLP up-projection launch");
  }
  cm::MlpDownParams dp{int(a->T), int(a->D), 128, int(nb), int(k_pad), a->k, int(a->D / 256), 256,
                       cm::kDownAccumulate, static_cast<const uint16_t *>(a->w2_8), int(a->H), a->idx, nullptr,
                       a->y_cache, static_cast<uint16_t *>(a->out), status, a->s_delta};
  CUtensorMap tm_d;
  if (a->k > 0) {
    const uint64_t dims[3] = {128, uint64_t(k_pad), uint64_t(nb)};
    const uint64_t strides[2] = {128, uint64_t(k_pad) * 128};
    const uint32_t box[3] = {128, 128, 1};
    CM_CHECK(make_map(&tm_d, ws, 3, dims, strides, box, "delta codes", true));
  }
  CM_CUDA(cm::launch_mlp_down_fp8(dp, tm_d, s), "FP8 MLP down-projection launch");
  return CHIPMUNK_OK;
}

chipmunk_status chipmunk_quantize_e4m3_rows(const void *x, int64_t rows, int64_t cols, void *codes, float *scales,
                                            chipmunk_stream stream) {
  if (rows < 0 || cols < 16 || cols % 16 != 0) return fail(CHIPMUNK_ERR_SHAPE, "rows/cols out of range (cols a multiple of 16)");
  if (rows == 0) return CHIPMUNK_OK;
  if (x == nullptr || codes == nullptr || scales == nullptr) return fail(CHIPMUNK_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(x) || !aligned16(codes)) return fail(CHIPMUNK_ERR_ALIGNMENT, "x or codes not 16-byte aligned");
  int *status = nullptr;
  CM_CHECK(device_setup(&status));
  CM_CUDA(cm::launch_quantize_e4m3_rows(static_cast<const uint16_t *>(x), rows, cols, static_cast<uint8_t *>(codes),
                                        scales, status, static_cast<cudaStream_t>(stream)),
          "quantize launch");
  return CHIPMUNK_OK;
}

chipmunk_status chipmunk_attn_delta(const chipmunk_attn_args *a, void *ws, size_t ws_bytes, chipmunk_stream stream) {
  (void)ws;
  (void)ws_bytes;
  CM_CHECK(check_attn(a, false));
  int *status = nullptr;
  CM_CHECK(device_setup(&status));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t nb = ceil_div(a->T, 128);
  const uint64_t cols = uint64_t(a->h) * 128;
  CUtensorMap tm_q, tm_k, tm_v;
  CM_CHECK(map2d(&tm_q, a->q, a->T, cols, 64, 128, "q"));
  CM_CHECK(map2d(&tm_k, a->kk, a->T, cols, 64, 128, "k"));
  CM_CHECK(map2d(&tm_v, a->v, a->T, cols, 64, 128, "v"));
  cm::AttnParams p{int(a->T), a->h, int(nb), a->k, a->scale * 1.4426950408889634f,
                   static_cast<const uint16_t *>(a->kk), static_cast<const uint16_t *>(a->v), a->idx, a->m_c,
                   a->l_c, a->acc_c, static_cast<uint16_t *>(a->o), nullptr, status,
                   a->cache_format == CHIPMUNK_ATTN_CACHE_COMPACT, a->lse_c, static_cast<uint16_t *>(a->o_c)};
  CM_CUDA(cm::launch_attn(cm::kAttnDelta, p, tm_q, tm_k, tm_v, s), "attention delta launch");
  return CHIPMUNK_OK;
}

chipmunk_status chipmunk_dense_refresh(const chipmunk_refresh_args *r, void *ws, size_t ws_bytes,
                                       chipmunk_stream stream) {
  if (r == nullptr) return fail(CHIPMUNK_ERR_INVALID_ARG, "args is NULL");
  if (r->scores != nullptr && !aligned16(r->scores)) return fail(CHIPMUNK_ERR_ALIGNMENT, "scores is not 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (r->kind == CHIPMUNK_REFRESH_MLP) {
    if (r->scores == nullptr) return fail(CHIPMUNK_ERR_INVALID_ARG, "scores is NULL (the MLP refresh needs it)");
    const chipmunk_mlp_args *a = &r->mlp;
    CM_CHECK(check_mlp(a, true));
    int *status = nullptr;
    CM_CHECK(device_setup(&status));
    const int64_t nb = ceil_div(a->T, a->Bt);
    const int64_t nchunks = ceil_div(a->H, 128);
    const int bn = down_bn(a->D);
    CUtensorMap tm_w1t, tm_x, tm_a, tm_w2;
    CM_CHECK(map2d(&tm_w1t, a->w1t, a->H, a->D, 64, 128, "w1t"));
    CM_CHECK(map2d(&tm_x, a->x, a->T, a->D, 64, a->Bt, "x"));
    CM_CHECK(map_blocks(&tm_a, a->a_cache, nb, a->H, a->Bt, "activation cache"));
    CM_CHECK(map2d(&tm_w2, a->w2, a->H, a->D, 64, 64, "w2 tile"));
    cm::MlpUpParams up{int(a->T), int(a->D), int(a->H), int(a->H), a->Bt, int(nb), int(nchunks), int(nchunks * 128),
                       r->first_step ? cm::kUpRefreshFirst : cm::kUpRefresh, static_cast<const uint16_t *>(a->w1t),
                       nullptr, static_cast<const uint16_t *>(a->b1), static_cast<uint16_t *>(a->a_cache), nullptr,
                       r->scores, status};
    CM_CUDA(cm::launch_mlp_up(up, tm_w1t, tm_x, s), "MLP refresh up-projection launch");
    cm::MlpDownParams dp{int(a->T), int(a->D), a->Bt, int(nb), int(a->H), int(a->H), int(a->D / bn), bn,
                         cm::kDownOverwrite, static_cast<const uint16_t *>(a->w2), int(a->H), nullptr,
                         static_cast<const uint16_t *>(a->b2), a->y_cache, static_cast<uint16_t *>(a->out), status};
    CM_CUDA(cm::launch_mlp_down(dp, tm_a, tm_w2, true, s), "MLP refresh down-projection launch");
    return topk_impl(r->scores, nb, a->H, a->H, a->k, a->idx, a->k, status, s);
  }
  if (r->kind == CHIPMUNK_REFRESH_ATTN) {
    const chipmunk_attn_args *a = &r->attn;
    CM_CHECK(check_attn(a, true));
    const size_t need = attn_refresh_ws(r);
    if (ws == nullptr || ws_bytes < need)
      return fail(CHIPMUNK_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws_bytes);
    if (!aligned16(ws)) return fail(CHIPMUNK_ERR_ALIGNMENT, "ws is not 16-byte aligned");
    int *status = nullptr;
    CM_CHECK(device_setup(&status));
    const int64_t nb = ceil_div(a->T, 128);
    const uint64_t cols = uint64_t(a->h) * 128;
    CUtensorMap tm_q, tm_k, tm_v;
    CM_CHECK(map2d(&tm_q, a->q, a->T, cols, 64, 128, "q"));
    CM_CHECK(map2d(&tm_k, a->kk, a->T, cols, 64, 128, "k tile"));
    CM_CHECK(map2d(&tm_v, a->v, a->T, cols, 64, 128, "v tile"));
    float *lse = static_cast<float *>(ws);
    const float sl2 = a->scale * 1.4426950408889634f;
    cm::AttnParams dense{int(a->T), a->h, int(nb), a->k, sl2, static_cast<const uint16_t *>(a->kk),
                         static_cast<const uint16_t *>(a->v), a->idx, a->m_c, a->l_c, a->acc_c,
                         static_cast<uint16_t *>(a->o), lse, status,
                         a->cache_format == CHIPMUNK_ATTN_CACHE_COMPACT, a->lse_c, static_cast<uint16_t *>(a->o_c)};
    CM_CUDA(cm::launch_attn(cm::kAttnDense, dense, tm_q, tm_k, tm_v, s), "attention refresh dense launch");
    const uintptr_t rows_at = (reinterpret_cast<uintptr_t>(ws) + attn_refresh_lse_bytes(a) + 127) & ~uintptr_t(127);
    float *row_buf = r->scores != nullptr ? nullptr : reinterpret_cast<float *>(rows_at);
    cm::MassParams mp{int(a->T), a->h, int(nb), a->k, sl2, lse, r->scores, row_buf, a->idx, status};
    CM_CUDA(cm::launch_attn_mass_select(mp, tm_q, tm_k, s), "attention mass and top-k launch");
    CM_CUDA(cm::launch_attn(cm::kAttnComplement, dense, tm_q, tm_k, tm_v, s), "attention complement launch");
    return CHIPMUNK_OK;
  }
  return fail(CHIPMUNK_ERR_INVALID_ARG, "refresh kind %d unknown", r->kind);
}

chipmunk_status chipmunk_gather_cols(const void *a_cache, int64_t nb, int64_t H, int32_t Bt, const int32_t *idx,
                                     int32_t k, void *packed, chipmunk_stream stream) {
  if (Bt != 64 && Bt != 128) return fail(CHIPMUNK_ERR_SHAPE, "Bt=%d must be 64 or 128", Bt);
  if (nb < 0 || H < 1 || k < 0 || k > H) return fail(CHIPMUNK_ERR_SHAPE, "nb/H/k out of range");
  if (nb == 0 || k == 0) return CHIPMUNK_OK;
  if (!a_cache || !idx || !packed) return fail(CHIPMUNK_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(a_cache) || !aligned16(idx) || !aligned16(packed))
    return fail(CHIPMUNK_ERR_ALIGNMENT, "pointer not 16-byte aligned");
  int *status = nullptr;
  CM_CHECK(device_setup(&status));
  CM_CUDA(cm::launch_gather_cols(static_cast<const uint16_t *>(a_cache), nb, H, Bt, idx, k,
                                 static_cast<uint16_t *>(packed), status, static_cast<cudaStream_t>(stream)),
          "gather launch");
  return CHIPMUNK_OK;
}

chipmunk_status chipmunk_scatter_cols(const void *packed, int64_t nb, int64_t H, int32_t Bt, const int32_t *idx,
                                      int32_t k, void *a_cache, chipmunk_stream stream) {
  if (Bt != 64 && Bt != 128) return fail(CHIPMUNK_ERR_SHAPE, "Bt=%d must be 64 or 128", Bt);
  if (nb < 0 || H < 1 || k < 0 || k > H) return fail(CHIPMUNK_ERR_SHAPE, "nb/H/k out of range");
  if (nb == 0 || k == 0) return CHIPMUNK_OK;
  if (!a_cache || !idx || !packed) return fail(CHIPMUNK_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(a_cache) || !aligned16(idx) || !aligned16(packed))
    return fail(CHIPMUNK_ERR_ALIGNMENT, "pointer not 16-byte aligned");
  int *status = nullptr;
  CM_CHECK(device_setup(&status));
  CM_CUDA(cm::launch_scatter_cols(static_cast<const uint16_t *>(packed), nb, H, Bt, idx, k,
                                  static_cast<uint16_t *>(a_cache), status, static_cast<cudaStream_t>(stream)),
          "scatter launch");
  return CHIPMUNK_OK;
}

chipmunk_status chipmunk_selftest_bounded_wait(chipmunk_stream stream) {
  int *status = nullptr;
  CM_CHECK(device_setup(&status));
  CM_CUDA(cm::launch_selftest_wait(status, static_cast<cudaStream_t>(stream)), "self-test launch");
  return CHIPMUNK_OK;
}

chipmunk_status chipmunk_read_device_status(int32_t *host_out, chipmunk_stream stream) {
  if (host_out == nullptr) return fail(CHIPMUNK_ERR_INVALID_ARG, "host_out is NULL");
  int *status = nullptr;
  CM_CHECK(device_setup(&status));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  CM_CUDA(cudaStreamSynchronize(s), "stream synchronize");
  int v = 0;
  CM_CUDA(cudaMemcpy(&v, status, sizeof(int), cudaMemcpyDeviceToHost), "status read");
  if (v != 0) {
    const int zero = 0;
    CM_CUDA(cudaMemcpy(status, &zero, sizeof(int), cudaMemcpyHostToDevice), "status clear");
  }
  *host_out = v;
  if (v != 0) return fail(CHIPMUNK_ERR_DEVICE, "device status word was %d", v);
  return CHIPMUNK_OK;
}

}  // extern "C"
