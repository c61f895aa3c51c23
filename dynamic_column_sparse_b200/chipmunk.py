"""Python binding of ``libchipmunk.so`` (the C ABI in include/chipmunk.h).

Argument marshalling only: each function checks dtypes, shapes and devices of
the torch tensors it is given, passes their device pointers and the current
CUDA stream to the C entry point of the same name, and raises
``ChipmunkError`` on a non-zero status. Every step runs in the library's CUDA
kernels; there is no fallback. If the library is missing or cannot be loaded
the first call raises.

Layouts (all tensors on the same CUDA device, contiguous):

* MLP: x [T][D] bf16, w1t [H][D] bf16 (W1 transposed), b1 [H] bf16,
  w2 [H][D] bf16, b2 [D] bf16, idx [nb][k] int32, a_cache [nb][H][Bt] bf16,
  y_cache [T][D] fp32, out [T][D] bf16.
* Attention: q, k, v [T][h][128] bf16, idx [h][nb][k] int32, m_c, l_c [h][T]
  fp32, acc_c [h][T][128] fp32, o [T][h][128] bf16.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libchipmunk.so")

OK = 0
ERR_INVALID_ARG, ERR_SHAPE, ERR_ALIGNMENT, ERR_CUDA, ERR_DEVICE, ERR_UNSUPPORTED, ERR_WORKSPACE = 1, 2, 3, 4, 5, 6, 7
OP_TOPK, OP_MLP_DELTA, OP_ATTN_DELTA, OP_REFRESH, OP_MLP_DELTA_FP8 = 0, 1, 2, 3, 4
REFRESH_MLP, REFRESH_ATTN = 0, 1

EXPORTS = (
    "chipmunk_topk_cols", "chipmunk_mlp_delta", "chipmunk_mlp_delta_up", "chipmunk_mlp_delta_down",
    "chipmunk_attn_delta", "chipmunk_dense_refresh",
    "chipmunk_gather_cols", "chipmunk_scatter_cols", "chipmunk_workspace_bytes", "chipmunk_status_string",
    "chipmunk_last_error", "chipmunk_read_device_status", "chipmunk_version", "chipmunk_mlp_delta_noalloc",
    "chipmunk_selftest_bounded_wait", "chipmunk_mlp_delta_fp8", "chipmunk_quantize_e4m3_rows",
)
NOALLOC_SCRATCH_BYTES = 64 << 20


class ChipmunkError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"chipmunk status {status}: {message}")
        self.status = status


class MlpArgs(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int64), ("D", ctypes.c_int64), ("H", ctypes.c_int64),
        ("Bt", ctypes.c_int32), ("k", ctypes.c_int32),
        ("x", ctypes.c_void_p), ("w1t", ctypes.c_void_p), ("b1", ctypes.c_void_p),
        ("w2", ctypes.c_void_p), ("b2", ctypes.c_void_p), ("idx", ctypes.c_void_p),
        ("a_cache", ctypes.c_void_p), ("y_cache", ctypes.c_void_p), ("out", ctypes.c_void_p),
    ]


class MlpFp8Args(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int64), ("D", ctypes.c_int64), ("H", ctypes.c_int64),
        ("Bt", ctypes.c_int32), ("k", ctypes.c_int32),
        ("x8", ctypes.c_void_p), ("sx", ctypes.c_void_p), ("w1t8", ctypes.c_void_p), ("s1", ctypes.c_void_p),
        ("b1", ctypes.c_void_p), ("w2_8", ctypes.c_void_p), ("g2", ctypes.c_void_p), ("s_delta", ctypes.c_float),
        ("idx", ctypes.c_void_p), ("a_cache", ctypes.c_void_p), ("y_cache", ctypes.c_void_p), ("out", ctypes.c_void_p),
    ]


class AttnArgs(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int64), ("h", ctypes.c_int32), ("d", ctypes.c_int32),
        ("Bt", ctypes.c_int32), ("k", ctypes.c_int32), ("scale", ctypes.c_float),
        ("q", ctypes.c_void_p), ("kk", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("idx", ctypes.c_void_p), ("m_c", ctypes.c_void_p), ("l_c", ctypes.c_void_p),
        ("acc_c", ctypes.c_void_p), ("o", ctypes.c_void_p),
        ("cache_format", ctypes.c_int32), ("lse_c", ctypes.c_void_p), ("o_c", ctypes.c_void_p),
    ]


class RefreshArgs(ctypes.Structure):
    _fields_ = [
        ("kind", ctypes.c_int32), ("first_step", ctypes.c_int32),
        ("mlp", MlpArgs), ("attn", AttnArgs), ("scores", ctypes.c_void_p),
    ]


_lib = None
_lock = threading.Lock()


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads the shared library once (raises if it is missing)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise ChipmunkError(6, f"{path} not found: build it with `python -m dynamic_column_sparse_b200.build`")
        lib = ctypes.CDLL(path)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        sig = {
            "chipmunk_topk_cols": [vp, i64, i64, i64, i32, vp, i64, vp, sz, vp],
            "chipmunk_mlp_delta": [ctypes.POINTER(MlpArgs), vp, sz, vp],
            "chipmunk_mlp_delta_up": [ctypes.POINTER(MlpArgs), vp, sz, vp],
            "chipmunk_mlp_delta_down": [ctypes.POINTER(MlpArgs), vp, sz, vp],
            "chipmunk_attn_delta": [ctypes.POINTER(AttnArgs), vp, sz, vp],
            "chipmunk_dense_refresh": [ctypes.POINTER(RefreshArgs), vp, sz, vp],
            "chipmunk_gather_cols": [vp, i64, i64, i32, vp, i32, vp, vp],
            "chipmunk_scatter_cols": [vp, i64, i64, i32, vp, i32, vp, vp],
            "chipmunk_read_device_status": [ctypes.POINTER(i32), vp],
            "chipmunk_mlp_delta_noalloc": [ctypes.POINTER(MlpArgs), vp],
            "chipmunk_selftest_bounded_wait": [vp],
            "chipmunk_mlp_delta_fp8": [ctypes.POINTER(MlpFp8Args), vp, sz, vp],
            "chipmunk_quantize_e4m3_rows": [vp, i64, i64, vp, vp, vp],
        }
        for name, argtypes in sig.items():
            fn = getattr(lib, name)
            fn.argtypes = argtypes
            fn.restype = i32
        lib.chipmunk_workspace_bytes.argtypes = [i32, vp]
        lib.chipmunk_workspace_bytes.restype = sz
        lib.chipmunk_status_string.argtypes = [i32]
        lib.chipmunk_status_string.restype = ctypes.c_char_p
        lib.chipmunk_last_error.argtypes = []
        lib.chipmunk_last_error.restype = ctypes.c_char_p
        lib.chipmunk_version.argtypes = []
        lib.chipmunk_version.restype = ctypes.c_char_p
        _lib = lib
        return lib


def _check(st: int):
    if st != OK:
        lib = load_library()
        raise ChipmunkError(st, f"{lib.chipmunk_status_string(st).decode()}: {lib.chipmunk_last_error().decode()}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def version() -> str:
    return load_library().chipmunk_version().decode()


def workspace_bytes(op: int, args=None) -> int:
    lib = load_library()
    return int(lib.chipmunk_workspace_bytes(op, None if args is None else ctypes.byref(args)))


def read_device_status(stream=None) -> int:
    lib = load_library()
    v = ctypes.c_int32(0)
    st = lib.chipmunk_read_device_status(ctypes.byref(v), _stream(stream))
    if st not in (OK, ERR_DEVICE):
        _check(st)
    return int(v.value)


# ------------------------------------------------------------------ top-k

def topk_cols(scores: torch.Tensor, k: int, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """k largest fp32 scores of each row (ties to the lower index) as ascending int32 indices."""
    lib = load_library()
    _need(scores, "scores", torch.float32)
    if scores.dim() != 2:
        raise ValueError("scores must be 2-D [rows][n]")
    rows, n = scores.shape
    if out is None:
        out = torch.empty((rows, k), dtype=torch.int32, device=scores.device)
    _need(out, "out", torch.int32, (rows, k))
    _check(lib.chipmunk_topk_cols(_ptr(scores), rows, n, n, k, _ptr(out), k, None, 0, _stream(stream)))
    return out


# ------------------------------------------------------------------ MLP

def _mlp_args(x, w1t, b1, w2, b2, idx, a_cache, y_cache, out, Bt, k):
    T, D = x.shape
    H = w1t.shape[0]
    nb = (T + Bt - 1) // Bt
    _need(x, "x", torch.bfloat16, (T, D))
    _need(w1t, "w1t", torch.bfloat16, (H, D))
    _need(b1, "b1", torch.bfloat16, (H,))
    _need(w2, "w2", torch.bfloat16, (H, D))
    if b2 is not None:
        _need(b2, "b2", torch.bfloat16, (D,))
    if idx is not None:
        _need(idx, "idx", torch.int32, (nb, k))
    _need(a_cache, "a_cache", torch.bfloat16, (nb, H, Bt))
    _need(y_cache, "y_cache", torch.float32, (T, D))
    if out is not None:
        _need(out, "out", torch.bfloat16, (T, D))
    return MlpArgs(T, D, H, Bt, k, x.data_ptr(), w1t.data_ptr(), b1.data_ptr(), w2.data_ptr(),
                   0 if b2 is None else b2.data_ptr(), 0 if idx is None else idx.data_ptr(),
                   a_cache.data_ptr(), y_cache.data_ptr(), 0 if out is None else out.data_ptr())


def mlp_workspace_bytes(T: int, H: int, k: int, Bt: int = 128) -> int:
    a = MlpArgs(T, 64, H, Bt, k)
    return workspace_bytes(OP_MLP_DELTA, a)


def mlp_delta(x, w1t, b1, w2, idx, a_cache, y_cache, out=None, Bt=128, workspace=None, stream=None, part=None):
    """Sparse MLP step: recompute the selected columns, update a_cache / y_cache in place, write out.

    ``part`` = "up" or "down" runs only that kernel (chipmunk_mlp_delta_up /
    _down); both need the same workspace.
    """
    lib = load_library()
    k = idx.shape[1]
    a = _mlp_args(x, w1t, b1, w2, None, idx, a_cache, y_cache, out, Bt, k)
    need = workspace_bytes(OP_MLP_DELTA, a)
    if need and workspace is None:
        if part is not None:
            raise ValueError("a split MLP step needs an explicit workspace shared by both parts")
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    fn = {None: lib.chipmunk_mlp_delta, "up": lib.chipmunk_mlp_delta_up, "down": lib.chipmunk_mlp_delta_down}[part]
    _check(fn(ctypes.byref(a), _ptr(workspace), ws_bytes, _stream(stream)))
    return out


def mlp_delta_noalloc(x, w1t, b1, w2, idx, a_cache, y_cache, out=None, Bt=128, stream=None):
    """mlp_delta without caller scratch: for callers that cannot allocate device
    memory. The library's fixed 64 MiB scratch array (reserved on a device at
    this call's first use there) is shared by every call, so calls must not
    overlap on the GPU; larger problems raise with status ERR_WORKSPACE."""
    lib = load_library()
    a = _mlp_args(x, w1t, b1, w2, None, idx, a_cache, y_cache, out, Bt, idx.shape[1])
    _check(lib.chipmunk_mlp_delta_noalloc(ctypes.byref(a), _stream(stream)))
    return out


def mlp_refresh(x, w1t, b1, w2, b2, a_cache, y_cache, idx, scores, out=None, Bt=128, first_step=False, stream=None):
    """Dense MLP step: rebuild a_cache / y_cache, write the column scores and the new selection idx."""
    lib = load_library()
    k = idx.shape[1]
    a = _mlp_args(x, w1t, b1, w2, b2, idx, a_cache, y_cache, out, Bt, k)
    _need(scores, "scores", torch.float32, (a_cache.shape[0], w1t.shape[0]))
    r = RefreshArgs(REFRESH_MLP, 1 if first_step else 0, a, AttnArgs(), scores.data_ptr())
    _check(lib.chipmunk_dense_refresh(ctypes.byref(r), None, 0, _stream(stream)))
    return out


# ------------------------------------------------------------------ FP8 MLP step

def _need_codes(t, name, shape):
    """e4m3 codes: torch.uint8 or torch.float8_e4m3fn storage."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype not in (torch.uint8, getattr(torch, "float8_e4m3fn", torch.uint8)):
        raise TypeError(f"{name} must hold e4m3 codes (uint8 or float8_e4m3fn), got {t.dtype}")
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def quantize_e4m3_rows(x, codes=None, scales=None, stream=None):
    """Rows of bf16 x [R][C] to e4m3 codes [R][C] (uint8) and per-row fp32 scales [R]: x ~ scale * code."""
    lib = load_library()
    _need(x, "x", torch.bfloat16)
    if x.dim() != 2:
        raise ValueError("x must be 2-D")
    R, C = x.shape
    if codes is None:
        codes = torch.empty((R, C), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((R,), dtype=torch.float32, device=x.device)
    _need_codes(codes, "codes", (R, C))
    _need(scales, "scales", torch.float32, (R,))
    _check(lib.chipmunk_quantize_e4m3_rows(_ptr(x), R, C, _ptr(codes), _ptr(scales), _stream(stream)))
    return codes, scales


def mlp_fp8_workspace_bytes(T: int, H: int, k: int) -> int:
    return workspace_bytes(OP_MLP_DELTA_FP8, MlpFp8Args(T, 256, H, 128, k))


def mlp_delta_fp8(x8, sx, w1t8, s1, b1, w2_8, g2, s_delta, idx, a_cache, y_cache, out=None, workspace=None,
                  stream=None):
    """FP8 form of the sparse MLP step (chipmunk_mlp_delta_fp8): e4m3 operands with per-token (sx),
    per-hidden-unit (s1) scales, deltas rounded to e4m3 after multiplying by g2 = s2 / s_delta."""
    lib = load_library()
    T, D = x8.shape
    H = w1t8.shape[0]
    nb = (T + 127) // 128
    k = idx.shape[1]
    _need_codes(x8, "x8", (T, D))
    _need(sx, "sx", torch.float32, (T,))
    _need_codes(w1t8, "w1t8", (H, D))
    _need(s1, "s1", torch.float32, (H,))
    _need(b1, "b1", torch.bfloat16, (H,))
    _need_codes(w2_8, "w2_8", (H, D))
    _need(g2, "g2", torch.float32, (H,))
    _need(idx, "idx", torch.int32, (nb, k))
    _need(a_cache, "a_cache", torch.bfloat16, (nb, H, 128))
    _need(y_cache, "y_cache", torch.float32, (T, D))
    if out is not None:
        _need(out, "out", torch.bfloat16, (T, D))
    a = MlpFp8Args(T, D, H, 128, k, x8.data_ptr(), sx.data_ptr(), w1t8.data_ptr(), s1.data_ptr(), b1.data_ptr(),
                   w2_8.data_ptr(), g2.data_ptr(), float(s_delta), idx.data_ptr(), a_cache.data_ptr(),
                   y_cache.data_ptr(), 0 if out is None else out.data_ptr())
    need = workspace_bytes(OP_MLP_DELTA_FP8, a)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x8.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.chipmunk_mlp_delta_fp8(ctypes.byref(a), _ptr(workspace), ws_bytes, _stream(stream)))
    return out


# ------------------------------------------------------------------ attention

ATTN_CACHE_PARTIAL = 0
ATTN_CACHE_COMPACT = 1


def _attn_args(q, k, v, idx, m_c, l_c, acc_c, o, scale, kk, lse_c=None, o_c=None):
    """Partial-form cache (m_c, l_c, acc_c) or, with lse_c / o_c given, the compact form."""
    T, h, d = q.shape
    nb = (T + 127) // 128
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _need(t, name, torch.bfloat16, (T, h, d))
    _need(idx, "idx", torch.int32, (h, nb, kk))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if lse_c is not None:
        _need(lse_c, "lse_c", torch.float32, (h, T))
        _need(o_c, "o_c", torch.bfloat16, (h, T, d))
        return AttnArgs(T, h, d, 128, kk, float(scale), q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(),
                        None, None, None, o.data_ptr(), ATTN_CACHE_COMPACT, lse_c.data_ptr(), o_c.data_ptr())
    _need(m_c, "m_c", torch.float32, (h, T))
    _need(l_c, "l_c", torch.float32, (h, T))
    _need(acc_c, "acc_c", torch.float32, (h, T, d))
    return AttnArgs(T, h, d, 128, kk, float(scale), q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(),
                    m_c.data_ptr(), l_c.data_ptr(), acc_c.data_ptr(), o.data_ptr(), ATTN_CACHE_PARTIAL, None, None)


def attn_delta(q, k, v, idx, m_c, l_c, acc_c, o, scale=None, stream=None):
    """Sparse attention step: selected keys recomputed, merged with the cached complement partial into o."""
    lib = load_library()
    a = _attn_args(q, k, v, idx, m_c, l_c, acc_c, o, scale, idx.shape[2])
    _check(lib.chipmunk_attn_delta(ctypes.byref(a), None, 0, _stream(stream)))
    return o


def attn_delta_compact(q, k, v, idx, lse_c, o_c, o, scale=None, stream=None):
    """Sparse attention step against the compact complement cache (lse_c fp32 [h][T], o_c bf16 [h][T][d])."""
    lib = load_library()
    a = _attn_args(q, k, v, idx, None, None, None, o, scale, idx.shape[2], lse_c=lse_c, o_c=o_c)
    _check(lib.chipmunk_attn_delta(ctypes.byref(a), None, 0, _stream(stream)))
    return o


def attn_refresh_workspace_bytes(T: int, h: int, k: int, keep_mass: bool) -> int:
    """Workspace of an attention refresh: the row log-sum-exp, plus the fused mass/top-k kernel's row
    buffers when the mass is not kept (``scores=None``)."""
    a = AttnArgs(T, h, 128, 128, k, 1.0)
    return workspace_bytes(OP_REFRESH, RefreshArgs(REFRESH_ATTN, 0, MlpArgs(), a, 16 if keep_mass else None))


def attn_refresh(q, k, v, idx, m_c, l_c, acc_c, o, scores=None, scale=None, workspace=None, stream=None, lse_c=None,
                 o_c=None):
    """Dense attention step: o, new selection idx and the complement cache (partial form m_c, l_c, acc_c;
    or, with lse_c and o_c given and m_c, l_c, acc_c None, the compact form). With ``scores`` [h][nb][T]
    fp32 the attention mass is also written there; without it the mass stays in the workspace's row
    buffers (the top-k is taken on it inside the mass kernel)."""
    lib = load_library()
    a = _attn_args(q, k, v, idx, m_c, l_c, acc_c, o, scale, idx.shape[2], lse_c=lse_c, o_c=o_c)
    T, h = q.shape[0], q.shape[1]
    if scores is not None:
        _need(scores, "scores", torch.float32, (h, (T + 127) // 128, T))
    r = RefreshArgs(REFRESH_ATTN, 0, MlpArgs(), a, None if scores is None else scores.data_ptr())
    need = workspace_bytes(OP_REFRESH, r)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.chipmunk_dense_refresh(ctypes.byref(r), _ptr(workspace), ws_bytes, _stream(stream)))
    return o


# ------------------------------------------------------------------ cache columns

def gather_cols(a_cache, idx, packed=None, stream=None):
    """packed[b][j] = a_cache[b][idx[b][j]] (each a run of Bt bf16)."""
    lib = load_library()
    nb, H, Bt = a_cache.shape
    k = idx.shape[1]
    _need(a_cache, "a_cache", torch.bfloat16)
    _need(idx, "idx", torch.int32, (nb, k))
    if packed is None:
        packed = torch.empty((nb, k, Bt), dtype=torch.bfloat16, device=a_cache.device)
    _need(packed, "packed", torch.bfloat16, (nb, k, Bt))
    _check(lib.chipmunk_gather_cols(_ptr(a_cache), nb, H, Bt, _ptr(idx), k, _ptr(packed), _stream(stream)))
    return packed


def scatter_cols(packed, idx, a_cache, stream=None):
    """a_cache[b][idx[b][j]] = packed[b][j]."""
    lib = load_library()
    nb, H, Bt = a_cache.shape
    k = idx.shape[1]
    _need(a_cache, "a_cache", torch.bfloat16)
    _need(idx, "idx", torch.int32, (nb, k))
    _need(packed, "packed", torch.bfloat16, (nb, k, Bt))
    _check(lib.chipmunk_scatter_cols(_ptr(packed), nb, H, Bt, _ptr(idx), k, _ptr(a_cache), _stream(stream)))
    return a_cache
