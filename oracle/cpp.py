"""Python face of the C++ fp64 oracle (``oracle/chipmunk_oracle.cpp``).

TEST INFRASTRUCTURE ONLY, like the C++ source it loads: only the tests, the
smoke check in ``__graft_entry__`` and the CPU-baseline / reference legs of
``bench.py`` may use it. It imports nothing from the CUDA package.

``CppOracle(path)`` wraps one build of the C++ oracle with the same functions,
argument conventions and return values as the numpy oracle
(``oracle/chipmunk_oracle.py``); every function's arithmetic runs in C++ and
this file only converts arrays and shapes. ``build()`` compiles the shared
library with g++ (it is rebuilt when the source is newer).
"""
from __future__ import annotations

import ctypes
import math
import os
import shutil
import subprocess
import threading

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "chipmunk_oracle.cpp")
LIB = os.path.join(HERE, "liboracle.so")
CXXFLAGS = ["-O3", "-march=x86-64-v3", "-std=c++17", "-fPIC", "-shared", "-Wall", "-Wextra"]
NEG_INF = -math.inf

_build_lock = threading.Lock()


def compile_source(src: str, out: str) -> str:
    """g++ build of one oracle source file into a shared library."""
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        raise RuntimeError("no C++ compiler found to build the oracle")
    res = subprocess.run([cxx] + CXXFLAGS + ["-o", out, src, "-lpthread"], capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"oracle build failed:\n{res.stdout}{res.stderr}")
    return out


def build(force: bool = False) -> str:
    """Builds oracle/liboracle.so from the C++ source if it is missing or older than the source."""
    with _build_lock:
        if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
            tmp = LIB + f".tmp{os.getpid()}"
            compile_source(SRC, tmp)
            os.replace(tmp, LIB)
    return LIB


_D = ctypes.POINTER(ctypes.c_double)
_I32 = ctypes.POINTER(ctypes.c_int32)
_U16 = ctypes.POINTER(ctypes.c_uint16)
_U32 = ctypes.POINTER(ctypes.c_uint32)
_U8 = ctypes.POINTER(ctypes.c_uint8)
_F32 = ctypes.POINTER(ctypes.c_float)
_I64 = ctypes.c_int64
_SIGS = {
    "or_set_threads": (None, [ctypes.c_int]),
    "or_threads": (ctypes.c_int, []),
    "or_bf16_decode": (None, [_U16, _I64, _D]),
    "or_bf16_round": (None, [_D, _I64, _U16]),
    "or_k_from_density": (_I64, [_I64, _I64]),
    "or_block_count": (_I64, [_I64, _I64]),
    "or_block_range": (None, [_I64, _I64, _I64, ctypes.POINTER(_I64), ctypes.POINTER(_I64)]),
    "or_gelu_tanh": (None, [_D, _I64, _D]),
    "or_dense_mlp": (None, [_D, _D, _D, _D, _D, _I64, _I64, _I64, _D, _D]),
    "or_mlp_delta": (None, [_D, _D, _D, _D, _I32, _I64, _D, _D, _I64, _I64, _I64, _I64, _D, _D]),
    "or_mlp_scores": (None, [_D, _D, _I64, _I64, _I64, ctypes.c_int, _D]),
    "or_ordered_key": (None, [_F32, _I64, _U32]),
    "or_topk_cols": (None, [_F32, _I64, _I64, _I64, _I32]),
    "or_mlp_refresh": (None, [_D, _D, _D, _D, _D, _D, _I64, _I64, _I64, _I64, _I64, ctypes.c_int, _D, _D, _D, _I32]),
    "or_e4m3_encode": (None, [_F32, _I64, _U8]),
    "or_e4m3_decode": (None, [_U8, _I64, _D]),
    "or_quantize_rows_e4m3": (None, [_F32, _I64, _I64, _U8, _F32]),
    "or_mlp_delta_fp8": (None, [_U8, _F32, _U8, _F32, _D, _U8, _F32, ctypes.c_float, _I32, _I64, _D, _D, _I64, _I64,
                                _I64, _I64, _D, _D]),
    "or_attn_partial": (None, [_D, _I64, _D, _D, _I64, _I64, ctypes.c_double, _D, _D, _D]),
    "or_merge_partials": (None, [_D, _D, _D, _D, _D, _D, _I64, _I64, _D, _D, _D]),
    "or_finish": (None, [_D, _D, _I64, _I64, _D]),
    "or_attn_delta": (None, [_D, _D, _D, _I32, _I64, _D, _D, _D, _I64, _I64, _I64, ctypes.c_double, _I64, _D,
                             ctypes.POINTER(_I64), _I64]),
    "or_compact_partial": (None, [_D, _D, _D, _I64, _I64, _D, _D]),
    "or_attn_delta_compact": (None, [_D, _D, _D, _I32, _I64, _D, _D, _I64, _I64, _I64, ctypes.c_double, _I64, _D]),
    "or_dense_attention": (None, [_D, _D, _D, _I64, _I64, _I64, ctypes.c_double, _D, _D]),
    "or_attn_mass_rows": (None, [_D, _I64, _D, _I64, _I64, ctypes.c_double, _D]),
    "or_attn_mass": (None, [_D, _D, _I64, _I64, _I64, ctypes.c_double, _I64, _D]),
    "or_complement_partial": (None, [_D, _D, _D, _I32, _I64, _I64, _I64, _I64, ctypes.c_double, _I64, _D, _D, _D]),
    "or_attn_refresh": (None, [_D, _D, _D, _I64, _I64, _I64, ctypes.c_double, _I64, _I64, _D, _D, _D, _I32, _D, _D,
                               _D]),
}


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a, ptr_type):
    return a.ctypes.data_as(ptr_type)


class CppOracle:
    """One build of the C++ oracle, with the numpy oracle's function signatures."""

    NEG_INF = NEG_INF

    def __init__(self, path: str):
        self.path = path
        self.lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(self.lib, name)
            fn.restype = res
            fn.argtypes = args

    # ---------------------------------------------------------------- threads

    def set_threads(self, n: int) -> None:
        """Worker threads of the C++ oracle (0: one per hardware thread)."""
        self.lib.or_set_threads(int(n))

    def threads(self) -> int:
        return int(self.lib.or_threads())

    # ---------------------------------------------------------------- storage

    def bf16_decode(self, bits):
        b = np.ascontiguousarray(bits, dtype=np.uint16)
        out = np.empty(b.shape, dtype=np.float64)
        self.lib.or_bf16_decode(_p(b, _U16), b.size, _p(out, _D))
        return out

    def bf16_round(self, x):
        a = _f64(x)
        out = np.empty(a.shape, dtype=np.uint16)
        self.lib.or_bf16_round(_p(a, _D), a.size, _p(out, _U16))
        return out

    @staticmethod
    def f32(x):
        return np.asarray(x, dtype=np.float64).astype(np.float32)

    def k_from_density(self, n, density_permille):
        return int(self.lib.or_k_from_density(int(n), int(density_permille)))

    def blocks(self, T, Bt):
        r0, r1 = _I64(), _I64()
        out = []
        for b in range(int(self.lib.or_block_count(int(T), int(Bt)))):
            self.lib.or_block_range(b, int(T), int(Bt), ctypes.byref(r0), ctypes.byref(r1))
            out.append((b, r0.value, r1.value))
        return out

    # ---------------------------------------------------------------- MLP

    def gelu_tanh(self, u):
        a = _f64(u)
        out = np.empty(a.shape)
        self.lib.or_gelu_tanh(_p(a, _D), a.size, _p(out, _D))
        return out

    def dense_mlp(self, x, W1, b1, W2, b2):
        x, w1t, b1, W2, b2 = _f64(x), _f64(np.asarray(W1).T), _f64(b1), _f64(W2), _f64(b2)
        T, D = x.shape
        H = w1t.shape[0]
        a = np.empty((T, H))
        y = np.empty((T, D))
        self.lib.or_dense_mlp(_p(x, _D), _p(w1t, _D), _p(b1, _D), _p(W2, _D), _p(b2, _D), T, D, H, _p(a, _D),
                              _p(y, _D))
        return a, y

    def mlp_delta(self, x, W1, b1, W2, idx, A_cache, Y_cache, Bt):
        x, w1t, b1, W2 = _f64(x), _f64(np.asarray(W1).T), _f64(b1), _f64(W2)
        A, Y = _f64(A_cache), _f64(Y_cache)
        T, D = x.shape
        H = w1t.shape[0]
        nb = len(self.blocks(T, Bt))
        ix = np.ascontiguousarray(np.asarray(idx, dtype=np.int32).reshape(nb, -1))
        A_new = np.empty_like(A)
        Y_new = np.empty_like(Y)
        self.lib.or_mlp_delta(_p(x, _D), _p(w1t, _D), _p(b1, _D), _p(W2, _D), _p(ix, _I32), ix.shape[1], _p(A, _D),
                              _p(Y, _D), T, D, H, int(Bt), _p(A_new, _D), _p(Y_new, _D))
        return A_new, Y_new

    def mlp_scores(self, a, A_cache, Bt, first_step):
        a = _f64(a)
        T, H = a.shape
        A = a if A_cache is None else _f64(A_cache)
        out = np.empty((len(self.blocks(T, Bt)), H))
        self.lib.or_mlp_scores(_p(a, _D), _p(A, _D), T, H, int(Bt), 1 if first_step else 0, _p(out, _D))
        return out

    def mlp_refresh(self, x, W1, b1, W2, b2, A_old, Bt, k, first_step):
        x, w1t, b1, W2, b2 = _f64(x), _f64(np.asarray(W1).T), _f64(b1), _f64(W2), _f64(b2)
        T, D = x.shape
        H = w1t.shape[0]
        nb = len(self.blocks(T, Bt))
        if not 0 <= k <= H:
            raise ValueError("k out of range")
        A = np.zeros((T, H)) if A_old is None else _f64(A_old)
        a, y = np.empty((T, H)), np.empty((T, D))
        scores = np.empty((nb, H))
        idx = np.empty((nb, k), dtype=np.int32)
        self.lib.or_mlp_refresh(_p(x, _D), _p(w1t, _D), _p(b1, _D), _p(W2, _D), _p(b2, _D), _p(A, _D), T, D, H,
                                int(Bt), int(k), 1 if first_step else 0, _p(a, _D), _p(y, _D), _p(scores, _D),
                                _p(idx, _I32))
        return dict(a=a, y=y, scores=scores, idx=idx)

    # ---------------------------------------------------------------- FP8

    def e4m3_encode(self, x32):
        x = np.ascontiguousarray(x32, dtype=np.float32)
        out = np.empty(x.shape, dtype=np.uint8)
        self.lib.or_e4m3_encode(_p(x, _F32), x.size, _p(out, _U8))
        return out

    def e4m3_decode(self, codes):
        c = np.ascontiguousarray(codes, dtype=np.uint8)
        out = np.empty(c.shape)
        self.lib.or_e4m3_decode(_p(c, _U8), c.size, _p(out, _D))
        return out

    def quantize_rows_e4m3(self, x):
        x = np.ascontiguousarray(np.atleast_2d(x), dtype=np.float32)
        rows, cols = x.shape
        codes = np.empty((rows, cols), dtype=np.uint8)
        scales = np.empty(rows, dtype=np.float32)
        self.lib.or_quantize_rows_e4m3(_p(x, _F32), rows, cols, _p(codes, _U8), _p(scales, _F32))
        return codes, scales

    def mlp_delta_fp8(self, x8, sx, w1t8, s1, b1, w2_8, g2, s_delta, idx, A_cache, Y_cache, Bt):
        x8 = np.ascontiguousarray(x8, dtype=np.uint8)
        w1t8 = np.ascontiguousarray(w1t8, dtype=np.uint8)
        w2_8 = np.ascontiguousarray(w2_8, dtype=np.uint8)
        sx, s1, g2 = (np.ascontiguousarray(a, dtype=np.float32) for a in (sx, s1, g2))
        b1 = _f64(b1)
        A, Y = _f64(A_cache), _f64(Y_cache)
        T, D = x8.shape
        H = w1t8.shape[0]
        nb = len(self.blocks(T, Bt))
        ix = np.ascontiguousarray(np.asarray(idx, dtype=np.int32).reshape(nb, -1))
        A_new, Y_new = np.empty_like(A), np.empty_like(Y)
        self.lib.or_mlp_delta_fp8(_p(x8, _U8), _p(sx, _F32), _p(w1t8, _U8), _p(s1, _F32), _p(b1, _D), _p(w2_8, _U8),
                                  _p(g2, _F32), float(s_delta), _p(ix, _I32), ix.shape[1], _p(A, _D), _p(Y, _D), T, D,
                                  H, int(Bt), _p(A_new, _D), _p(Y_new, _D))
        return A_new, Y_new

    # ---------------------------------------------------------------- selection

    def ordered_key(self, s32):
        s = np.ascontiguousarray(s32, dtype=np.float32)
        out = np.empty(s.shape, dtype=np.uint32)
        self.lib.or_ordered_key(_p(s, _F32), s.size, _p(out, _U32))
        return out

    def topk_cols(self, scores32, k):
        s = np.ascontiguousarray(np.atleast_2d(np.asarray(scores32, dtype=np.float32)))
        rows, n = s.shape
        if not 0 <= k <= n:
            raise ValueError("k out of range")
        out = np.empty((rows, k), dtype=np.int32)
        self.lib.or_topk_cols(_p(s, _F32), rows, n, int(k), _p(out, _I32))
        return out

    # ---------------------------------------------------------------- attention

    def attn_partial(self, q, k, v, scale):
        q, k, v = _f64(q), _f64(k), _f64(v)
        n, d = q.shape
        m_out, l_out, acc = np.empty(n), np.empty(n), np.empty((n, v.shape[1]))
        self.lib.or_attn_partial(_p(q, _D), n, _p(k, _D), _p(v, _D), k.shape[0], d, float(scale), _p(m_out, _D),
                                 _p(l_out, _D), _p(acc, _D))
        return m_out, l_out, acc

    def merge_partials(self, p1, p2):
        (m1, l1, a1), (m2, l2, a2) = p1, p2
        m1, l1, a1, m2, l2, a2 = (_f64(t) for t in (m1, l1, a1, m2, l2, a2))
        n, d = m1.size, a1.shape[-1]
        M, L, A = np.empty(m1.shape), np.empty(m1.shape), np.empty(a1.shape)
        self.lib.or_merge_partials(_p(m1, _D), _p(l1, _D), _p(a1, _D), _p(m2, _D), _p(l2, _D), _p(a2, _D), n, d,
                                   _p(M, _D), _p(L, _D), _p(A, _D))
        return M, L, A

    def finish(self, p):
        _, l, acc = p
        l, acc = _f64(l), _f64(acc)
        out = np.empty(acc.shape)
        self.lib.or_finish(_p(l, _D), _p(acc, _D), l.size, acc.shape[-1], _p(out, _D))
        return out

    def _attn_args(self, q, k, v, idx, Bt):
        q, k, v = _f64(q), _f64(k), _f64(v)
        h, T, d = q.shape
        nb = len(self.blocks(T, Bt))
        ix = np.ascontiguousarray(np.asarray(idx, dtype=np.int32).reshape(h, nb, -1))
        return q, k, v, ix, h, T, d

    def attn_delta(self, q, k, v, idx, m_c, l_c, acc_c, scale, Bt, tiles=None):
        q, k, v, ix, h, T, d = self._attn_args(q, k, v, idx, Bt)
        m_c, l_c, acc_c = _f64(m_c), _f64(l_c), _f64(acc_c)
        if tiles is None:
            out = np.empty((h, T, d))
            self.lib.or_attn_delta(_p(q, _D), _p(k, _D), _p(v, _D), _p(ix, _I32), ix.shape[2], _p(m_c, _D),
                                   _p(l_c, _D), _p(acc_c, _D), h, T, d, float(scale), int(Bt), _p(out, _D), None, 0)
            return out
        tl = np.ascontiguousarray(np.asarray(tiles, dtype=np.int64).reshape(-1, 2))
        out = np.zeros((h, T, d))
        self.lib.or_attn_delta(_p(q, _D), _p(k, _D), _p(v, _D), _p(ix, _I32), ix.shape[2], _p(m_c, _D), _p(l_c, _D),
                               _p(acc_c, _D), h, T, d, float(scale), int(Bt), _p(out, _D), _p(tl, ctypes.POINTER(_I64)), tl.shape[0])
        return out

    def compact_partial(self, m, l, acc):
        m, l, acc = _f64(m), _f64(l), _f64(acc)
        lse, o = np.empty(m.shape), np.empty(acc.shape)
        self.lib.or_compact_partial(_p(m, _D), _p(l, _D), _p(acc, _D), m.size, acc.shape[-1], _p(lse, _D), _p(o, _D))
        return lse, o

    def attn_delta_compact(self, q, k, v, idx, lse_c, o_c, scale, Bt):
        q, k, v, ix, h, T, d = self._attn_args(q, k, v, idx, Bt)
        lse_c, o_c = _f64(lse_c), _f64(o_c)
        out = np.empty((h, T, d))
        self.lib.or_attn_delta_compact(_p(q, _D), _p(k, _D), _p(v, _D), _p(ix, _I32), ix.shape[2], _p(lse_c, _D),
                                       _p(o_c, _D), h, T, d, float(scale), int(Bt), _p(out, _D))
        return out

    def dense_attention(self, q, k, v, scale):
        q, k, v = _f64(q), _f64(k), _f64(v)
        h, T, d = q.shape
        O, lse = np.empty((h, T, d)), np.empty((h, T))
        self.lib.or_dense_attention(_p(q, _D), _p(k, _D), _p(v, _D), h, T, d, float(scale), _p(O, _D), _p(lse, _D))
        return O, lse

    def attn_mass_rows(self, q_rows, k, scale):
        q, k = _f64(q_rows), _f64(k)
        out = np.empty(k.shape[0])
        self.lib.or_attn_mass_rows(_p(q, _D), q.shape[0], _p(k, _D), k.shape[0], q.shape[1], float(scale),
                                   _p(out, _D))
        return out

    def attn_mass(self, q, k, scale, Bt):
        q, k = _f64(q), _f64(k)
        h, T, d = q.shape
        out = np.empty((h, len(self.blocks(T, Bt)), T))
        self.lib.or_attn_mass(_p(q, _D), _p(k, _D), h, T, d, float(scale), int(Bt), _p(out, _D))
        return out

    def complement_partial(self, q, k, v, idx, scale, Bt):
        q, k, v, ix, h, T, d = self._attn_args(q, k, v, idx, Bt)
        m_c, l_c, acc_c = np.empty((h, T)), np.empty((h, T)), np.empty((h, T, d))
        self.lib.or_complement_partial(_p(q, _D), _p(k, _D), _p(v, _D), _p(ix, _I32), ix.shape[2], h, T, d,
                                       float(scale), int(Bt), _p(m_c, _D), _p(l_c, _D), _p(acc_c, _D))
        return m_c, l_c, acc_c

    def attn_refresh(self, q, k, v, scale, Bt, kk):
        q, k, v = _f64(q), _f64(k), _f64(v)
        h, T, d = q.shape
        if not 0 <= kk <= T:
            raise ValueError("k out of range")
        nb = len(self.blocks(T, Bt))
        O, lse, mass = np.empty((h, T, d)), np.empty((h, T)), np.empty((h, nb, T))
        idx = np.empty((h, nb, kk), dtype=np.int32)
        m_c, l_c, acc_c = np.empty((h, T)), np.empty((h, T)), np.empty((h, T, d))
        self.lib.or_attn_refresh(_p(q, _D), _p(k, _D), _p(v, _D), h, T, d, float(scale), int(Bt), int(kk), _p(O, _D),
                                 _p(lse, _D), _p(mass, _D), _p(idx, _I32), _p(m_c, _D), _p(l_c, _D), _p(acc_c, _D))
        return dict(O=O, lse=lse, mass=mass, idx=idx, m_c=m_c, l_c=l_c, acc_c=acc_c)


FUNCTIONS = ("bf16_decode", "bf16_round", "f32", "k_from_density", "blocks", "gelu_tanh", "dense_mlp", "mlp_delta",
             "e4m3_encode", "e4m3_decode", "quantize_rows_e4m3", "mlp_delta_fp8",
             "mlp_scores", "mlp_refresh", "ordered_key", "topk_cols", "attn_partial", "merge_partials", "finish",
             "attn_delta", "compact_partial", "attn_delta_compact", "dense_attention", "attn_mass_rows", "attn_mass",
             "complement_partial", "attn_refresh")

_default = None


def default() -> CppOracle:
    """The oracle built from oracle/chipmunk_oracle.cpp (built on first use)."""
    global _default
    if _default is None:
        _default = CppOracle(build())
    return _default
