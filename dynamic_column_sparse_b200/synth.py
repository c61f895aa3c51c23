"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module draws numbers and nothing else: it holds none of the column-sparse
delta method's arithmetic (no GELU, no softmax, no selection, no cache update).
Both sides of every parity check receive arrays produced here.

Generator (counter based, so any element can be produced on its own):

* ``splitmix64`` (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014; the finaliser as popularised by Vigna) turns the
  counter ``n`` of a stream into 64 random bits: ``mix(key + (n + 1) * GOLDEN)``.
* A stream key is ``mix(seed * 2**32 + tensor_id)``; each tensor of a workload
  uses its own ``tensor_id`` so tensors never share bits.
* "Normal" values are an Irwin-Hall sum of the four 16-bit lanes of one 64-bit
  draw, centred and rescaled to unit variance: ``z = (S + 2) / 65536 - 2``
  times ``sqrt(3)``. Every step is exact or a single IEEE double operation, so a
  host and a device implementation agree bit for bit. The tails stop at
  +-2*sqrt(3); mean 0 and variance 1 are exact up to 2**-32.
* Values are formed in float64, converted to float32 (round to nearest even)
  and then to bfloat16 (round to nearest even) where a tensor is stored as bf16.

The drift model of the configurations (activations that change slowly across
diffusion steps, Chipmunk blog post, "Slow-Changing, Sparse Activations") is
``next = prev + sigma * z`` on the decoded bf16 values, re-rounded to bf16.
"""
from __future__ import annotations

import math

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_C1 = np.uint64(0xBF58476D1CE4E5B9)
_C2 = np.uint64(0x94D049BB133111EB)
SQRT3 = math.sqrt(3.0)

# tensor ids of one layer workload; kept stable so fixtures stay reproducible
TID = {
    "x_prev": 1, "x_drift": 2, "w1t": 3, "b1": 4, "w2": 5, "b2": 6,
    "q_prev": 11, "k_prev": 12, "v_prev": 13, "q_drift": 14, "k_drift": 15, "v_drift": 16,
    "scores": 21, "scores_ties": 22, "a_cache": 31, "y_cache": 32,
    "m_c": 41, "l_c": 42, "acc_c": 43,
}


def _mix(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.uint64, copy=True)
    with np.errstate(over="ignore"):
        z ^= z >> np.uint64(30)
        z *= _C1
        z ^= z >> np.uint64(27)
        z *= _C2
        z ^= z >> np.uint64(31)
    return z


def stream_key(seed: int, tensor_id: int) -> np.uint64:
    base = np.array([(int(seed) << 32) + int(tensor_id)], dtype=np.uint64)
    return _mix(base)[0]


def raw_bits(seed: int, tensor_id: int, start: int, count: int) -> np.ndarray:
    """64-bit draws number ``start .. start+count-1`` of stream (seed, tensor_id)."""
    key = stream_key(seed, tensor_id)
    n = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(key + n * GOLDEN)


_CHUNK = 1 << 20


def _normal_chunk(key: np.uint64, start: int, count: int, out: np.ndarray) -> None:
    z = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z *= GOLDEN
        z += key
        t = np.empty_like(z)
        np.right_shift(z, np.uint64(30), out=t)
        z ^= t
        z *= _C1
        np.right_shift(z, np.uint64(27), out=t)
        z ^= t
        z *= _C2
        np.right_shift(z, np.uint64(31), out=t)
        z ^= t
    m16 = np.uint64(0xFFFF)
    np.bitwise_and(z, m16, out=t)
    s = t.copy()
    for sh in (16, 32):
        np.right_shift(z, np.uint64(sh), out=t)
        t &= m16
        s += t
    np.right_shift(z, np.uint64(48), out=t)
    s += t
    np.multiply(s.astype(np.float64) + 2.0, 1.0 / 65536.0, out=out)
    out -= 2.0
    out *= SQRT3


def normal_f64(seed: int, tensor_id: int, count: int, start: int = 0) -> np.ndarray:
    """Irwin-Hall(4) normals of stream (seed, tensor_id), draws start .. start+count-1."""
    key = stream_key(seed, tensor_id)
    out = np.empty(count, dtype=np.float64)
    for c0 in range(0, count, _CHUNK):
        n = min(_CHUNK, count - c0)
        _normal_chunk(key, start + c0, n, out[c0:c0 + n])
    return out


def normal_f64_at(seed: int, tensor_id: int, counters: np.ndarray) -> np.ndarray:
    """The normals of stream (seed, tensor_id) at arbitrary draw numbers
    (the same values normal_f64 gives at those positions)."""
    key = stream_key(seed, tensor_id)
    cnt = np.asarray(counters, dtype=np.uint64).ravel()
    bits = np.empty(cnt.size, dtype=np.uint64)
    with np.errstate(over="ignore"):
        for c0 in range(0, cnt.size, _CHUNK):
            bits[c0:c0 + _CHUNK] = _mix(key + (cnt[c0:c0 + _CHUNK] + np.uint64(1)) * GOLDEN)
    m16 = np.uint64(0xFFFF)
    s = (bits & m16) + ((bits >> np.uint64(16)) & m16) + ((bits >> np.uint64(32)) & m16) + (bits >> np.uint64(48))
    return (((s.astype(np.float64) + 2.0) / 65536.0 - 2.0) * SQRT3).reshape(np.shape(counters))


def rows_bf16(seed: int, tensor_id: int, row_len: int, rows: np.ndarray, std: float = 1.0) -> np.ndarray:
    """Selected rows of the row-major tensor normal_bf16(seed, tensor_id, (R, row_len), std)."""
    rows = np.asarray(rows, dtype=np.uint64)
    counters = rows[:, None] * np.uint64(row_len) + np.arange(row_len, dtype=np.uint64)[None, :]
    return to_bf16(std * normal_f64_at(seed, tensor_id, counters))


def drift_rows_bf16(prev_rows_bits: np.ndarray, seed: int, tensor_id: int, row_len: int, rows: np.ndarray,
                    sigma: float) -> np.ndarray:
    """drift_bf16 restricted to selected rows of a row-major tensor."""
    rows = np.asarray(rows, dtype=np.uint64)
    counters = rows[:, None] * np.uint64(row_len) + np.arange(row_len, dtype=np.uint64)[None, :]
    return to_bf16(bf16_bits_to_f64(prev_rows_bits) + sigma * normal_f64_at(seed, tensor_id, counters))


def uniform_f64(seed: int, tensor_id: int, count: int, start: int = 0) -> np.ndarray:
    bits = raw_bits(seed, tensor_id, start, count)
    return (bits >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


def f32_to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even; NaN stays a quiet NaN."""
    b = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32)
    nan = (b & np.uint32(0x7FFFFFFF)) > np.uint32(0x7F800000)
    rounded = (b + (np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1)))) >> np.uint32(16)
    out = rounded.astype(np.uint16)
    out[nan] = np.uint16(0x7FC0)
    return out


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def to_bf16(x64: np.ndarray) -> np.ndarray:
    return f32_to_bf16_bits(np.asarray(x64, dtype=np.float64).astype(np.float32))


def normal_bf16(seed: int, tensor_id: int, shape, std: float = 1.0, mean: float = 0.0) -> np.ndarray:
    count = int(np.prod(shape))
    return to_bf16(mean + std * normal_f64(seed, tensor_id, count)).reshape(shape)


def drift_bf16(prev_bits: np.ndarray, seed: int, tensor_id: int, sigma: float) -> np.ndarray:
    """``bf16(prev + sigma * z)``: the slow drift of activations between steps."""
    z = normal_f64(seed, tensor_id, prev_bits.size).reshape(prev_bits.shape)
    return to_bf16(bf16_bits_to_f64(prev_bits) + sigma * z)


# --------------------------------------------------------------------------- workloads

def mlp_layer(seed: int, T: int, D: int, H: int, sigma: float, step: int = 1):
    """bf16 bit arrays of one MLP layer: x_prev, x_t (after ``step`` drift draws), W1^T, b1, W2, b2.

    W ~ N(0, 1/fan_in) (fan_in = D for W1, H for W2), biases ~ N(0, 0.02^2),
    x_prev ~ N(0, 1).
    """
    x_prev = normal_bf16(seed, TID["x_prev"], (T, D))
    x_t = x_prev
    for s in range(step):
        x_t = drift_bf16(x_t, seed + 1000 * s, TID["x_drift"], sigma)
    w1t = normal_bf16(seed, TID["w1t"], (H, D), std=1.0 / math.sqrt(D))
    b1 = normal_bf16(seed, TID["b1"], (H,), std=0.02)
    w2 = normal_bf16(seed, TID["w2"], (H, D), std=1.0 / math.sqrt(H))
    b2 = normal_bf16(seed, TID["b2"], (D,), std=0.02)
    return dict(x_prev=x_prev, x_t=x_t, w1t=w1t, b1=b1, w2=w2, b2=b2)


def attn_layer(seed: int, T: int, h: int, d: int, sigma: float, step: int = 1):
    """bf16 bit arrays [T][h][d] of Q, K, V at the previous and the current step."""
    out = {}
    for name in ("q", "k", "v"):
        prev = normal_bf16(seed, TID[name + "_prev"], (T, h, d))
        cur = prev
        for s in range(step):
            cur = drift_bf16(cur, seed + 1000 * s, TID[name + "_drift"], sigma)
        out[name + "_prev"] = prev
        out[name] = cur
    return out


def score_rows(seed: int, rows: int, n: int, ties: bool = False) -> np.ndarray:
    """Non-negative fp32 scores shaped like column-L1 / attention-mass rows.

    With ``ties`` about a third of the entries are snapped to a coarse grid so
    that equal keys straddle the selection threshold.
    """
    z = normal_f64(seed, TID["scores"], rows * n).reshape(rows, n)
    s = np.abs(z) * (1.0 + 0.25 * np.abs(normal_f64(seed, TID["scores"], rows * n, start=rows * n).reshape(rows, n)))
    if ties:
        u = uniform_f64(seed, TID["scores_ties"], rows * n).reshape(rows, n)
        snap = u < 0.35
        s = np.where(snap, np.round(s * 4.0) / 4.0, s)
    return s.astype(np.float32)
