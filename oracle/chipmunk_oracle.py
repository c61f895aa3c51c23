"""Oracle for Chipmunk-style column-sparse cross-step deltas, in plain fp64.

TEST INFRASTRUCTURE ONLY. This module is a slow, direct CPU restatement of
what the method computes, used to check the CUDA library. Only the tests, the
smoke check in ``__graft_entry__`` and the CPU-baseline / reference legs of
``bench.py`` may import it. It shares no code with the CUDA path and imports
nothing from the package.

Source: "Chipmunk: Training-Free Acceleration of Diffusion Transformers with
Dynamic Column-Sparse Deltas" (Together AI blog post, 4/21/2025), sections
"Slow-Changing, Sparse Activations" and "Activation Deltas Across Diffusion
Steps are Very Sparse" (the attention and MLP equations and the cache-delta
identity that follows them).

Conventions (all arrays float64 unless stated):

* MLP: ``x`` [T][D], ``W1`` [D][H], ``b1`` [H], ``W2`` [H][D], ``b2`` [D];
  activations ``A`` [T][H]; outputs ``Y`` [T][D].
* Attention, per head: ``q, k, v`` [h][T][d]; partial state ``m, l`` [h][T],
  ``acc`` [h][T][d] (unnormalised, relative to ``m``).
* Tokens are grouped in blocks of ``Bt`` consecutive rows; the last block may
  be short. Selected sets are int32 index arrays, ascending, one per block
  (MLP: ``idx`` [nb][k]) or per head and query block (attention: [h][nb][k]).
* bf16 values enter decoded exactly; nothing here rounds unless a function
  says so.

Readings where the post is silent (each is listed with its reason in the
design notes): GELU is the tanh form; attention logits carry the usual
``1/sqrt(d)`` scale, passed in; the MLP column score is the block's column L1
norm of ``a - A_cache`` (``sum |a|`` on a first step with no cache); the
attention score is the block's column sum of softmax probabilities; selection
keeps the k largest fp32 scores, ties to the lower index.
"""
from __future__ import annotations

import math

import numpy as np

NEG_INF = -math.inf


# --------------------------------------------------------------------------- storage

def bf16_decode(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact float64 values."""
    with np.errstate(invalid="ignore"):
        return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """float64 -> bf16 bit patterns: to float32 (nearest even), then to bf16 (nearest even).

    Used only to store the oracle's own results in the library's storage type
    (for example a cache that both sides then start from).
    """
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    is_nan = np.isnan(f)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    r[is_nan] = 0x7FC0
    return r


def f32(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def k_from_density(n: int, density_permille: int) -> int:
    """Selected count for a kept fraction given in per mille, rounded down."""
    return (int(n) * int(density_permille)) // 1000


def blocks(T: int, Bt: int):
    """(b, first row, end row) of each token block; the last may be short."""
    return [(b, b * Bt, min((b + 1) * Bt, T)) for b in range((T + Bt - 1) // Bt)]


# --------------------------------------------------------------------------- MLP

def gelu_tanh(u: np.ndarray) -> np.ndarray:
    """GELU, tanh form (Hendrycks and Gimpel): the post's MLP non-linearity."""
    u = np.asarray(u, dtype=np.float64)
    return 0.5 * u * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (u + 0.044715 * u * u * u)))


def dense_mlp(x, W1, b1, W2, b2):
    """``gelu(x W1 + b1) W2 + b2`` (post: "MLP" equation; the bias is one more static vector).

    Returns the activations and the output.
    """
    a = gelu_tanh(x @ W1 + b1[None, :])
    return a, a @ W2 + b2[None, :]


def mlp_delta(x, W1, b1, W2, idx, A_cache, Y_cache, Bt):
    """One sparse step of the MLP against its cache.

    The output is a sum of rows of W2 weighted by the activations. For each
    token block the selected activation columns are recomputed; the old
    vectors ``A_cache[r, c] * W2[c]`` are subtracted from the cached output and
    the new ones added (post: the dense step rewritten as "subtract the old
    output vectors, add the new ones", restricted to the recomputed subset).
    Unselected columns keep their cached value.

    Returns (A_new, Y_new); the layer output is Y_new.
    """
    T = x.shape[0]
    A_new = np.array(A_cache, dtype=np.float64, copy=True)
    Y_new = np.array(Y_cache, dtype=np.float64, copy=True)
    for b, r0, r1 in blocks(T, Bt):
        S = np.asarray(idx[b], dtype=np.int64)
        if S.size == 0:
            continue
        a = gelu_tanh(x[r0:r1] @ W1[:, S] + b1[S][None, :])
        old = A_cache[r0:r1][:, S]
        Y_new[r0:r1] += (a - old) @ W2[S, :]
        A_new[r0:r1, S] = a
    return A_new, Y_new


def mlp_scores(a, A_cache, Bt, first_step):
    """Per block and hidden column: ``sum over the block's rows of |a - A_cache|``.

    On a first step there is no cache and the score is ``sum |a|``: the
    largest activations carry the output (post: "Activations are sparse").
    Result [nb][H] in float64.
    """
    T, H = a.shape
    out = np.zeros(((T + Bt - 1) // Bt, H))
    for b, r0, r1 in blocks(T, Bt):
        d = a[r0:r1] if first_step else a[r0:r1] - A_cache[r0:r1]
        out[b] = np.abs(d).sum(axis=0)
    return out


def mlp_refresh(x, W1, b1, W2, b2, A_old, Bt, k, first_step):
    """Dense step: full activations and output, new scores and selection, rebuilt cache.

    Returns dict(a, y, scores (float64), idx (top-k of the fp32-rounded scores)).
    The rebuilt cache is ``A = a`` and ``Y = y``.
    """
    a, y = dense_mlp(x, W1, b1, W2, b2)
    scores = mlp_scores(a, A_old, Bt, first_step)
    return dict(a=a, y=y, scores=scores, idx=topk_cols(f32(scores), k))


# --------------------------------------------------------------------------- FP8 form of the MLP step

def e4m3_encode(x32: np.ndarray) -> np.ndarray:
    """fp32 values -> e4m3 codes (OCP FP8 E4M3: bias 7, 3 mantissa bits, no infinities, NaN S.1111.111,
    largest finite 448): nearest representable value, ties to the even code, magnitudes above 448
    saturated to 448."""
    x = np.asarray(x32, dtype=np.float32).astype(np.float64)
    out = np.zeros(x.shape, dtype=np.uint8)
    flat, res = x.reshape(-1), out.reshape(-1)
    for i, v in enumerate(flat):
        if math.isnan(v):
            res[i] = 0x7F
            continue
        sign = 0x80 if math.copysign(1.0, v) < 0 else 0
        a = abs(v)
        if a >= 448.0:
            res[i] = sign | 0x7E
            continue
        if a < 2.0 ** -6:
            res[i] = sign | int(round(a * 512.0))      # round() is half-to-even
            continue
        e = math.floor(math.log2(a))
        if 2.0 ** e > a:                              # guard the logarithm's rounding
            e -= 1
        elif 2.0 ** (e + 1) <= a:
            e += 1
        r = round(a / 2.0 ** (e - 3))
        if r == 16:
            r, e = 8, e + 1
        be, m = e + 7, r - 8
        res[i] = sign | (0x7E if be > 15 or (be == 15 and m == 7) else (be << 3) | m)
    return out


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """e4m3 codes -> exact float64 values (NaN for S.1111.111)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    be, m = (c >> 3) & 15, c & 7
    val = np.where(be == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(be - 7.0))
    return np.where((be == 15) & (m == 7), np.nan, sign * val)


def quantize_rows_e4m3(x):
    """Rows of fp32 values to e4m3 codes with one scale per row, in float arithmetic:
    amax = max |x|, inv = 448 / amax, scale = amax / 448 (both 1 when amax is 0),
    code = e4m3(x * inv), so that x ~ scale * code. Returns (codes uint8, scales float32)."""
    x = np.atleast_2d(np.asarray(x, dtype=np.float32))
    amax = np.abs(x).max(axis=1)
    pos = amax > 0
    safe = np.where(pos, amax, np.float32(1.0)).astype(np.float32)
    inv = np.where(pos, np.float32(448.0) / safe, np.float32(1.0)).astype(np.float32)
    scales = np.where(pos, safe / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    return e4m3_encode((x * inv[:, None]).astype(np.float32)), scales


def mlp_delta_fp8(x8, sx, w1t8, s1, b1, w2_8, g2, s_delta, idx, A_cache, Y_cache, Bt):
    """One sparse MLP step on e4m3 operands (the library's own scaling scheme for the post's FP8
    FLUX result): x[t] ~ sx[t] x8[t], W1^T[c] ~ s1[c] w1t8[c], W2[c] ~ s2[c] w2_8[c]. For each block
    and selected column c: a = gelu(s1[c] sx[t] (x8[t] . w1t8[c]) + b1[c]); the delta against the
    cache is taken from a rounded to bf16 (as stored), multiplied by g2[c] = s2[c] / s_delta as
    floats and rounded to an e4m3 code; the cached output gains s_delta * sum_c code * w2_8[c].
    Returns (A_new, Y_new); A_new takes a."""
    xd, w1d, w2d = e4m3_decode(x8), e4m3_decode(w1t8), e4m3_decode(w2_8)
    sx, s1, g2 = (np.asarray(a, dtype=np.float32) for a in (sx, s1, g2))
    T = xd.shape[0]
    A_new = np.array(A_cache, dtype=np.float64, copy=True)
    Y_new = np.array(Y_cache, dtype=np.float64, copy=True)
    for b, r0, r1 in blocks(T, Bt):
        S = np.asarray(idx[b], dtype=np.int64)
        if S.size == 0:
            continue
        u = (xd[r0:r1] @ w1d[S].T) * s1[S].astype(np.float64)[None, :] * sx[r0:r1].astype(np.float64)[:, None]
        a = gelu_tanh(u + np.asarray(b1, dtype=np.float64)[S][None, :])
        stored = bf16_decode(bf16_round(a))
        d = (stored - A_cache[r0:r1][:, S]).astype(np.float32)
        code = e4m3_decode(e4m3_encode((d * g2[S][None, :]).astype(np.float32)))
        Y_new[r0:r1] += np.float64(np.float32(s_delta)) * (code @ w2d[S, :])
        A_new[r0:r1, S] = a
    return A_new, Y_new


# --------------------------------------------------------------------------- selection

def ordered_key(s32: np.ndarray) -> np.ndarray:
    """fp32 values -> uint32 keys whose unsigned order is the numeric order.

    Negative values have all bits flipped, others get the sign bit set; -0 is
    first mapped to +0 so the two compare equal. A NaN lands by its bits
    (+NaN above +inf, -NaN below -inf).
    """
    bits = np.ascontiguousarray(s32, dtype=np.float32).view(np.uint32).copy()
    bits[bits == np.uint32(0x80000000)] = 0
    neg = (bits & np.uint32(0x80000000)) != 0
    return np.where(neg, ~bits, bits | np.uint32(0x80000000)).astype(np.uint32)


def topk_cols(scores32: np.ndarray, k: int) -> np.ndarray:
    """k largest fp32 scores of each row, ties to the lower index, as ascending indices.

    Stable sort of (key descending, index ascending); the first k are kept.
    """
    scores32 = np.atleast_2d(np.asarray(scores32, dtype=np.float32))
    rows, n = scores32.shape
    if not 0 <= k <= n:
        raise ValueError("k out of range")
    out = np.empty((rows, k), dtype=np.int32)
    keys = ordered_key(scores32).astype(np.int64)
    for r in range(rows):
        order = np.argsort(-keys[r], kind="stable")
        out[r] = np.sort(order[:k])
    return out


# --------------------------------------------------------------------------- attention

def attn_partial(q, k, v, scale):
    """Softmax partial state of queries ``q`` [n][d] over keys ``k``, values ``v`` [m][d].

    ``m`` = row max of the logits ``scale * q k^T``, ``l`` = sum of
    ``exp(s - m)``, ``acc`` = sum of ``exp(s - m) v``. No keys: (-inf, 0, 0).
    """
    n = q.shape[0]
    if k.shape[0] == 0:
        return np.full(n, NEG_INF), np.zeros(n), np.zeros((n, v.shape[1]))
    s = scale * (q @ k.T)
    m = s.max(axis=1)
    p = np.exp(s - m[:, None])
    return m, p.sum(axis=1), p @ v


def merge_partials(p1, p2):
    """Online-softmax merge of two partial states over disjoint key sets."""
    m1, l1, a1 = p1
    m2, l2, a2 = p2
    M = np.maximum(m1, m2)
    with np.errstate(invalid="ignore"):
        w1 = np.where(m1 == NEG_INF, 0.0, np.exp(m1 - M))
        w2 = np.where(m2 == NEG_INF, 0.0, np.exp(m2 - M))
    return M, l1 * w1 + l2 * w2, a1 * w1[:, None] + a2 * w2[:, None]


def finish(p):
    """Normalised output ``acc / l`` of a partial state (0 where no key contributed)."""
    m, l, acc = p
    safe = np.where(l > 0, l, 1.0)
    return np.where((l > 0)[:, None], acc / safe[:, None], 0.0)


def attn_delta(q, k, v, idx, m_c, l_c, acc_c, scale, Bt, tiles=None):
    """Sparse attention step: recompute the selected keys, reuse the cached rest.

    For each head and query block the selected keys are attended with the
    current q, k, v and merged with the cached partial over the complementary
    keys (post: attention output as a sum of scaled rows of V, of which only a
    subset is replaced on each step). Returns O [h][T][d]. With ``tiles`` (a
    list of (head, query block) pairs) only those tiles are computed; the rest
    of O is zero.
    """
    h, T, d = q.shape
    O = np.zeros((h, T, d))
    todo = None if tiles is None else {(int(a), int(b)) for a, b in np.asarray(tiles).reshape(-1, 2)}
    for hh in range(h):
        for b, r0, r1 in blocks(T, Bt):
            if todo is not None and (hh, b) not in todo:
                continue
            S = np.asarray(idx[hh][b], dtype=np.int64)
            sel = attn_partial(q[hh, r0:r1], k[hh, S], v[hh, S], scale)
            cached = (m_c[hh, r0:r1], l_c[hh, r0:r1], acc_c[hh, r0:r1])
            O[hh, r0:r1] = finish(merge_partials(cached, sel))
    return O


def compact_partial(m, l, acc):
    """The same partial state in log-sum-exp form: ``lse = m + ln l`` and the
    normalised output ``o = acc / l``; an empty partial (l = 0) gives
    ``(-inf, 0)``. Since ``e^lse = l e^m`` and ``o e^lse = acc e^m``, a merge
    needs nothing else. (A denser encoding of the cached partial of the post's
    attention step; the encoding is this library's.)
    """
    l = np.asarray(l, dtype=np.float64)
    safe = np.where(l > 0, l, 1.0)
    lse = np.where(l > 0, np.asarray(m, dtype=np.float64) + np.log(safe), NEG_INF)
    o = np.where((l > 0)[..., None], np.asarray(acc, dtype=np.float64) / safe[..., None], 0.0)
    return lse, o


def attn_delta_compact(q, k, v, idx, lse_c, o_c, scale, Bt):
    """Sparse attention step against a complement cached as ``(lse_c, o_c)``.

    The cached complement enters the online-softmax merge as the partial
    ``(lse_c, 1, o_c)``: relative to a shared maximum M its weight is
    ``e^(lse_c - M)`` and its numerator ``o_c e^(lse_c - M)``. Returns O [h][T][d].
    """
    h, T, d = q.shape
    O = np.zeros((h, T, d))
    for hh in range(h):
        for b, r0, r1 in blocks(T, Bt):
            S = np.asarray(idx[hh][b], dtype=np.int64)
            sel = attn_partial(q[hh, r0:r1], k[hh, S], v[hh, S], scale)
            cached = (lse_c[hh, r0:r1], np.ones(r1 - r0), o_c[hh, r0:r1])
            O[hh, r0:r1] = finish(merge_partials(cached, sel))
    return O


def dense_attention(q, k, v, scale):
    """``softmax(scale q k^T) v`` per head (post: "Attention" equation) and the row log-sum-exp."""
    h, T, d = q.shape
    O = np.zeros((h, T, d))
    lse = np.zeros((h, T))
    for hh in range(h):
        m, l, acc = attn_partial(q[hh], k[hh], v[hh], scale)
        O[hh] = acc / l[:, None]
        lse[hh] = m + np.log(l)
    return O, lse


def attn_mass_rows(q_rows, k, scale):
    """Attention mass of each key for one query block ``q_rows`` [n][d] over keys ``k`` [m][d]:
    the column sums of the row softmax, ``sum over i of softmax_i(j)``."""
    s = scale * (q_rows @ k.T)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    return p.sum(axis=0)


def attn_mass(q, k, scale, Bt):
    """Attention mass of each key for each query block: column sums of the softmax.

    ``mass[h][b][j] = sum over rows i of block b of softmax_i(j)``. Result [h][nb][T].
    """
    h, T, d = q.shape
    nb = (T + Bt - 1) // Bt
    out = np.zeros((h, nb, T))
    for hh in range(h):
        for b, r0, r1 in blocks(T, Bt):
            out[hh, b] = attn_mass_rows(q[hh, r0:r1], k[hh], scale)
    return out


def complement_partial(q, k, v, idx, scale, Bt):
    """Partial state of every query over the keys its block did NOT select.

    Computed directly over the complement (not as dense minus selected), so a
    complement that holds little mass keeps its relative precision.
    Returns m_c, l_c [h][T] and acc_c [h][T][d].
    """
    h, T, d = q.shape
    m_c = np.full((h, T), NEG_INF)
    l_c = np.zeros((h, T))
    acc_c = np.zeros((h, T, d))
    for hh in range(h):
        for b, r0, r1 in blocks(T, Bt):
            keep = np.ones(T, dtype=bool)
            keep[np.asarray(idx[hh][b], dtype=np.int64)] = False
            m, l, acc = attn_partial(q[hh, r0:r1], k[hh, keep], v[hh, keep], scale)
            m_c[hh, r0:r1], l_c[hh, r0:r1], acc_c[hh, r0:r1] = m, l, acc
    return m_c, l_c, acc_c


def attn_refresh(q, k, v, scale, Bt, kk):
    """Dense step: output, mass scores, new selection and the complement cache."""
    O, lse = dense_attention(q, k, v, scale)
    mass = attn_mass(q, k, scale, Bt)
    h, nb, T = mass.shape
    idx = topk_cols(f32(mass.reshape(h * nb, T)), kk).reshape(h, nb, kk)
    m_c, l_c, acc_c = complement_partial(q, k, v, idx, scale, Bt)
    return dict(O=O, lse=lse, mass=mass, idx=idx, m_c=m_c, l_c=l_c, acc_c=acc_c)
