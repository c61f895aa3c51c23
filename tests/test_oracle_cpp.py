"""The C++ oracle against its numpy restatement, function by function.

The two are written independently from the same equations; on the same
inputs every float result must agree to 1e-12 relative to the result's
largest magnitude, and every integer result (bf16 bits, keys, indices, block
ranges, k) exactly. The inputs span the cases the pins cover (short last
blocks, empty and full selections, ties) at sizes beyond one row group,
output chunk and term chunk of the C++ loops.
"""
import numpy as np
import pytest

import oracle
from oracle import numpy_oracle as N

C = oracle.default()
g = np.random.default_rng(2024)
REL = 1e-12


def close(a, b, what):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, what
    fin = np.isfinite(b)
    assert np.array_equal(np.isfinite(a), fin), what
    assert np.array_equal(a[~fin], b[~fin]), what
    scale = max(1.0, float(np.max(np.abs(b[fin])))) if fin.any() else 1.0
    err = float(np.max(np.abs(a[fin] - b[fin]))) if fin.any() else 0.0
    assert err <= REL * scale, f"{what}: {err:.3e} > {REL} * {scale:.3e}"


def test_storage_and_counts():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    a, b = C.bf16_decode(bits), N.bf16_decode(bits)
    assert np.array_equal(np.isnan(a), np.isnan(b)) and np.array_equal(a[~np.isnan(a)], b[~np.isnan(b)])
    x = g.standard_normal(100000) * 10.0 ** g.integers(-30, 30, 100000)
    x = np.concatenate([x, [0.0, -0.0, np.inf, -np.inf, np.nan, 3.4e38, -3.4e38, 1e-45]])
    assert np.array_equal(C.bf16_round(x), N.bf16_round(x))
    for n, pm in ((12288, 300), (4352, 165), (118800, 70), (7, 999), (0, 5)):
        assert C.k_from_density(n, pm) == N.k_from_density(n, pm)
    for T, Bt in ((256, 64), (300, 128), (118800, 128), (5, 8), (128, 128)):
        assert C.blocks(T, Bt) == N.blocks(T, Bt)


def test_selection():
    s = np.concatenate([g.standard_normal((5, 300)), np.round(g.standard_normal((5, 300)) * 2) / 2]).astype(np.float32)
    s[0, :5] = [0.0, -0.0, np.inf, -np.inf, 1e-45]
    assert np.array_equal(C.ordered_key(s), N.ordered_key(s))
    for k in (0, 1, 37, 299, 300):
        assert np.array_equal(C.topk_cols(s, k), N.topk_cols(s, k)), k


def _mlp(T, D, H):
    x = g.standard_normal((T, D))
    W1 = g.standard_normal((D, H)) / np.sqrt(D)
    b1 = 0.02 * g.standard_normal(H)
    W2 = g.standard_normal((H, D)) / np.sqrt(H)
    b2 = 0.02 * g.standard_normal(D)
    return x, W1, b1, W2, b2


@pytest.mark.parametrize("T,D,H,Bt,k", [(18, 40, 300, 8, 150), (300, 192, 700, 128, 301), (64, 64, 200, 64, 0),
                                        (70, 24, 130, 64, 130)])
def test_mlp_functions(T, D, H, Bt, k):
    u = np.linspace(-9, 9, 1001)
    close(C.gelu_tanh(u), N.gelu_tanh(u), "gelu_tanh")
    x, W1, b1, W2, b2 = _mlp(T, D, H)
    for got, ref, what in zip(C.dense_mlp(x, W1, b1, W2, b2), N.dense_mlp(x, W1, b1, W2, b2), ("a", "y")):
        close(got, ref, f"dense_mlp {what}")
    A = g.standard_normal((T, H))
    Y = g.standard_normal((T, D))
    nb = (T + Bt - 1) // Bt
    idx = np.sort(np.stack([g.choice(H, k, replace=False) for _ in range(nb)]), axis=1).astype(np.int32)
    for got, ref, what in zip(C.mlp_delta(x, W1, b1, W2, idx, A, Y, Bt), N.mlp_delta(x, W1, b1, W2, idx, A, Y, Bt),
                              ("A", "Y")):
        close(got, ref, f"mlp_delta {what}")
    for first in (False, True):
        close(C.mlp_scores(A, Y[:, :1] * A, Bt, first), N.mlp_scores(A, Y[:, :1] * A, Bt, first), "mlp_scores")
        rc = C.mlp_refresh(x, W1, b1, W2, b2, A, Bt, min(k, H), first)
        rn = N.mlp_refresh(x, W1, b1, W2, b2, A, Bt, min(k, H), first)
        for key in ("a", "y", "scores"):
            close(rc[key], rn[key], f"mlp_refresh {key}")
        assert np.array_equal(rc["idx"], rn["idx"])


def _qkv(h, T, d, spread=1.0):
    return tuple(g.standard_normal((h, T, d)) * spread for _ in range(3))


@pytest.mark.parametrize("h,T,Bt,kk", [(2, 22, 8, 5), (3, 300, 128, 50), (1, 130, 64, 130), (2, 70, 64, 0)])
def test_attention_functions(h, T, Bt, kk):
    d = 16
    q, k, v = _qkv(h, T, d)
    scale = 0.3
    nb = (T + Bt - 1) // Bt
    idx = np.sort(np.stack([[g.choice(T, kk, replace=False) for _ in range(nb)] for _ in range(h)]),
                  axis=2).astype(np.int32)
    pc, pn = C.attn_partial(q[0], k[0], v[0], scale), N.attn_partial(q[0], k[0], v[0], scale)
    for a, b, what in zip(pc, pn, "mla"):
        close(a, b, f"attn_partial {what}")
    p2 = N.attn_partial(q[0], k[0, :7] * 2, v[0, :7], scale)
    for a, b, what in zip(C.merge_partials(pn, p2), N.merge_partials(pn, p2), "MLA"):
        close(a, b, f"merge_partials {what}")
    empty = (np.full(T, -np.inf), np.zeros(T), np.zeros((T, d)))
    for a, b, what in zip(C.merge_partials(empty, p2), N.merge_partials(empty, p2), "MLA"):
        close(a, b, f"merge_partials with an empty side {what}")
    close(C.finish(pn), N.finish(pn), "finish")
    close(C.finish(empty), N.finish(empty), "finish of an empty partial")
    m_c, l_c, acc_c = N.complement_partial(q, k, v, idx, scale, Bt)
    for a, b, what in zip(C.complement_partial(q, k, v, idx, scale, Bt), (m_c, l_c, acc_c), ("m", "l", "acc")):
        close(a, b, f"complement_partial {what}")
    close(C.attn_delta(q, k, v, idx, m_c, l_c, acc_c, scale, Bt), N.attn_delta(q, k, v, idx, m_c, l_c, acc_c, scale, Bt),
          "attn_delta")
    tiles = [(h - 1, nb - 1), (0, 0)]
    sub = C.attn_delta(q, k, v, idx, m_c, l_c, acc_c, scale, Bt, tiles=tiles)
    close(sub, N.attn_delta(q, k, v, idx, m_c, l_c, acc_c, scale, Bt, tiles=tiles), "attn_delta on two tiles")
    close(sub[0, :min(Bt, T)], C.attn_delta(q, k, v, idx, m_c, l_c, acc_c, scale, Bt)[0, :min(Bt, T)],
          "attn_delta, one tile against all tiles")
    lse_c, o_c = N.compact_partial(m_c, l_c, acc_c)
    for a, b, what in zip(C.compact_partial(m_c, l_c, acc_c), (lse_c, o_c), ("lse", "o")):
        close(a, b, f"compact_partial {what}")
    close(C.attn_delta_compact(q, k, v, idx, lse_c, o_c, scale, Bt),
          N.attn_delta_compact(q, k, v, idx, lse_c, o_c, scale, Bt), "attn_delta_compact")
    for a, b, what in zip(C.dense_attention(q, k, v, scale), N.dense_attention(q, k, v, scale), ("O", "lse")):
        close(a, b, f"dense_attention {what}")
    close(C.attn_mass_rows(q[0, :9], k[0], scale), N.attn_mass_rows(q[0, :9], k[0], scale), "attn_mass_rows")
    close(C.attn_mass(q, k, scale, Bt), N.attn_mass(q, k, scale, Bt), "attn_mass")
    rc, rn = C.attn_refresh(q, k, v, scale, Bt, kk), N.attn_refresh(q, k, v, scale, Bt, kk)
    assert np.array_equal(rc["idx"], rn["idx"])
    for key in ("O", "lse", "mass", "m_c", "l_c", "acc_c"):
        close(rc[key], rn[key], f"attn_refresh {key}")


def test_thread_count_does_not_change_results():
    x, W1, b1, W2, b2 = _mlp(40, 24, 150)
    q, k, v = _qkv(2, 100, 16)
    before = C.threads()
    try:
        outs = []
        for n in (1, 3):
            C.set_threads(n)
            outs.append((C.dense_mlp(x, W1, b1, W2, b2), C.attn_mass(q, k, 0.3, 32)))
    finally:
        C.set_threads(0)
    assert C.threads() == before
    assert np.array_equal(outs[0][0][0], outs[1][0][0]) and np.array_equal(outs[0][0][1], outs[1][0][1])
    assert np.array_equal(outs[0][1], outs[1][1])


def test_fp8_functions():
    codes = np.arange(256, dtype=np.uint32).astype(np.uint8)
    a, b = C.e4m3_decode(codes), N.e4m3_decode(codes)
    assert np.array_equal(np.isnan(a), np.isnan(b)) and np.array_equal(a[~np.isnan(a)], b[~np.isnan(b)])
    x = (g.standard_normal(30000) * 10.0 ** g.integers(-5, 4, 30000)).astype(np.float32)
    x[:6] = [0.0, -0.0, 448.0, 1e9, -np.inf, 2.0 ** -10]
    assert np.array_equal(C.e4m3_encode(x), N.e4m3_encode(x))
    rows = x.reshape(30, 1000).copy()
    rows[0, 4] = -1e9                                    # quantised rows hold finite values
    rows[3] = 0.0
    qc, qn = C.quantize_rows_e4m3(rows), N.quantize_rows_e4m3(rows)
    assert np.array_equal(qc[0], qn[0]) and np.array_equal(qc[1], qn[1])
    T, D, H, Bt, k = 40, 48, 70, 16, 30
    x8, sx = N.quantize_rows_e4m3(g.standard_normal((T, D)).astype(np.float32))
    w1t8, s1 = N.quantize_rows_e4m3((g.standard_normal((H, D)) / 7).astype(np.float32))
    w2_8, s2 = N.quantize_rows_e4m3((g.standard_normal((H, D)) / 8).astype(np.float32))
    b1 = 0.02 * g.standard_normal(H)
    A = N.bf16_decode(N.bf16_round(0.5 * g.standard_normal((T, H))))
    Y = g.standard_normal((T, D))
    idx = np.sort(np.stack([g.choice(H, k, replace=False) for _ in range(3)]), axis=1).astype(np.int32)
    g2 = (s2 / np.float32(1e-4)).astype(np.float32)
    rc = C.mlp_delta_fp8(x8, sx, w1t8, s1, b1, w2_8, g2, np.float32(1e-4), idx, A, Y, Bt)
    rn = N.mlp_delta_fp8(x8, sx, w1t8, s1, b1, w2_8, g2, np.float32(1e-4), idx, A, Y, Bt)
    for got, ref, what in zip(rc, rn, ("A", "Y")):
        close(got, ref, f"mlp_delta_fp8 {what}")
