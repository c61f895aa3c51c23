"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each test checks one oracle function against something fixed independently:
brute force written another way, a closed form, an invariant of the
mathematics, a special case that reduces to a textbook result, or a fixture
under tests/golden/ with its citation. A plausible mistake (a dropped term, a
wrong sign or index, a transposed operand) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest

import oracle
from oracle import numpy_oracle

# The pins run against both oracles: the C++ one (oracle.default(), what the
# GPU parity tests use) and its numpy cross-check. ``O`` is the one under test.
IMPLS = {"cpp": oracle.default, "numpy": lambda: numpy_oracle}
O = oracle


@pytest.fixture(autouse=True, params=sorted(IMPLS))
def impl(request):
    global O
    saved = O
    O = IMPLS[request.param]()
    yield request.param
    O = saved


GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def _gelu_erf(u):
    return 0.5 * u * (1.0 + math.erf(u / math.sqrt(2.0)))


# --------------------------------------------------------------------------- storage

def test_bf16_bits_fixture():
    rows = [ln.split() for ln in open(os.path.join(GOLDEN, "bf16_bits.txt")) if ln.strip() and not ln.startswith("#")]
    for expr, bits in rows:
        val = float(eval(expr, {"inf": math.inf}))  # fixture holds plain arithmetic only
        got = int(O.bf16_round(np.array([val]))[0])
        assert got == int(bits, 16), (expr, hex(got), bits)
        if not math.isinf(val) and expr not in ("1.0+2**-8", "1.0+3*2**-8", "1.0+2**-8+2**-20"):
            assert O.bf16_decode(np.array([got], dtype=np.uint16))[0] == val


def test_bf16_roundtrip_is_identity_on_all_finite_patterns():
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = O.bf16_decode(bits)
    finite = np.isfinite(vals)
    back = O.bf16_round(vals[finite])
    same = (back == bits[finite]) | ((vals[finite] == 0) & (back & 0x7FFF == 0))
    assert same.all()


def test_bf16_round_is_nearest():
    # bf16_round's definition: to float32 first, then to the nearest bf16 (ties to even) of that
    # float32 value, as the library stores a float32 result; the double rounding is not always
    # nearest to the float64 input itself, so the float32 value is the reference here
    g = np.random.default_rng(46)
    x = g.standard_normal(200000) * 10.0 ** g.integers(-3, 4, 200000)
    x32 = x.astype(np.float32).astype(np.float64)
    r = O.bf16_decode(O.bf16_round(x))
    ulp = 2.0 ** (np.floor(np.log2(np.abs(x32))) - 7)
    err = np.abs(r - x32)
    assert np.all(err <= 0.5 * ulp)
    tie = err == 0.5 * ulp   # exact midpoints go to the even bf16 (low mantissa bit 0)
    assert np.all((O.bf16_round(r[tie]) & 1) == 0)


# --------------------------------------------------------------------------- GELU

def test_gelu_matches_erf_form_within_tanh_approximation_error():
    u = np.linspace(-8, 8, 4001)
    ref = np.array([_gelu_erf(t) for t in u])
    # the tanh form approximates the erf form to about 2e-4 absolute everywhere
    assert np.max(np.abs(O.gelu_tanh(u) - ref)) < 5e-4


def test_gelu_closed_form_identities():
    u = np.linspace(-6, 6, 1201)
    g = O.gelu_tanh(u)
    assert O.gelu_tanh(np.array([0.0]))[0] == 0.0
    np.testing.assert_allclose(g - O.gelu_tanh(-u), u, atol=1e-12)  # tanh is odd
    big = np.array([12.0, 30.0])
    np.testing.assert_allclose(O.gelu_tanh(big), big, rtol=1e-12)
    assert np.all(np.abs(O.gelu_tanh(-big)) < 1e-12)
    eps = 1e-6
    slope0 = (O.gelu_tanh(np.array([eps]))[0] - O.gelu_tanh(np.array([-eps]))[0]) / (2 * eps)
    assert abs(slope0 - 0.5) < 1e-9


# --------------------------------------------------------------------------- selection

def test_ordered_key_is_monotone():
    vals = np.array([-np.inf, -3e38, -1.0, -1e-30, -1e-45, -0.0, 0.0, 1e-45, 1e-30, 1.0, 3e38, np.inf], dtype=np.float32)
    keys = O.ordered_key(vals).astype(np.int64)
    d = np.diff(keys)
    assert d[5] == 0  # -0 == +0
    assert np.all(np.delete(d, 5) > 0)


def _topk_by_counting(row, k):
    """Element i is kept iff fewer than k elements precede it in (value desc, index asc)."""
    n = len(row)
    keep = []
    for i in range(n):
        ahead = 0
        for j in range(n):
            if row[j] > row[i] or (row[j] == row[i] and j < i):
                ahead += 1
        if ahead < k:
            keep.append(i)
    return keep


@pytest.mark.parametrize("n,k", [(1, 0), (1, 1), (7, 3), (33, 5), (64, 64), (64, 0), (100, 37)])
def test_topk_against_counting_definition(n, k):
    for trial in range(4):
        row = rng.integers(-4, 5, n).astype(np.float32) * np.float32(0.5)  # heavy ties
        if trial % 2:
            row = rng.standard_normal(n).astype(np.float32)
        got = O.topk_cols(row[None, :], k)[0].tolist()
        assert got == _topk_by_counting(row.tolist(), k)


def test_topk_special_cases():
    n = 50
    eq = np.full((2, n), 0.25, dtype=np.float32)
    assert O.topk_cols(eq, 7)[0].tolist() == list(range(7))
    z = np.array([[0.0, -0.0, 0.0, -0.0, -1.0]], dtype=np.float32)
    assert O.topk_cols(z, 2)[0].tolist() == [0, 1]  # -0 ties +0, lower index wins
    r = rng.standard_normal((3, 40)).astype(np.float32)
    assert O.topk_cols(r, 40).tolist() == [list(range(40))] * 3
    assert O.topk_cols(r, 0).shape == (3, 0)
    out = O.topk_cols(r, 9)
    assert np.all(np.diff(out, axis=1) > 0)


def test_k_fixture_from_pages_sparsity():
    for ln in open(os.path.join(GOLDEN, "sparsity_k.txt")):
        if not ln.strip() or ln.startswith("#"):
            continue
        name, n, permille, k = ln.split()
        assert O.k_from_density(int(n), int(permille)) == int(k), name


# --------------------------------------------------------------------------- FP8

def test_e4m3_codes_fixture_and_roundtrip():
    rows = [ln.split() for ln in open(os.path.join(GOLDEN, "e4m3_codes.txt")) if ln.strip() and not ln.startswith("#")]
    for code, expr in rows:
        val = float(eval(expr))  # fixture holds plain arithmetic only
        got = O.e4m3_decode(np.array([int(code, 16)], dtype=np.uint8))[0]
        assert got == val and math.copysign(1.0, got) == math.copysign(1.0, val), (code, got, val)
        assert int(O.e4m3_encode(np.array([val], dtype=np.float32))[0]) == int(code, 16), code
    codes = np.arange(256, dtype=np.uint32).astype(np.uint8)
    vals = O.e4m3_decode(codes)
    nan = np.isnan(vals)
    assert sorted(codes[nan].tolist()) == [0x7F, 0xFF]
    np.testing.assert_array_equal(O.e4m3_encode(vals[~nan].astype(np.float32)), codes[~nan])


def test_e4m3_rounds_to_nearest_even_and_saturates():
    pos = np.arange(0, 0x7F, dtype=np.uint32).astype(np.uint8)   # 0 .. 448, increasing
    v = O.e4m3_decode(pos)
    assert np.all(np.diff(v) > 0)
    for lo in range(len(v) - 1):
        a, b = v[lo], v[lo + 1]
        mid = np.float32((a + b) / 2)                    # at most 5 significant bits: exact
        assert float(mid) == (a + b) / 2
        want = lo if lo % 2 == 0 else lo + 1              # the even code (lowest mantissa bit 0)
        assert int(O.e4m3_encode(np.array([mid]))[0]) == want, (a, b)
        assert int(O.e4m3_encode(np.array([np.nextafter(mid, np.float32(0))]))[0]) == lo
        assert int(O.e4m3_encode(np.array([np.nextafter(mid, np.float32(1e9))]))[0]) == lo + 1
        assert int(O.e4m3_encode(np.array([-mid]))[0]) == want | 0x80
    big = np.array([448.0, 449.0, 464.0, 1e6, np.inf], dtype=np.float32)
    assert O.e4m3_encode(big).tolist() == [0x7E] * 5
    assert O.e4m3_encode(-big).tolist() == [0xFE] * 5


def test_quantize_rows_e4m3():
    g = np.random.default_rng(21)
    x = (g.standard_normal((6, 96)) * 10.0 ** g.integers(-3, 3, (6, 1))).astype(np.float32)
    x[4] = 0.0
    x[5, :] = 1e-3
    x[5, 7] = -7.5                                       # one large value sets the row's scale
    codes, scales = O.quantize_rows_e4m3(x)
    assert codes.shape == x.shape and codes.dtype == np.uint8 and scales.dtype == np.float32
    for r in range(6):
        amax = np.float32(np.abs(x[r]).max())
        if amax == 0:
            assert scales[r] == 1.0 and not codes[r].any()
            continue
        assert scales[r] == amax / np.float32(448.0)
        j = int(np.abs(x[r]).argmax())
        assert codes[r, j] in (0x7E, 0xFE)               # the largest magnitude lands on +-448
        back = O.e4m3_decode(codes[r]) * float(scales[r])
        # within half an e4m3 step (2^-4 relative) of the value, or of the subnormal step for tiny ones
        bound = 2.0 ** -4 * np.abs(x[r]) + 2.0 ** -10 * float(scales[r]) + 1e-6 * float(amax)
        assert np.all(np.abs(back - x[r]) <= bound), r


def _fp8_case(T=20, D=32, H=50, k=12, Bt=8, seed=3):
    g = np.random.default_rng(seed)
    x8, sx = O.quantize_rows_e4m3(g.standard_normal((T, D)).astype(np.float32))
    w1t8, s1 = O.quantize_rows_e4m3((g.standard_normal((H, D)) / math.sqrt(D)).astype(np.float32))
    w2_8, s2 = O.quantize_rows_e4m3((g.standard_normal((H, D)) / math.sqrt(H)).astype(np.float32))
    b1 = 0.02 * g.standard_normal(H)
    A = O.bf16_decode(O.bf16_round(0.5 * g.standard_normal((T, H))))
    Y = g.standard_normal((T, D))
    nb = (T + Bt - 1) // Bt
    idx = np.sort(np.stack([g.choice(H, k, replace=False) for _ in range(nb)]), axis=1).astype(np.int32)
    s_delta = np.float32(1e-4)
    g2 = (s2 / s_delta).astype(np.float32)
    return dict(x8=x8, sx=sx, w1t8=w1t8, s1=s1, b1=b1, w2_8=w2_8, s2=s2, g2=g2, s_delta=s_delta, A=A, Y=Y, idx=idx,
                Bt=Bt, T=T, D=D, H=H)


def test_mlp_delta_fp8_written_out():
    c = _fp8_case()
    A1, Y1 = O.mlp_delta_fp8(c["x8"], c["sx"], c["w1t8"], c["s1"], c["b1"], c["w2_8"], c["g2"], c["s_delta"], c["idx"],
                             c["A"], c["Y"], c["Bt"])
    xd, w1d, w2d = O.e4m3_decode(c["x8"]), O.e4m3_decode(c["w1t8"]), O.e4m3_decode(c["w2_8"])
    for b, r0, r1 in [(0, 0, 8), (1, 8, 16), (2, 16, 20)]:
        for t in range(r0, r1):
            change = [0.0] * c["D"]
            for col in c["idx"][b]:
                dot = 0.0
                for d in range(c["D"]):
                    dot += xd[t, d] * w1d[col, d]
                u = dot * float(c["s1"][col]) * float(c["sx"][t]) + c["b1"][col]
                a = 0.5 * u * (1.0 + math.tanh(math.sqrt(2.0 / math.pi) * (u + 0.044715 * u ** 3)))
                assert abs(A1[t, col] - a) <= 1e-12 * max(1.0, abs(a))
                stored = O.bf16_decode(O.bf16_round(np.array([a])))[0]
                dlt = np.float32(stored - c["A"][t, col]) * np.float32(c["g2"][col])
                q = O.e4m3_decode(O.e4m3_encode(np.array([dlt], dtype=np.float32)))[0]
                for n in range(c["D"]):
                    change[n] += q * w2d[col, n]
            for n in range(c["D"]):
                assert abs(Y1[t, n] - (c["Y"][t, n] + float(c["s_delta"]) * change[n])) <= 1e-12 * max(1.0, abs(Y1[t, n]))
    sel = np.zeros((c["T"], c["H"]), dtype=bool)
    for b, r0, r1 in [(0, 0, 8), (1, 8, 16), (2, 16, 20)]:
        sel[r0:r1, c["idx"][b]] = True
    np.testing.assert_array_equal(A1[~sel], c["A"][~sel])


def test_mlp_delta_fp8_no_columns_and_the_unquantised_step():
    c = _fp8_case()
    none = np.zeros((3, 0), dtype=np.int32)
    A0, Y0 = O.mlp_delta_fp8(c["x8"], c["sx"], c["w1t8"], c["s1"], c["b1"], c["w2_8"], c["g2"], c["s_delta"], none,
                             c["A"], c["Y"], c["Bt"])
    np.testing.assert_array_equal(A0, c["A"])
    np.testing.assert_array_equal(Y0, c["Y"])
    # against the bf16-path step on the dequantised operands: the same activations, and outputs within
    # the rounding of the deltas to e4m3 (half a step, 2^-4 relative, per term)
    A1, Y1 = O.mlp_delta_fp8(c["x8"], c["sx"], c["w1t8"], c["s1"], c["b1"], c["w2_8"], c["g2"], c["s_delta"], c["idx"],
                             c["A"], c["Y"], c["Bt"])
    x = O.e4m3_decode(c["x8"]) * c["sx"].astype(np.float64)[:, None]
    W1 = (O.e4m3_decode(c["w1t8"]) * c["s1"].astype(np.float64)[:, None]).T
    W2 = O.e4m3_decode(c["w2_8"]) * c["s2"].astype(np.float64)[:, None]
    A2, Y2 = O.mlp_delta(x, W1, c["b1"], W2, c["idx"], c["A"], c["Y"], c["Bt"])
    np.testing.assert_allclose(A1, A2, rtol=1e-12, atol=1e-12)
    dY = np.abs((Y1 - c["Y"]) - (Y2 - c["Y"]))
    ref = np.abs(Y2 - c["Y"])
    assert dY.max() <= 0.1 * ref.max() and dY.max() > 0


# --------------------------------------------------------------------------- MLP

def _mlp_case(T=24, D=8, H=20, seed=0):
    g = np.random.default_rng(seed)
    x = g.standard_normal((T, D))
    W1 = g.standard_normal((D, H)) / math.sqrt(D)
    b1 = 0.02 * g.standard_normal(H)
    W2 = g.standard_normal((H, D)) / math.sqrt(H)
    b2 = 0.02 * g.standard_normal(D)
    return x, W1, b1, W2, b2


def test_dense_mlp_identity_weights_reduce_to_elementwise_gelu():
    x = rng.standard_normal((5, 6))
    I = np.eye(6)
    a, y = O.dense_mlp(x, I, np.zeros(6), I, np.zeros(6))
    ref = np.vectorize(_gelu_erf)(x)
    assert np.max(np.abs(y - ref)) < 5e-4
    np.testing.assert_array_equal(a, y)


def test_dense_mlp_permutation_and_bias_structure():
    x, W1, b1, W2, b2 = _mlp_case()
    _, y = O.dense_mlp(x, W1, b1, W2, b2)
    p = rng.permutation(W1.shape[1])
    _, yp = O.dense_mlp(x, W1[:, p], b1[p], W2[p, :], b2)
    np.testing.assert_allclose(yp, y, atol=1e-12)
    _, y0 = O.dense_mlp(x, W1, b1, W2, np.zeros_like(b2))
    np.testing.assert_allclose(y - y0, np.broadcast_to(b2, y.shape), atol=1e-12)
    # one hidden unit, written out per scalar
    c = 3
    _, y1 = O.dense_mlp(x, W1[:, [c]], b1[[c]], W2[[c], :], np.zeros_like(b2))
    for t in range(x.shape[0]):
        u = sum(x[t, d] * W1[d, c] for d in range(x.shape[1])) + b1[c]
        for n in range(W2.shape[1]):
            assert abs(y1[t, n] - _gelu_erf(u) * W2[c, n]) < 5e-4 * abs(W2[c, n]) + 1e-12


def _mlp_brute(x, W1, b1, W2, b2, cols=None):
    """gelu(x W1 + b1) W2 + b2 by plain loops, one term at a time (hidden units ``cols`` only, no
    b2, when given)."""
    T, D = x.shape
    H = W1.shape[1]
    cols = range(H) if cols is None else cols
    y = np.zeros((T, W2.shape[1]))
    a = {}
    for t in range(T):
        for c in cols:
            u = 0.0
            for d in range(D):
                u += x[t, d] * W1[d, c]
            u += b1[c]
            a[t, c] = 0.5 * u * (1.0 + math.tanh(math.sqrt(2.0 / math.pi) * (u + 0.044715 * u ** 3)))
        for n in range(W2.shape[1]):
            s = 0.0
            for c in cols:
                s += a[t, c] * W2[c, n]
            y[t, n] = s
    return a, y


def test_dense_mlp_brute_force_at_a_moderate_size():
    # 18 tokens, 40 features, 300 hidden units: more rows, features and hidden units than one
    # group of the C++ oracle's loops handles at a time (16 rows, 16 outputs, 128 terms)
    x, W1, b1, W2, b2 = _mlp_case(T=18, D=40, H=300, seed=7)
    a, y = O.dense_mlp(x, W1, b1, W2, b2)
    a_ref, y_ref = _mlp_brute(x, W1, b1, W2, b2)
    for (t, c), v in a_ref.items():
        assert abs(a[t, c] - v) <= 1e-13 * max(1.0, abs(v))
    np.testing.assert_allclose(y, y_ref + b2, rtol=0, atol=1e-12)


def test_mlp_delta_brute_force_at_a_moderate_size():
    # 150 selected columns of 300 in blocks of 8 of 18 tokens: the update is the old output plus,
    # per selected column, (new - old activation) times its W2 row, written out term by term
    x, W1, b1, W2, b2 = _mlp_case(T=18, D=40, H=300, seed=8)
    g = np.random.default_rng(13)
    A = g.standard_normal((18, 300))
    Y = g.standard_normal((18, 40))
    idx = np.sort(np.stack([g.choice(300, 150, replace=False) for _ in range(3)]), axis=1).astype(np.int32)
    A1, Y1 = O.mlp_delta(x, W1, b1, W2, idx, A, Y, Bt=8)
    for b, r0, r1 in [(0, 0, 8), (1, 8, 16), (2, 16, 18)]:
        a_new, _ = _mlp_brute(x[r0:r1], W1, b1, W2, b2, cols=idx[b].tolist())
        for t in range(r1 - r0):
            for n in range(40):
                s = 0.0
                for c in idx[b]:
                    s += (a_new[t, c] - A[r0 + t, c]) * W2[c, n]
                assert abs(Y1[r0 + t, n] - (Y[r0 + t, n] + s)) <= 1e-12
            for c in idx[b]:
                assert abs(A1[r0 + t, c] - a_new[t, c]) <= 1e-13 * max(1.0, abs(a_new[t, c]))
    sel = np.zeros((18, 300), dtype=bool)
    for b, r0, r1 in [(0, 0, 8), (1, 8, 16), (2, 16, 18)]:
        sel[r0:r1, idx[b]] = True
    np.testing.assert_array_equal(A1[~sel], A[~sel])


def _consistent_cache(x_prev, W1, b1, W2, b2):
    a, y = O.dense_mlp(x_prev, W1, b1, W2, b2)
    return a, y


def test_mlp_delta_all_columns_equals_dense_at_new_input():
    x, W1, b1, W2, b2 = _mlp_case()
    A, Y = _consistent_cache(x, W1, b1, W2, b2)
    x_t = x + 0.05 * rng.standard_normal(x.shape)
    H = W1.shape[1]
    idx = np.tile(np.arange(H, dtype=np.int32), (3, 1))
    A1, Y1 = O.mlp_delta(x_t, W1, b1, W2, idx, A, Y, Bt=8)
    a_ref, y_ref = O.dense_mlp(x_t, W1, b1, W2, b2)
    np.testing.assert_allclose(Y1, y_ref, atol=1e-12)
    np.testing.assert_allclose(A1, a_ref, atol=1e-12)


def test_mlp_delta_no_columns_keeps_cache():
    x, W1, b1, W2, b2 = _mlp_case()
    A = rng.standard_normal((24, 20))
    Y = rng.standard_normal((24, 8))
    idx = np.zeros((3, 0), dtype=np.int32)
    A1, Y1 = O.mlp_delta(x, W1, b1, W2, idx, A, Y, Bt=8)
    np.testing.assert_array_equal(A1, A)
    np.testing.assert_array_equal(Y1, Y)


def test_mlp_delta_keeps_cache_invariant_and_unselected_columns():
    x, W1, b1, W2, b2 = _mlp_case(T=30)  # 30 rows, Bt=8 -> short last block
    A, Y = _consistent_cache(x, W1, b1, W2, b2)
    for step in range(4):
        x = x + 0.05 * rng.standard_normal(x.shape)
        idx = np.sort(np.stack([rng.choice(20, 6, replace=False) for _ in range(4)]), axis=1).astype(np.int32)
        A1, Y1 = O.mlp_delta(x, W1, b1, W2, idx, A, Y, Bt=8)
        np.testing.assert_allclose(Y1, A1 @ W2 + b2, atol=1e-12)
        for b, r0, r1 in O.blocks(30, 8):
            un = np.setdiff1d(np.arange(20), idx[b])
            np.testing.assert_array_equal(A1[r0:r1][:, un], A[r0:r1][:, un])
        A, Y = A1, Y1


def test_mlp_delta_single_column_written_out():
    x, W1, b1, W2, b2 = _mlp_case(T=8)
    A = rng.standard_normal((8, 20))
    Y = rng.standard_normal((8, 8))
    c = 11
    A1, Y1 = O.mlp_delta(x, W1, b1, W2, np.array([[c]], dtype=np.int32), A, Y, Bt=8)
    for t in range(8):
        u = sum(x[t, d] * W1[d, c] for d in range(8)) + b1[c]
        a = O.gelu_tanh(np.array([u]))[0]
        assert abs(a - _gelu_erf(u)) < 5e-4
        for n in range(8):
            assert abs(Y1[t, n] - (Y[t, n] + (a - A[t, c]) * W2[c, n])) < 1e-12
        assert abs(A1[t, c] - a) < 1e-12


def test_mlp_scores_written_out():
    a = rng.standard_normal((10, 5))
    A = rng.standard_normal((10, 5))
    s = O.mlp_scores(a, A, Bt=4, first_step=False)
    s0 = O.mlp_scores(a, A, Bt=4, first_step=True)
    assert s.shape == (3, 5)
    for b, r0, r1 in [(0, 0, 4), (1, 4, 8), (2, 8, 10)]:
        for c in range(5):
            assert abs(s[b, c] - sum(abs(a[r, c] - A[r, c]) for r in range(r0, r1))) < 1e-12
            assert abs(s0[b, c] - sum(abs(a[r, c]) for r in range(r0, r1))) < 1e-12


def test_mlp_refresh_selects_top_scores_and_rebuilds_cache():
    x, W1, b1, W2, b2 = _mlp_case(T=16)
    A_old = rng.standard_normal((16, 20))
    r = O.mlp_refresh(x, W1, b1, W2, b2, A_old, Bt=8, k=5, first_step=False)
    np.testing.assert_allclose(r["y"], r["a"] @ W2 + b2, atol=1e-12)
    for b in range(2):
        sel = set(r["idx"][b].tolist())
        s = r["scores"][b]
        assert min(s[list(sel)]) >= max(s[[c for c in range(20) if c not in sel]])


def test_mlp_refresh_first_step_scores_ignore_the_cache():
    # a first step has no cache: the score of a column is the sum over the
    # block's rows of |a|, written out term by term, whatever A_old holds
    x, W1, b1, W2, b2 = _mlp_case(T=16)
    r0 = O.mlp_refresh(x, W1, b1, W2, b2, np.zeros((16, 20)), Bt=8, k=5, first_step=True)
    r1 = O.mlp_refresh(x, W1, b1, W2, b2, rng.standard_normal((16, 20)), Bt=8, k=5, first_step=True)
    for r in (r0, r1):
        for b in range(2):
            for c in range(20):
                want = 0.0
                for row in range(8 * b, 8 * b + 8):
                    want += abs(r["a"][row, c])
                assert abs(r["scores"][b, c] - want) <= 1e-12 * max(1.0, want)
    np.testing.assert_array_equal(r0["idx"], r1["idx"])


# --------------------------------------------------------------------------- attention

def _softmax_attention_brute(q, k, v, scale, keys=None):
    """Normalised softmax attention of each query row, summed term by term."""
    n, d = q.shape
    keys = range(k.shape[0]) if keys is None else keys
    out = np.zeros((n, d))
    for i in range(n):
        w = [math.exp(scale * sum(q[i, t] * k[j, t] for t in range(d))) for j in keys]
        tot = sum(w)
        for jj, j in enumerate(keys):
            out[i] += (w[jj] / tot) * v[j]
    return out


def _attn_case(h=2, T=20, d=4, seed=3):
    g = np.random.default_rng(seed)
    return g.standard_normal((h, T, d)), g.standard_normal((h, T, d)), g.standard_normal((h, T, d))


def test_dense_attention_brute_force_and_lse():
    q, k, v = _attn_case()
    scale = 0.5
    Od, lse = O.dense_attention(q, k, v, scale)
    for hh in range(2):
        np.testing.assert_allclose(Od[hh], _softmax_attention_brute(q[hh], k[hh], v[hh], scale), atol=1e-12)
        for i in range(20):
            tot = sum(math.exp(scale * float(q[hh, i] @ k[hh, j])) for j in range(20))
            assert abs(lse[hh, i] - math.log(tot)) < 1e-12


def test_attention_zero_scale_is_mean_of_values():
    q, k, v = _attn_case()
    Od, _ = O.dense_attention(q, k, v, 0.0)
    for hh in range(2):
        np.testing.assert_allclose(Od[hh], np.broadcast_to(v[hh].mean(axis=0), (20, 4)), atol=1e-13)


def _random_idx(h, nb, T, kk, seed=5):
    g = np.random.default_rng(seed)
    return np.sort(np.stack([[g.choice(T, kk, replace=False) for _ in range(nb)] for _ in range(h)]), axis=2).astype(np.int32)


def test_attn_delta_fresh_cache_equals_dense():
    q, k, v = _attn_case(T=22)
    scale, Bt = 0.4, 8
    idx = _random_idx(2, 3, 22, 5)
    m_c, l_c, acc_c = O.complement_partial(q, k, v, idx, scale, Bt)
    out = O.attn_delta(q, k, v, idx, m_c, l_c, acc_c, scale, Bt)
    for hh in range(2):
        np.testing.assert_allclose(out[hh], _softmax_attention_brute(q[hh], k[hh], v[hh], scale), atol=1e-12)


def test_attn_delta_all_keys_ignores_cache_and_no_keys_returns_cache():
    q, k, v = _attn_case(T=16)
    scale, Bt = 0.3, 8
    g = np.random.default_rng(9)
    m_c = g.standard_normal((2, 16))
    l_c = 1.0 + g.random((2, 16))
    acc_c = g.standard_normal((2, 16, 4))
    allk = np.tile(np.arange(16, dtype=np.int32), (2, 2, 1))
    # empty complement: m = -inf, l = 0, acc = 0
    out = O.attn_delta(q, k, v, allk, np.full((2, 16), -np.inf), np.zeros((2, 16)), np.zeros((2, 16, 4)), scale, Bt)
    for hh in range(2):
        np.testing.assert_allclose(out[hh], _softmax_attention_brute(q[hh], k[hh], v[hh], scale), atol=1e-12)
    none = np.zeros((2, 2, 0), dtype=np.int32)
    out0 = O.attn_delta(q, k, v, none, m_c, l_c, acc_c, scale, Bt)
    np.testing.assert_allclose(out0, acc_c / l_c[:, :, None], atol=1e-14)
    one = np.full((2, 2, 1), 7, dtype=np.int32)
    out1 = O.attn_delta(q, k, v, one, np.full((2, 16), -np.inf), np.zeros((2, 16)), np.zeros((2, 16, 4)), scale, Bt)
    np.testing.assert_allclose(out1, np.broadcast_to(v[:, 7:8, :], (2, 16, 4)), atol=1e-14)


def _compact_brute(q, k, v, idx, scale, Bt):
    """lse and normalised output over each row's complementary keys, summed term by term."""
    h, T, d = q.shape
    lse = np.full((h, T), -np.inf)
    oc = np.zeros((h, T, d))
    for hh in range(h):
        for i in range(T):
            sel = set(int(j) for j in idx[hh][i // Bt])
            ws = [(math.exp(scale * float(q[hh, i] @ k[hh, j])), j) for j in range(T) if j not in sel]
            if ws:
                tot = math.fsum(w for w, _ in ws)
                lse[hh, i] = math.log(tot)
                oc[hh, i] = sum(w * v[hh, j] for w, j in ws) / tot
    return lse, oc


def test_compact_cache_matches_its_definition_and_gives_dense():
    q, k, v = _attn_case(T=22)
    scale, Bt = 0.4, 8
    idx = _random_idx(2, 3, 22, 5)
    lse_b, oc_b = _compact_brute(q, k, v, idx, scale, Bt)
    lse, oc = O.compact_partial(*O.complement_partial(q, k, v, idx, scale, Bt))
    np.testing.assert_allclose(lse, lse_b, atol=1e-12)
    np.testing.assert_allclose(oc, oc_b, atol=1e-12)
    out = O.attn_delta_compact(q, k, v, idx, lse_b, oc_b, scale, Bt)
    for hh in range(2):
        np.testing.assert_allclose(out[hh], _softmax_attention_brute(q[hh], k[hh], v[hh], scale), atol=1e-12)


def test_compact_cache_empty_sides():
    q, k, v = _attn_case(T=16)
    scale, Bt = 0.3, 8
    g = np.random.default_rng(12)
    lse_c = g.standard_normal((2, 16))
    o_c = g.standard_normal((2, 16, 4))
    allk = np.tile(np.arange(16, dtype=np.int32), (2, 2, 1))
    out = O.attn_delta_compact(q, k, v, allk, np.full((2, 16), -np.inf), np.zeros((2, 16, 4)), scale, Bt)
    for hh in range(2):
        np.testing.assert_allclose(out[hh], _softmax_attention_brute(q[hh], k[hh], v[hh], scale), atol=1e-12)
    none = np.zeros((2, 2, 0), dtype=np.int32)
    np.testing.assert_allclose(O.attn_delta_compact(q, k, v, none, lse_c, o_c, scale, Bt), o_c, atol=1e-14)
    lse0, o0 = O.compact_partial(np.full(3, -np.inf), np.zeros(3), np.zeros((3, 4)))
    assert np.all(lse0 == -np.inf) and np.all(o0 == 0)


def test_merge_is_associative_and_split_invariant():
    g = np.random.default_rng(11)
    q = g.standard_normal((6, 4))
    k = g.standard_normal((30, 4)) * 3
    v = g.standard_normal((30, 4))
    parts = [O.attn_partial(q, k[s], v[s], 0.7) for s in (slice(0, 9), slice(9, 21), slice(21, 30))]
    left = O.merge_partials(O.merge_partials(parts[0], parts[1]), parts[2])
    right = O.merge_partials(parts[0], O.merge_partials(parts[1], parts[2]))
    whole = O.attn_partial(q, k, v, 0.7)
    for a, b in ((left, right), (left, whole)):
        np.testing.assert_allclose(O.finish(a), O.finish(b), atol=1e-13)
        np.testing.assert_allclose(a[1] * np.exp(a[0] - b[0]), b[1], rtol=1e-12)


def test_attn_mass_sums_and_uniform_case():
    q, k, v = _attn_case(T=20)
    mass = O.attn_mass(q, k, 0.5, Bt=8)
    assert mass.shape == (2, 3, 20)
    np.testing.assert_allclose(mass.sum(axis=2), np.broadcast_to([8, 8, 4], (2, 3)), atol=1e-12)
    flat = O.attn_mass(np.zeros_like(q), k, 0.5, Bt=8)
    np.testing.assert_allclose(flat[:, 2, :], 4 / 20, atol=1e-14)
    # one block, brute force
    for j in range(20):
        tot = 0.0
        for i in range(8, 16):
            w = [math.exp(0.5 * float(q[1, i] @ k[1, jj])) for jj in range(20)]
            tot += w[j] / sum(w)
        assert abs(mass[1, 1, j] - tot) < 1e-12


def test_attn_refresh_complement_and_selection():
    q, k, v = _attn_case(T=24)
    r = O.attn_refresh(q, k, v, 0.5, Bt=8, kk=6)
    # complement merged with the selected keys at the same q, k, v is the dense output
    out = O.attn_delta(q, k, v, r["idx"], r["m_c"], r["l_c"], r["acc_c"], 0.5, 8)
    np.testing.assert_allclose(out, r["O"], atol=1e-12)
    for hh in range(2):
        for b in range(3):
            sel = set(r["idx"][hh, b].tolist())
            m = r["mass"][hh, b]
            assert min(m[list(sel)]) >= max(m[[j for j in range(24) if j not in sel]])
            rows = range(8 * b, 8 * b + 8)
            keys = [j for j in range(24) if j not in sel]
            brute = _softmax_attention_brute(q[hh, list(rows)], k[hh], v[hh], 0.5, keys=keys)
            np.testing.assert_allclose(r["acc_c"][hh, 8 * b:8 * b + 8] / r["l_c"][hh, 8 * b:8 * b + 8, None], brute, atol=1e-12)


# --------------------------------------------------------------------------- input generator

def test_generator_draws_at_counters_match_the_stream():
    from dynamic_column_sparse_b200 import synth
    full = synth.normal_bf16(9, 5, (40, 24), std=0.5)
    rows = np.array([0, 7, 39])
    np.testing.assert_array_equal(synth.rows_bf16(9, 5, 24, rows, std=0.5), full[rows])
    drifted = synth.drift_bf16(full, 10, 6, 0.03)
    np.testing.assert_array_equal(synth.drift_rows_bf16(full[rows], 10, 6, 24, rows, 0.03), drifted[rows])
    z = synth.normal_f64(3, 4, 1 << 21)
    assert abs(z.mean()) < 3e-3 and abs(z.std() - 1.0) < 3e-3
