"""Mistakes planted in the oracle must be caught by its pins.

Both oracles are mutated, one plausible error at a time (a dropped term, a
wrong sign or index, a transposed reduction, a wrong tie rule, a missing
scale):

* the numpy oracle, by replacing one of its functions with a copy carrying
  the error;
* the C++ oracle, by rebuilding it from a copy of its source in which one
  snippet is replaced (each snippet must occur exactly once).

The pin suite in test_oracle_pins.py is then run against the mutated oracle;
at least one pin must fail. The unmutated oracles must pass every pin.
Everything runs on the CPU.
"""
import concurrent.futures as cf
import inspect
import math
import os

import numpy as np
import pytest

import oracle.chipmunk_oracle as OC
import test_oracle_pins as pins
from oracle import cpp

ORIG = {name: getattr(OC, name) for name in ("mlp_delta", "attn_partial")}


def _all_pins():
    calls = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        marks = getattr(fn, "pytestmark", [])
        params = [m for m in marks if m.name == "parametrize"]
        if params:
            argnames = [a.strip() for a in params[0].args[0].split(",")]
            for values in params[0].args[1]:
                calls.append((name, fn, dict(zip(argnames, values))))
        else:
            calls.append((name, fn, {}))
    return calls


def _failed_pins(monkeypatch, impl):
    monkeypatch.setattr(pins, "O", impl)
    failed = []
    for name, fn, kwargs in _all_pins():
        try:
            fn(**kwargs)
        except (AssertionError, ValueError, IndexError):
            failed.append(name)
    return failed


def _caught(monkeypatch, fname, mutant):
    monkeypatch.setattr(OC, fname, mutant)
    return _failed_pins(monkeypatch, OC)


def _gelu_no_cubic(u):
    u = np.asarray(u, dtype=np.float64)
    return 0.5 * u * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * u))


def _gelu_sign(u):
    u = np.asarray(u, dtype=np.float64)
    return 0.5 * u * (1.0 - np.tanh(math.sqrt(2.0 / math.pi) * (u + 0.044715 * u ** 3)))


def _mlp_delta_sign(x, W1, b1, W2, idx, A_cache, Y_cache, Bt):
    A_new, Y_new = np.array(A_cache, dtype=float), np.array(Y_cache, dtype=float)
    for b, r0, r1 in OC.blocks(x.shape[0], Bt):
        S = np.asarray(idx[b], dtype=np.int64)
        if S.size:
            a = OC.gelu_tanh(x[r0:r1] @ W1[:, S] + b1[S])
            Y_new[r0:r1] += (A_cache[r0:r1][:, S] - a) @ W2[S, :]
            A_new[r0:r1, S] = a
    return A_new, Y_new


def _mlp_delta_no_bias(x, W1, b1, W2, idx, A_cache, Y_cache, Bt):
    return ORIG["mlp_delta"](x, W1, np.zeros_like(b1), W2, idx, A_cache, Y_cache, Bt)


def _mlp_delta_stale_cache(x, W1, b1, W2, idx, A_cache, Y_cache, Bt):
    _, Y_new = ORIG["mlp_delta"](x, W1, b1, W2, idx, A_cache, Y_cache, Bt)
    return np.array(A_cache, dtype=float), Y_new


def _topk_high_ties(scores32, k):
    scores32 = np.atleast_2d(np.asarray(scores32, dtype=np.float32))
    keys = OC.ordered_key(scores32).astype(np.int64)
    out = np.empty((scores32.shape[0], k), dtype=np.int32)
    for r in range(scores32.shape[0]):
        n = scores32.shape[1]
        order = n - 1 - np.argsort(-keys[r][::-1], kind="stable")
        out[r] = np.sort(order[:k])
    return out


def _topk_unsorted(scores32, k):
    scores32 = np.atleast_2d(np.asarray(scores32, dtype=np.float32))
    keys = OC.ordered_key(scores32).astype(np.int64)
    out = np.empty((scores32.shape[0], k), dtype=np.int32)
    for r in range(scores32.shape[0]):
        out[r] = np.argsort(-keys[r], kind="stable")[:k]
    return out


def _key_no_neg_zero(s32):
    bits = np.ascontiguousarray(s32, dtype=np.float32).view(np.uint32).copy()
    neg = (bits & np.uint32(0x80000000)) != 0
    return np.where(neg, ~bits, bits | np.uint32(0x80000000)).astype(np.uint32)


def _merge_wrong_weight(p1, p2):
    m1, l1, a1 = p1
    m2, l2, a2 = p2
    M = np.maximum(m1, m2)
    with np.errstate(invalid="ignore", over="ignore"):
        w1 = np.where(m1 == -np.inf, 0.0, np.exp(M - m1))
        w2 = np.where(m2 == -np.inf, 0.0, np.exp(M - m2))
    return M, l1 * w1 + l2 * w2, a1 * w1[:, None] + a2 * w2[:, None]


def _partial_no_scale(q, k, v, scale):
    return ORIG["attn_partial"](q, k, v, 1.0)


def _mass_wrong_axis(q, k, scale, Bt):
    h, T, d = q.shape
    nb = (T + Bt - 1) // Bt
    out = np.zeros((h, nb, T))
    for hh in range(h):
        for b, r0, r1 in OC.blocks(T, Bt):
            s = scale * (q[hh, r0:r1] @ k[hh].T)
            p = np.exp(s - s.max(axis=0, keepdims=True))
            p /= p.sum(axis=0, keepdims=True)
            out[hh, b] = p.sum(axis=0)
    return out


def _complement_keeps_selected(q, k, v, idx, scale, Bt):
    h, T, d = q.shape
    m_c, l_c, acc_c = np.full((h, T), -np.inf), np.zeros((h, T)), np.zeros((h, T, d))
    for hh in range(h):
        for b, r0, r1 in OC.blocks(T, Bt):
            m_c[hh, r0:r1], l_c[hh, r0:r1], acc_c[hh, r0:r1] = OC.attn_partial(q[hh, r0:r1], k[hh], v[hh], scale)
    return m_c, l_c, acc_c


def _scores_no_abs(a, A_cache, Bt, first_step):
    T, H = a.shape
    out = np.zeros(((T + Bt - 1) // Bt, H))
    for b, r0, r1 in OC.blocks(T, Bt):
        d = a[r0:r1] if first_step else a[r0:r1] - A_cache[r0:r1]
        out[b] = d.sum(axis=0)
    return out


def _bf16_truncate(x):
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def _compact_no_log(m, l, acc):
    l = np.asarray(l, dtype=np.float64)
    safe = np.where(l > 0, l, 1.0)
    o = np.where((l > 0)[..., None], np.asarray(acc, dtype=np.float64) / safe[..., None], 0.0)
    return np.where(l > 0, np.asarray(m, dtype=np.float64) + l, -np.inf), o


def _delta_compact_unweighted(q, k, v, idx, lse_c, o_c, scale, Bt):
    h, T, d = q.shape
    out = np.zeros((h, T, d))
    for hh in range(h):
        for b, r0, r1 in OC.blocks(T, Bt):
            S = np.asarray(idx[hh][b], dtype=np.int64)
            sel = OC.attn_partial(q[hh, r0:r1], k[hh, S], v[hh, S], scale)
            cached = (np.zeros(r1 - r0), np.ones(r1 - r0), o_c[hh, r0:r1])  # lse dropped from the weight
            out[hh, r0:r1] = OC.finish(OC.merge_partials(cached, sel))
    return out


def _k_round_up(n, density_permille):
    return -((-int(n) * int(density_permille)) // 1000)


def _dense_mlp_no_b2(x, W1, b1, W2, b2):
    a = OC.gelu_tanh(x @ W1 + b1[None, :])
    return a, a @ W2


def _finish_unnormalised(p):
    m, l, acc = p
    return np.asarray(acc, dtype=np.float64)


def _attn_delta_ignores_cache(q, k, v, idx, m_c, l_c, acc_c, scale, Bt):
    h, T, d = q.shape
    out = np.zeros((h, T, d))
    for hh in range(h):
        for b, r0, r1 in OC.blocks(T, Bt):
            S = np.asarray(idx[hh][b], dtype=np.int64)
            out[hh, r0:r1] = OC.finish(OC.attn_partial(q[hh, r0:r1], k[hh, S], v[hh, S], scale))
    return out


def _dense_attention_lse_without_max(q, k, v, scale):
    h, T, d = q.shape
    O = np.zeros((h, T, d))
    lse = np.zeros((h, T))
    for hh in range(h):
        m, l, acc = OC.attn_partial(q[hh], k[hh], v[hh], scale)
        O[hh] = acc / l[:, None]
        lse[hh] = np.log(l)
    return O, lse


def _mass_rows_no_scale(q_rows, k, scale):
    s = q_rows @ k.T
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    return p.sum(axis=0)


def _mlp_refresh_ignores_first_step(x, W1, b1, W2, b2, A_old, Bt, k, first_step):
    a, y = OC.dense_mlp(x, W1, b1, W2, b2)
    scores = OC.mlp_scores(a, A_old if A_old is not None else np.zeros_like(a), Bt, False)
    return dict(a=a, y=y, scores=scores, idx=OC.topk_cols(OC.f32(scores), k))


def _attn_refresh_smallest_mass(q, k, v, scale, Bt, kk):
    O, lse = OC.dense_attention(q, k, v, scale)
    mass = OC.attn_mass(q, k, scale, Bt)
    h, nb, T = mass.shape
    idx = OC.topk_cols(OC.f32(-mass.reshape(h * nb, T)), kk).reshape(h, nb, kk)
    m_c, l_c, acc_c = OC.complement_partial(q, k, v, idx, scale, Bt)
    return dict(O=O, lse=lse, mass=mass, idx=idx, m_c=m_c, l_c=l_c, acc_c=acc_c)


def _blocks_drop_short_tail(T, Bt):
    return [(b, b * Bt, (b + 1) * Bt) for b in range(T // Bt)]


def _bf16_decode_low_half(bits):
    with np.errstate(invalid="ignore"):
        return (np.asarray(bits, dtype=np.uint32) << np.uint32(15)).view(np.float32).astype(np.float64)


def _e4m3_truncate(x32):
    x = np.asarray(x32, dtype=np.float32)
    out = ORIG_E4M3(x)
    back = OC.e4m3_decode(out)
    over = np.abs(back) > np.abs(x.astype(np.float64))      # rounded away from zero: step back one code
    return np.where(over & (out & 0x7F > 0), out - 1, out).astype(np.uint8)


def _e4m3_no_saturation(x32):
    x = np.asarray(x32, dtype=np.float32)
    out = ORIG_E4M3(x)
    return np.where(np.abs(x) > 448.0, np.uint8(0x7F), out).astype(np.uint8)


def _quantize_scale_off_by_one_code(x):
    codes, scales = ORIG_QUANT(x)
    return codes, (scales * np.float32(1.0625)).astype(np.float32)


def _fp8_no_delta_scale(x8, sx, w1t8, s1, b1, w2_8, g2, s_delta, idx, A_cache, Y_cache, Bt):
    return ORIG_FP8(x8, sx, w1t8, s1, b1, w2_8, g2, np.float32(1.0), idx, A_cache, Y_cache, Bt)


def _fp8_no_g2(x8, sx, w1t8, s1, b1, w2_8, g2, s_delta, idx, A_cache, Y_cache, Bt):
    return ORIG_FP8(x8, sx, w1t8, s1, b1, w2_8, np.ones_like(np.asarray(g2)), s_delta, idx, A_cache, Y_cache, Bt)


def _fp8_no_s1(x8, sx, w1t8, s1, b1, w2_8, g2, s_delta, idx, A_cache, Y_cache, Bt):
    return ORIG_FP8(x8, sx, w1t8, np.ones_like(np.asarray(s1)), b1, w2_8, g2, s_delta, idx, A_cache, Y_cache, Bt)


ORIG_E4M3 = OC.e4m3_encode
ORIG_QUANT = OC.quantize_rows_e4m3
ORIG_FP8 = OC.mlp_delta_fp8

MUTATIONS = {
    "e4m3_encode: truncation instead of nearest-even": ("e4m3_encode", _e4m3_truncate),
    "e4m3_encode: no saturation at 448": ("e4m3_encode", _e4m3_no_saturation),
    "quantize_rows_e4m3: scale off": ("quantize_rows_e4m3", _quantize_scale_off_by_one_code),
    "mlp_delta_fp8: delta scale dropped": ("mlp_delta_fp8", _fp8_no_delta_scale),
    "mlp_delta_fp8: g2 not applied": ("mlp_delta_fp8", _fp8_no_g2),
    "mlp_delta_fp8: W1 row scale dropped": ("mlp_delta_fp8", _fp8_no_s1),
    "gelu_tanh: cubic term dropped": ("gelu_tanh", _gelu_no_cubic),
    "gelu_tanh: sign of tanh flipped": ("gelu_tanh", _gelu_sign),
    "mlp_delta: delta sign flipped": ("mlp_delta", _mlp_delta_sign),
    "mlp_delta: bias b1 dropped": ("mlp_delta", _mlp_delta_no_bias),
    "mlp_delta: cache not written back": ("mlp_delta", _mlp_delta_stale_cache),
    "topk_cols: ties to the higher index": ("topk_cols", _topk_high_ties),
    "topk_cols: indices not ascending": ("topk_cols", _topk_unsorted),
    "ordered_key: -0 not equal to +0": ("ordered_key", _key_no_neg_zero),
    "merge_partials: weights inverted": ("merge_partials", _merge_wrong_weight),
    "attn_partial: logit scale dropped": ("attn_partial", _partial_no_scale),
    "attn_mass: softmax over the wrong axis": ("attn_mass", _mass_wrong_axis),
    "complement_partial: selected keys kept": ("complement_partial", _complement_keeps_selected),
    "mlp_scores: absolute value dropped": ("mlp_scores", _scores_no_abs),
    "bf16_round: truncation instead of nearest-even": ("bf16_round", _bf16_truncate),
    "compact_partial: log of l dropped": ("compact_partial", _compact_no_log),
    "attn_delta_compact: cached weight e^lse dropped": ("attn_delta_compact", _delta_compact_unweighted),
    "k_from_density: rounded up": ("k_from_density", _k_round_up),
    "dense_mlp: bias b2 dropped": ("dense_mlp", _dense_mlp_no_b2),
    "finish: not divided by l": ("finish", _finish_unnormalised),
    "attn_delta: cached complement ignored": ("attn_delta", _attn_delta_ignores_cache),
    "dense_attention: lse without the row maximum": ("dense_attention", _dense_attention_lse_without_max),
    "attn_mass_rows: logit scale dropped": ("attn_mass_rows", _mass_rows_no_scale),
    "mlp_refresh: first-step rule ignored": ("mlp_refresh", _mlp_refresh_ignores_first_step),
    "attn_refresh: smallest mass selected": ("attn_refresh", _attn_refresh_smallest_mass),
    "blocks: short last block dropped": ("blocks", _blocks_drop_short_tail),
    "bf16_decode: bits shifted by 15": ("bf16_decode", _bf16_decode_low_half),
}


@pytest.mark.parametrize("what", sorted(MUTATIONS))
def test_planted_mistake_is_caught(monkeypatch, what):
    fname, mutant = MUTATIONS[what]
    failed = _caught(monkeypatch, fname, mutant)
    assert failed, f"no pin caught: {what}"


def test_unmutated_oracle_passes_every_pin(monkeypatch):
    assert _caught(monkeypatch, "gelu_tanh", OC.gelu_tanh) == []


# --------------------------------------------------------------------------- C++ oracle

CPP_MUTATIONS = {
    "gelu: cubic term dropped": ("(u + 0.044715 * u * u * u)", "(u)"),
    "gelu: sign of tanh flipped": ("0.5 * u * (1.0 + std::tanh(", "0.5 * u * (1.0 - std::tanh("),
    "mlp_delta: delta sign flipped": ("delta[r * k + j] = an - A_cache[(r0 + r) * H + c];",
                                      "delta[r * k + j] = A_cache[(r0 + r) * H + c] - an;"),
    "preactivation: bias b1 dropped": ("u[r] = acc[r] + b1[c];", "u[r] = acc[r];"),
    "preactivation: first input feature skipped": ("  for (int64_t d = 0; d < D; ++d) {\n    const double *xd",
                                                   "  for (int64_t d = 1; d < D; ++d) {\n    const double *xd"),
    "mlp_delta: cache not written back": ("delta[r * k + j] = an - A_cache[(r0 + r) * H + c];\n          A_new[(r0 + r) * H + c] = an;",
                                          "delta[r * k + j] = an - A_cache[(r0 + r) * H + c];"),
    "weighted_row_sums: last term of every chunk dropped": ("const int64_t j1 = std::min(j0 + kTerms, ncoef);",
                                                            "const int64_t j1 = std::min(j0 + kTerms - 1, ncoef);"),
    "weighted_row_sums: ragged output tail skipped": ("for (int64_t e = 0; e < nn; ++e) o[e] += coef[r * ldc + j] * rows[j][n0 + e];",
                                                      "(void)nn;"),
    "topk: ties to the higher index": ("[&](int64_t a, int64_t b) { return key[a] > key[b]; }",
                                       "[&](int64_t a, int64_t b) { return key[a] != key[b] ? key[a] > key[b] : a > b; }"),
    "topk: indices not ascending": ("std::sort(order.begin(), order.begin() + k);", ""),
    "ordered_key: -0 not equal to +0": ("if (b == 0x80000000u) b = 0u;", ""),
    "merge: weights inverted": ("const double w1 = (m1 == kNegInf) ? 0.0 : std::exp(m1 - mm);\n  const double w2 = (m2 == kNegInf) ? 0.0 : std::exp(m2 - mm);",
                                "const double w1 = (m1 == kNegInf) ? 0.0 : std::exp(mm - m1);\n  const double w2 = (m2 == kNegInf) ? 0.0 : std::exp(mm - m2);"),
    "partial: logit scale dropped": ("      s[j] *= scale;\n      mx = std::max(mx, s[j]);\n    }\n    double l = 0.0;\n    for (int64_t j = 0; j < m; ++j) {",
                                     "      s[j] *= 1.0;\n      mx = std::max(mx, s[j]);\n    }\n    double l = 0.0;\n    for (int64_t j = 0; j < m; ++j) {"),
    "mass: probabilities not normalised": ("out[j] += s[j] / l;", "out[j] += s[j];"),
    "mass: logit scale dropped": ("      s[j] *= scale;\n      mx = std::max(mx, s[j]);\n    }\n    double l = 0.0;\n    for (int64_t j = 0; j < T; ++j) {",
                                  "      s[j] *= 1.0;\n      mx = std::max(mx, s[j]);\n    }\n    double l = 0.0;\n    for (int64_t j = 0; j < T; ++j) {"),
    "complement: selected keys kept": ("if (!selected[j]) keys.push_back(j);", "keys.push_back(j);"),
    "mlp_scores: absolute value dropped": ("s += std::fabs(first_step ? a[r * H + c] : a[r * H + c] - A_cache[r * H + c]);",
                                           "s += (first_step ? a[r * H + c] : a[r * H + c] - A_cache[r * H + c]);"),
    "bf16_round: truncation instead of nearest-even": ("(static_cast<uint64_t>(u) + 0x7FFFu + lsb) >> 16",
                                                       "(static_cast<uint64_t>(u) + 0u * lsb) >> 16"),
    "compact_partial: log of l dropped": ("lse[i] = l[i] > 0 ? m[i] + std::log(l[i]) : kNegInf;",
                                          "lse[i] = l[i] > 0 ? m[i] + l[i] : kNegInf;"),
    "attn_delta_compact: cached weight e^lse dropped": ("merge_row(lse_c[row], 1.0,", "merge_row(0.0, 1.0,"),
    "k_from_density: rounded up": ("return (n * permille) / 1000;", "return (n * permille + 999) / 1000;"),
    "dense_mlp: bias b2 dropped": ("for (int64_t n = 0; n < D; ++n) y[r * D + n] += b2[n];", "(void)b2;"),
    "finish: not divided by l": ("out[e] = l > 0 ? acc[e] / l : 0.0;", "out[e] = l > 0 ? acc[e] : 0.0;"),
    "attn_delta: cached complement ignored": ("merge_row(m_c[row], l_c[row], acc_c + row * d,",
                                              "merge_row(kNegInf, 0.0, acc_c + row * d,"),
    "dense_attention: lse without the row maximum": ("lse[row] = m[i] + std::log(l[i]);", "lse[row] = std::log(l[i]);"),
    "mlp_refresh: first-step rule ignored": ("or_mlp_scores(a, A_old, T, H, Bt, first_step, scores);",
                                             "or_mlp_scores(a, A_old, T, H, Bt, 0, scores);"),
    "attn_refresh: smallest mass selected": ("m32[i] = static_cast<float>(mass[i]);",
                                             "m32[i] = static_cast<float>(-mass[i]);"),
    "blocks: short last block dropped": ("int64_t block_count(int64_t T, int64_t Bt) { return (T + Bt - 1) / Bt; }",
                                         "int64_t block_count(int64_t T, int64_t Bt) { return T / Bt; }"),
    "bf16_decode: bits shifted by 15": ("static_cast<uint32_t>(bits) << 16;", "static_cast<uint32_t>(bits) << 15;"),
    "e4m3: subnormals truncated": ("const double m = std::nearbyint(a * 512.0);", "const double m = std::floor(a * 512.0);"),
    "e4m3: normals truncated": ("double r = std::nearbyint(std::ldexp(a, 3 - e));", "double r = std::floor(std::ldexp(a, 3 - e));"),
    "e4m3: exponent bias 8": ("return sign | static_cast<uint8_t>((be << 3) | m);", "return sign | static_cast<uint8_t>(((be + 1) << 3) | m);"),
    "e4m3 decode: subnormal scale 2^-7": ("if (be == 0) return sign * std::ldexp(m / 8.0, -6);", "if (be == 0) return sign * std::ldexp(m / 8.0, -7);"),
    "quantize_rows: inverse scale 1/448": ("const float inv = amax > 0.f ? 448.f / amax : 1.f;", "const float inv = amax > 0.f ? 1.f / amax : 1.f;"),
    "mlp_delta_fp8: delta from the unrounded activation": ("const double stored = bf16_to_double(double_to_bf16(an));", "const double stored = an;"),
    "mlp_delta_fp8: delta scale dropped": ("yr[n] += static_cast<double>(s_delta) * change[r * D + n];", "yr[n] += change[r * D + n];"),
    "mlp_delta_fp8: token scale dropped": ("const double an = gelu(u[r] * s1[c] * sx[r0 + r] + b1[c]);", "const double an = gelu(u[r] * s1[c] + b1[c]);"),
}


@pytest.fixture(scope="module")
def cpp_mutants(tmp_path_factory):
    """Every C++ mutant, built once (in parallel) into its own shared library."""
    src = open(cpp.SRC).read()
    out_dir = tmp_path_factory.mktemp("oracle_mutants")
    jobs = {}
    for i, (what, (old, new)) in enumerate(sorted(CPP_MUTATIONS.items())):
        assert src.count(old) == 1, f"{what}: the snippet must occur exactly once in the source"
        path = os.path.join(out_dir, f"m{i}.cpp")
        with open(path, "w") as f:
            f.write(src.replace(old, new))
        jobs[what] = path
    with cf.ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
        futs = {what: ex.submit(cpp.compile_source, p, p[:-4] + ".so") for what, p in jobs.items()}
        return {what: f.result() for what, f in futs.items()}


@pytest.mark.parametrize("what", sorted(CPP_MUTATIONS))
def test_planted_mistake_in_cpp_oracle_is_caught(monkeypatch, cpp_mutants, what):
    failed = _failed_pins(monkeypatch, cpp.CppOracle(cpp_mutants[what]))
    assert failed, f"no pin caught: {what}"


def test_unmutated_cpp_oracle_passes_every_pin(monkeypatch):
    assert _failed_pins(monkeypatch, cpp.CppOracle(cpp.build())) == []
