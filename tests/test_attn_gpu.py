"""Sparse attention delta step on the GPU against the fp64 oracle."""
import math

import numpy as np
import pytest

import oracle as O
from cases import attn_case
from helpers import assert_parity, dev_bf16, dev_f32, dev_i32, f64_of_bf16, heads_first

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cm():
    from dynamic_column_sparse_b200 import chipmunk
    chipmunk.load_library()
    return chipmunk


def run_gpu(cm, c, idx, m_c=None, l_c=None, acc_c=None):
    import torch
    L = c["L"]
    T, h = c["T"], c["h"]
    o = torch.empty((T, h, 128), dtype=torch.bfloat16, device="cuda")
    cm.attn_delta(dev_bf16(L["q"]), dev_bf16(L["k"]), dev_bf16(L["v"]), dev_i32(idx),
                  dev_f32(c["m_c"] if m_c is None else m_c), dev_f32(c["l_c"] if l_c is None else l_c),
                  dev_f32(c["acc_c"] if acc_c is None else acc_c), o, scale=c["scale"])
    torch.cuda.synchronize()
    assert cm.read_device_status() == 0
    return heads_first(f64_of_bf16(o))


def oracle_delta(c, idx, m_c=None, l_c=None, acc_c=None):
    f = lambda a, d: (c[d] if a is None else a).astype(np.float64)
    return O.attn_delta(c["q"], c["k"], c["v"], idx, f(m_c, "m_c"), f(l_c, "l_c"), f(acc_c, "acc_c"), c["scale"], 128)


@pytest.mark.parametrize("T,h,permille", [
    (300, 2, 165),    # ragged query block (300 = 2*128 + 44), one key chunk
    (700, 3, 400),    # three key chunks, ragged last chunk
    (1000, 1, 70),
])
def test_attn_delta_small(cm, T, h, permille):
    c = attn_case(1, T, h, permille, 0.03)
    assert_parity(run_gpu(cm, c, c["idx"]), oracle_delta(c, c["idx"]), "o", bf16_out=True)


def test_attn_delta_flux_shape(cm):
    c = attn_case(0, 4352, 24, 165, 0.03)
    assert c["kk"] == 718
    assert_parity(run_gpu(cm, c, c["idx"]), oracle_delta(c, c["idx"]), "o", bf16_out=True)


def test_attn_delta_no_keys_returns_cached_output(cm):
    c = attn_case(1, 300, 2, 165, 0.03)
    idx = np.zeros((2, 3, 0), dtype=np.int32)
    got = run_gpu(cm, c, idx)
    assert_parity(got, c["acc_c"].astype(np.float64) / c["l_c"].astype(np.float64)[:, :, None], "o = acc_c / l_c", bf16_out=True)


def test_attn_delta_all_keys_empty_complement_is_dense(cm):
    c = attn_case(2, 300, 2, 1000, 0.03)
    idx = np.tile(np.arange(300, dtype=np.int32), (2, 3, 1))
    m_c = np.full((2, 300), -np.inf, dtype=np.float32)
    l_c = np.zeros((2, 300), dtype=np.float32)
    acc_c = np.zeros((2, 300, 128), dtype=np.float32)
    got = run_gpu(cm, c, idx, m_c, l_c, acc_c)
    dense, _ = O.dense_attention(c["q"], c["k"], c["v"], c["scale"])
    assert_parity(got, dense, "o vs dense attention", bf16_out=True)


def test_attn_delta_fresh_cache_is_dense(cm):
    """Complement cached at the same q, k, v: the merge is the dense softmax."""
    c = attn_case(3, 700, 2, 300, 0.0)
    got = run_gpu(cm, c, c["idx"])
    dense, _ = O.dense_attention(c["q"], c["k"], c["v"], c["scale"])
    assert_parity(got, dense, "o vs dense attention", bf16_out=True)


# --------------------------------------------------------------- compact complement cache

def compact_of(c):
    """The case's complement partial in compact form, at storage precision (lse fp32, o_c bf16 bits)."""
    lse, oc = O.compact_partial(c["m_c"].astype(np.float64), c["l_c"].astype(np.float64), c["acc_c"].astype(np.float64))
    return O.f32(lse), O.bf16_round(oc)


def run_gpu_compact(cm, c, idx, lse32, oc_bits):
    import torch
    T, h, L = c["T"], c["h"], c["L"]
    o = torch.empty((T, h, 128), dtype=torch.bfloat16, device="cuda")
    cm.attn_delta_compact(dev_bf16(L["q"]), dev_bf16(L["k"]), dev_bf16(L["v"]), dev_i32(idx), dev_f32(lse32),
                          dev_bf16(oc_bits), o, scale=c["scale"])
    torch.cuda.synchronize()
    assert cm.read_device_status() == 0
    return heads_first(f64_of_bf16(o))


@pytest.mark.parametrize("seed,T,h,permille", [
    (1, 300, 2, 165),
    (1, 700, 3, 400),
    (0, 4352, 24, 165),   # FLUX layer
])
def test_attn_delta_compact_cache(cm, seed, T, h, permille):
    c = attn_case(seed, T, h, permille, 0.03)
    lse32, oc_bits = compact_of(c)
    got = run_gpu_compact(cm, c, c["idx"], lse32, oc_bits)
    ref = O.attn_delta_compact(c["q"], c["k"], c["v"], c["idx"], lse32.astype(np.float64), O.bf16_decode(oc_bits),
                               c["scale"], 128)
    assert_parity(got, ref, "o (compact cache)", bf16_out=True)


def test_attn_delta_compact_cache_empty_sides(cm):
    c = attn_case(1, 300, 2, 165, 0.03)
    lse32, oc_bits = compact_of(c)
    none = np.zeros((2, 3, 0), dtype=np.int32)
    assert_parity(run_gpu_compact(cm, c, none, lse32, oc_bits), O.bf16_decode(oc_bits), "o = o_c", bf16_out=True)
    allk = np.tile(np.arange(300, dtype=np.int32), (2, 3, 1))
    empty_lse = np.full((2, 300), -np.inf, dtype=np.float32)
    zeros = np.zeros((2, 300, 128), dtype=np.uint16)
    dense, _ = O.dense_attention(c["q"], c["k"], c["v"], c["scale"])
    assert_parity(run_gpu_compact(cm, c, allk, empty_lse, zeros), dense, "o vs dense attention", bf16_out=True)
