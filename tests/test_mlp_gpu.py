"""Sparse MLP delta step on the GPU against the fp64 oracle."""
import numpy as np
import pytest

import oracle as O
from cases import mlp_case
from helpers import (assert_bf16_storage, assert_parity, bits_of, dev_bf16, dev_f32, dev_i32, f64_of, f64_of_bf16, to_block_major,
                     to_token_major)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cm():
    from dynamic_column_sparse_b200 import chipmunk
    chipmunk.load_library()
    return chipmunk


def run_gpu(cm, c, idx, x_bits=None):
    import torch
    L = c["L"]
    Bt = c["Bt"]
    x = dev_bf16(L["x_t"] if x_bits is None else x_bits)
    a_cache = dev_bf16(to_block_major(c["A_bits"], Bt))
    y_cache = dev_f32(c["Y32"])
    out = torch.empty((c["T"], c["D"]), dtype=torch.bfloat16, device="cuda")
    cm.mlp_delta(x, dev_bf16(L["w1t"]), dev_bf16(L["b1"]), dev_bf16(L["w2"]), dev_i32(idx), a_cache, y_cache, out,
                 Bt=Bt)
    torch.cuda.synchronize()
    assert cm.read_device_status() == 0
    return a_cache, y_cache, out


def check_step(cm, c, idx):
    a_cache, y_cache, out = run_gpu(cm, c, idx)
    A_new, Y_new = O.mlp_delta(c["x_t"], c["W1"], c["b1"], c["W2"], idx, c["A64"], c["Y32"].astype(np.float64),
                               c["Bt"])
    assert_parity(f64_of_bf16(out), Y_new, "out", bf16_out=True)
    assert_parity(f64_of(y_cache), Y_new, "y_cache")
    got_A = to_token_major(bits_of(a_cache), c["T"])
    for b, r0, r1 in O.blocks(c["T"], c["Bt"]):
        sel = idx[b]
        un = np.setdiff1d(np.arange(c["H"]), sel)
        np.testing.assert_array_equal(got_A[r0:r1][:, un], c["A_bits"][r0:r1][:, un])
    sel_mask = np.zeros((c["T"], c["H"]), dtype=bool)
    for b, r0, r1 in O.blocks(c["T"], c["Bt"]):
        sel_mask[r0:r1, idx[b]] = True
    assert_bf16_storage(O.bf16_decode(got_A)[sel_mask], A_new[sel_mask], "a_cache (selected)")
    return out


@pytest.mark.parametrize("T,D,H,Bt,permille,sigma", [
    (256, 128, 512, 64, 250, 0.05),     # tiny config
    (300, 192, 700, 128, 430, 0.03),    # ragged block, ragged column chunk, D not a multiple of 128
    (200, 384, 1000, 64, 333, 0.03),    # Bt = 64 with a short last block
])
def test_mlp_delta_small(cm, T, D, H, Bt, permille, sigma):
    c = mlp_case(1, T, D, H, Bt, permille, sigma)
    check_step(cm, c, c["idx"])


def test_mlp_delta_flux_shape(cm):
    c = mlp_case(0, 4352, 3072, 12288, 128, 300, 0.03)
    assert c["k"] == 3686
    check_step(cm, c, c["idx"])


def test_mlp_delta_no_columns_keeps_cache(cm):
    c = mlp_case(1, 300, 192, 700, 128, 430, 0.03)
    nb = (300 + 127) // 128
    idx = np.zeros((nb, 0), dtype=np.int32)
    a_cache, y_cache, out = run_gpu(cm, c, idx)
    np.testing.assert_array_equal(to_token_major(bits_of(a_cache), 300), c["A_bits"])
    np.testing.assert_array_equal(f64_of(y_cache), c["Y32"].astype(np.float64))
    np.testing.assert_array_equal(bits_of(out), O.bf16_round(c["Y32"].astype(np.float64)))


def test_mlp_delta_all_columns_is_dense(cm):
    c = mlp_case(2, 256, 128, 512, 128, 1000, 0.05)
    idx = np.tile(np.arange(512, dtype=np.int32), (2, 1))
    out = check_step(cm, c, idx)
    assert_parity(f64_of_bf16(out), c["y_t"], "out vs dense at x_t", bf16_out=True)
