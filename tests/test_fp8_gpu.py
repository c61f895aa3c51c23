"""FP8 form of the sparse MLP step on the GPU against the oracle.

The operands are e4m3 codes with one scale per row (tokens of x, hidden units
of W1^T and W2), produced by the oracle's quantiser from the layer's bf16
values, so both sides start from the same codes. The GPU quantiser itself is
checked bit for bit against the oracle's on the same bf16 rows. The oracle
models every rounding of the FP8 step (the e4m3 codes of the deltas included);
the float results must meet the usual bar. How far the FP8 step's output moves
from the bf16 step's (the method's precision change, not a parity error) is
printed for information.
"""
import numpy as np
import pytest

import oracle as O
from cases import mlp_case
from dynamic_column_sparse_b200 import synth
from helpers import (assert_bf16_storage, assert_parity, bits_of, dev_bf16, dev_f32, dev_i32, err_stats, f64_of,
                     f64_of_bf16, to_block_major, to_token_major)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cm():
    from dynamic_column_sparse_b200 import chipmunk
    chipmunk.load_library()
    return chipmunk


def dev_u8(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def test_quantize_e4m3_rows_bit_exact(cm):
    rows = [synth.normal_bf16(31, 1, (40, 3072)), synth.normal_bf16(31, 2, (8, 256), std=1e-3)]
    odd = synth.normal_bf16(31, 3, (4, 256), std=0.02)
    odd[0] = 0                                                     # all-zero row
    odd[1, 5] = O.bf16_round(np.array([3.0e4]))[0]                 # one huge value: the rest fall to subnormal codes
    odd[2, ::3] = O.bf16_round(np.array([-2.5]))[0]                # ties in magnitude
    rows.append(odd)
    for bits in rows:
        codes, scales = cm.quantize_e4m3_rows(dev_bf16(bits))
        ref_codes, ref_scales = O.quantize_rows_e4m3(O.bf16_decode(bits).astype(np.float32))
        np.testing.assert_array_equal(codes.cpu().numpy(), ref_codes)
        np.testing.assert_array_equal(scales.cpu().numpy(), ref_scales)


def fp8_case(c):
    """The layer's operands as e4m3 codes and scales (the oracle's quantiser), and a delta scale
    that leaves the largest delta of the step a little inside the e4m3 range."""
    f32 = lambda bits: O.bf16_decode(bits).astype(np.float32)
    L = c["L"]
    x8, sx = O.quantize_rows_e4m3(f32(L["x_t"]))
    w1t8, s1 = O.quantize_rows_e4m3(f32(L["w1t"]))
    w2_8, s2 = O.quantize_rows_e4m3(f32(L["w2"]))
    A_new, _ = O.mlp_delta(c["x_t"], c["W1"], c["b1"], c["W2"], c["idx"], c["A64"], c["Y32"].astype(np.float64), c["Bt"])
    big = max(float(np.abs((A_new - c["A64"]) * s2.astype(np.float64)[None, :]).max()), 1e-30)
    s_delta = np.float32(big / 400.0)
    g2 = (s2 / s_delta).astype(np.float32)
    return dict(x8=x8, sx=sx, w1t8=w1t8, s1=s1, w2_8=w2_8, s2=s2, g2=g2, s_delta=s_delta)


def run_fp8(cm, c, q, idx):
    import torch
    a_cache = dev_bf16(to_block_major(c["A_bits"], c["Bt"]))
    y_cache = dev_f32(c["Y32"])
    out = torch.empty((c["T"], c["D"]), dtype=torch.bfloat16, device="cuda")
    cm.mlp_delta_fp8(dev_u8(q["x8"]), dev_f32(q["sx"]), dev_u8(q["w1t8"]), dev_f32(q["s1"]), dev_bf16(c["L"]["b1"]),
                     dev_u8(q["w2_8"]), dev_f32(q["g2"]), q["s_delta"], dev_i32(idx), a_cache, y_cache, out)
    torch.cuda.synchronize()
    assert cm.read_device_status() == 0
    return a_cache, y_cache, out


@pytest.mark.parametrize("T,D,H,permille", [
    (300, 256, 700, 430),        # ragged last block, ragged column chunk
    (4352, 3072, 12288, 300),    # FLUX.1-dev layer, 70% sparse
])
def test_mlp_delta_fp8_matches_oracle(cm, T, D, H, permille):
    c = mlp_case(9, T, D, H, 128, permille, 0.03)
    q = fp8_case(c)
    a_cache, y_cache, out = run_fp8(cm, c, q, c["idx"])
    A_ref, Y_ref = O.mlp_delta_fp8(q["x8"], q["sx"], q["w1t8"], q["s1"], c["b1"], q["w2_8"], q["g2"], q["s_delta"],
                                   c["idx"], c["A64"], c["Y32"].astype(np.float64), c["Bt"])
    r = assert_parity(f64_of_bf16(out), Y_ref, "out", bf16_out=True)
    assert_parity(f64_of(y_cache), Y_ref, "y_cache")
    got_A = to_token_major(bits_of(a_cache), T)
    sel = np.zeros((T, H), dtype=bool)
    for b, r0, r1 in O.blocks(T, c["Bt"]):
        sel[r0:r1, c["idx"][b]] = True
    assert_bf16_storage(O.bf16_decode(got_A)[sel], A_ref[sel], "a_cache (selected)")
    np.testing.assert_array_equal(got_A[~sel], c["A_bits"][~sel])
    _, Y_bf16 = O.mlp_delta(c["x_t"], c["W1"], c["b1"], c["W2"], c["idx"], c["A64"], c["Y32"].astype(np.float64),
                            c["Bt"])
    mx, rms, _ = err_stats(Y_ref, Y_bf16)
    print(f"FP8 step T={T}: max|err|/rms vs the FP8 oracle {r[0]:.4f}; the FP8 step's own distance from the "
          f"bf16 step {mx / rms:.4f} of RMS")


def test_mlp_delta_fp8_no_columns_keeps_cache(cm):
    c = mlp_case(9, 300, 256, 700, 128, 430, 0.03)
    q = fp8_case(c)
    idx = np.zeros((3, 0), dtype=np.int32)
    a_cache, y_cache, out = run_fp8(cm, c, q, idx)
    np.testing.assert_array_equal(to_token_major(bits_of(a_cache), 300), c["A_bits"])
    np.testing.assert_array_equal(f64_of(y_cache), c["Y32"].astype(np.float64))
    np.testing.assert_array_equal(bits_of(out), O.bf16_round(c["Y32"].astype(np.float64)))
