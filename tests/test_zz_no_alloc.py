"""chipmunk_mlp_delta_noalloc through the C ABI, against the fp64 oracle and
against chipmunk_mlp_delta.

The no-alloc entry point serves callers that cannot allocate device memory
(a host that owns all device memory and hands plugins no allocator, or a loop
where a cudaMalloc would synchronise the device): it takes its scratch from a
fixed array inside the library. Here both entry points run the same two
sparse steps in a row on separate copies of the same layer state. After each
call the no-alloc results must agree with the oracle's step (whose caches are
kept at the library's storage precision between the calls: activation cache
bf16, output cache fp32) within the parity tolerance, and with the workspace
entry point's results. The file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest

import oracle as O
from cases import mlp_case
from helpers import assert_bf16_storage, assert_parity, bits_of, dev_bf16, dev_f32, dev_i32, f64_of, f64_of_bf16
from helpers import to_block_major, to_token_major

pytestmark = pytest.mark.gpu


def _state(c):
    import torch
    return dict(a_cache=dev_bf16(to_block_major(c["A_bits"], c["Bt"])), y_cache=dev_f32(c["Y32"]),
                out=torch.empty((c["T"], c["D"]), dtype=torch.bfloat16, device="cuda"))


def _args(cm, c, x, st, idx, w):
    return cm.MlpArgs(c["T"], c["D"], c["H"], c["Bt"], idx.shape[1], x.data_ptr(), w["w1t"].data_ptr(),
                      w["b1"].data_ptr(), w["w2"].data_ptr(), 0, idx.data_ptr(), st["a_cache"].data_ptr(),
                      st["y_cache"].data_ptr(), st["out"].data_ptr())


def test_noalloc_matches_oracle_and_workspace_entry_point_on_two_calls():
    import torch
    from dynamic_column_sparse_b200 import chipmunk as cm
    lib = cm.load_library()
    c = mlp_case(4, 640, 256, 1536, 128, 300, 0.03)
    L = c["L"]
    w = {n: dev_bf16(L[n]) for n in ("w1t", "b1", "w2")}
    x_bits = [L["x_t"], L["x_prev"]]
    idx_np = c["idx"]
    idx = dev_i32(idx_np)
    ref, new = _state(c), _state(c)
    # the oracle's own chain, kept at storage precision between the calls
    A_o, Y_o = c["A64"], c["Y32"].astype(np.float64)
    sel = np.zeros((c["T"], c["H"]), dtype=bool)
    for b, r0, r1 in O.blocks(c["T"], c["Bt"]):
        sel[r0:r1, idx_np[b]] = True
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, xb in enumerate(x_bits):
        x = dev_bf16(xb)
        a_ref = _args(cm, c, x, ref, idx, w)
        need = lib.chipmunk_workspace_bytes(cm.OP_MLP_DELTA, ctypes.byref(a_ref))
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        assert lib.chipmunk_mlp_delta(ctypes.byref(a_ref), ctypes.c_void_p(ws.data_ptr()), need, stream) == 0
        a_new = _args(cm, c, x, new, idx, w)
        st = lib.chipmunk_mlp_delta_noalloc(ctypes.byref(a_new), stream)
        assert st == 0, lib.chipmunk_last_error()
        torch.cuda.synchronize()
        assert cm.read_device_status() == 0
        tag = f"call {call + 1}"
        # against the oracle
        A_new, Y_new = O.mlp_delta(O.bf16_decode(xb), c["W1"], c["b1"], c["W2"], idx_np, A_o, Y_o, c["Bt"])
        assert_parity(f64_of_bf16(new["out"]), Y_new, f"out vs oracle, {tag}", bf16_out=True)
        assert_parity(f64_of(new["y_cache"]), Y_new, f"y_cache vs oracle, {tag}")
        got_A = O.bf16_decode(to_token_major(bits_of(new["a_cache"]), c["T"]))
        assert_bf16_storage(got_A[sel], A_new[sel], f"a_cache (selected) vs oracle, {tag}")
        np.testing.assert_array_equal(got_A[~sel], O.bf16_decode(c["A_bits"])[~sel])
        A_o, Y_o = O.bf16_decode(O.bf16_round(A_new)), O.f32(Y_new).astype(np.float64)
        # against the workspace entry point
        assert_parity(f64_of_bf16(new["out"]), f64_of_bf16(ref["out"]), f"out vs workspace call, {tag}", bf16_out=True)
        assert_parity(f64_of(new["y_cache"]), f64_of(ref["y_cache"]), f"y_cache vs workspace call, {tag}")
        assert_bf16_storage(O.bf16_decode(bits_of(new["a_cache"])), O.bf16_decode(bits_of(ref["a_cache"])),
                            f"a_cache vs workspace call, {tag}")
    # the second call really changed the state
    assert not np.array_equal(bits_of(new["out"]), O.bf16_round(c["Y32"].astype(np.float64)))
