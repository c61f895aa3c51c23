"""chipmunk_mlp_delta_noalloc against chipmunk_mlp_delta, through the C ABI.

The no-alloc entry point serves callers that cannot allocate device memory
(a host that owns all device memory and hands plugins no allocator, or a loop
where a cudaMalloc would synchronise the device): it takes its scratch from a
fixed array inside the library. Here both entry points run the same two
sparse steps in a row on separate copies of the same layer state, and their
outputs and caches must agree within the parity tolerance after each call.
The file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest

import oracle as O
from cases import mlp_case
from helpers import assert_bf16_storage, assert_parity, bits_of, dev_bf16, dev_f32, dev_i32, f64_of, f64_of_bf16
from helpers import to_block_major

pytestmark = pytest.mark.gpu


def _state(c):
    import torch
    return dict(a_cache=dev_bf16(to_block_major(c["A_bits"], c["Bt"])), y_cache=dev_f32(c["Y32"]),
                out=torch.empty((c["T"], c["D"]), dtype=torch.bfloat16, device="cuda"))


def _args(cm, c, x, st, idx, w):
    return cm.MlpArgs(c["T"], c["D"], c["H"], c["Bt"], idx.shape[1], x.data_ptr(), w["w1t"].data_ptr(),
                      w["b1"].data_ptr(), w["w2"].data_ptr(), 0, idx.data_ptr(), st["a_cache"].data_ptr(),
                      st["y_cache"].data_ptr(), st["out"].data_ptr())


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    import torch
    from dynamic_column_sparse_b200 import chipmunk as cm
    lib = cm.load_library()
    c = mlp_case(4, 640, 256, 1536, 128, 300, 0.03)
    L = c["L"]
    w = {n: dev_bf16(L[n]) for n in ("w1t", "b1", "w2")}
    xs = [dev_bf16(L["x_t"]), dev_bf16(L["x_prev"])]
    idx = dev_i32(c["idx"])
    ref, new = _state(c), _state(c)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, x in enumerate(xs):
        a_ref = _args(cm, c, x, ref, idx, w)
        need = lib.chipmunk_workspace_bytes(cm.OP_MLP_DELTA, ctypes.byref(a_ref))
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        assert lib.chipmunk_mlp_delta(ctypes.byref(a_ref), ctypes.c_void_p(ws.data_ptr()), need, stream) == 0
        a_new = _args(cm, c, x, new, idx, w)
        st = lib.chipmunk_mlp_delta_noalloc(ctypes.byref(a_new), stream)
        assert st == 0, lib.chipmunk_last_error()
        torch.cuda.synchronize()
        assert cm.read_device_status() == 0
        assert_parity(f64_of_bf16(new["out"]), f64_of_bf16(ref["out"]), f"out, call {call + 1}", bf16_out=True)
        assert_parity(f64_of(new["y_cache"]), f64_of(ref["y_cache"]), f"y_cache, call {call + 1}")
        assert_bf16_storage(O.bf16_decode(bits_of(new["a_cache"])), O.bf16_decode(bits_of(ref["a_cache"])),
                            f"a_cache, call {call + 1}")
    # the second call really changed the state
    assert not np.array_equal(bits_of(new["out"]), O.bf16_round(c["Y32"].astype(np.float64)))


def test_noalloc_rejects_requests_beyond_its_scratch():
    from dynamic_column_sparse_b200 import chipmunk as cm
    lib = cm.load_library()
    # nb * round_up(k,128) * Bt * 2 = 600 * 1024 * 128 * 2 bytes > 64 MiB
    a = cm.MlpArgs(T=600 * 128, D=128, H=1024, Bt=128, k=1024, x=0x1000, w1t=0x2000, b1=0x3000, w2=0x4000,
                   b2=0, idx=0x5000, a_cache=0x6000, y_cache=0x7000, out=0)
    assert lib.chipmunk_mlp_delta_noalloc(ctypes.byref(a), None) == 7
    assert b"no-alloc" in lib.chipmunk_last_error() or b"scratch" in lib.chipmunk_last_error()
