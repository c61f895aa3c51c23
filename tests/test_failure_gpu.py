"""Failure detection on the GPU without a fault: a bounded wait that runs out.

A diagnostic kernel waits on a barrier nothing signals. The wait gives up
after about 2 s and records a timeout in the device status word; the host
reads it, the word is cleared, and the context keeps working. While the word
is set, later kernels return at entry without touching their outputs.
"""
import ctypes

import numpy as np
import pytest

import oracle as O
from dynamic_column_sparse_b200 import synth
from helpers import dev_f32

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    import torch
    from dynamic_column_sparse_b200 import chipmunk as cm
    lib = cm.load_library()
    assert cm.read_device_status() == 0
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.chipmunk_selftest_bounded_wait(stream) == 0
    # with the word set, a kernel returns at entry: the output keeps its fill
    s = synth.score_rows(1, 4, 512)
    out = torch.full((4, 16), -7, dtype=torch.int32, device="cuda")
    cm.topk_cols(dev_f32(s), 16, out=out)
    torch.cuda.synchronize()
    assert cm.read_device_status() == 1          # CHIPMUNK_DEV_WAIT_TIMEOUT, now cleared
    assert int(out.min()) == -7 and int(out.max()) == -7
    assert cm.read_device_status() == 0
    # the context is intact: the same call now runs and matches the oracle
    cm.topk_cols(dev_f32(s), 16, out=out)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out.cpu().numpy(), O.topk_cols(s, 16))
    assert cm.read_device_status() == 0
