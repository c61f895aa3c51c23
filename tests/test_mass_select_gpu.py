"""The attention refresh's fused scoring: the mass of each (head, query block) row and its top-k
taken inside one kernel, on the GPU.

The mass is compared with the oracle in tests/test_refresh_gpu.py and tests/test_workloads_gpu.py.
Here the in-kernel selection is checked on the cases that steer it down each of its paths: the exact
top-k of the kernel's own fp32 mass rows (a property check against the kept mass), rows where every
mass ties (all keys alike: the closed form is keys 0 .. k-1), rows whose k-th mass is far below the
histogram's range (a sharp softmax: many masses underflow to 0), rows too long for the candidate
buffer, rows whose length is not a multiple of 4, k = T, and many tiles per CTA, where the mass row
buffer is reused from tile to tile; and the refresh without a mass tensor (rows kept only in the
kernel's row buffers) gives the same selection, output and cache as the refresh with one.
"""
import math

import numpy as np
import pytest

import oracle as O
from dynamic_column_sparse_b200 import synth
from helpers import assert_is_topk_of, dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cm():
    from dynamic_column_sparse_b200 import chipmunk
    chipmunk.load_library()
    return chipmunk


def refresh(cm, q, k, v, kk, scale, keep_mass):
    import torch
    T, h = q.shape[0], q.shape[1]
    nb = (T + 127) // 128
    idx = torch.full((h, nb, kk), -1, dtype=torch.int32, device="cuda")
    m_c = torch.empty((h, T), dtype=torch.float32, device="cuda")
    l_c = torch.empty((h, T), dtype=torch.float32, device="cuda")
    acc_c = torch.empty((h, T, 128), dtype=torch.float32, device="cuda")
    o = torch.empty((T, h, 128), dtype=torch.bfloat16, device="cuda")
    mass = torch.full((h, nb, T), float("nan"), dtype=torch.float32, device="cuda") if keep_mass else None
    cm.attn_refresh(q, k, v, idx, m_c, l_c, acc_c, o, mass, scale=scale)
    torch.cuda.synchronize()
    assert cm.read_device_status() == 0
    return dict(idx=idx, m_c=m_c, l_c=l_c, acc_c=acc_c, o=o, mass=mass)


def inputs(T, h, seed=6):
    L = synth.attn_layer(seed, T, h, 128, 0.03)
    return dev_bf16(L["q"]), dev_bf16(L["k"]), dev_bf16(L["v"])


def check_both_forms(cm, q, k, v, kk, scale, what):
    """The kept-mass refresh selects the exact top-k of its own mass; the refresh without a mass
    tensor gives the same results. Returns the kept-mass run."""
    import torch
    T, h = q.shape[0], q.shape[1]
    nb = (T + 127) // 128
    a = refresh(cm, q, k, v, kk, scale, True)
    assert_is_topk_of(a["idx"].cpu().numpy().reshape(h * nb, kk), a["mass"].cpu().numpy().reshape(h * nb, T), what)
    b = refresh(cm, q, k, v, kk, scale, False)
    for key in ("idx", "o", "m_c", "l_c", "acc_c"):
        assert torch.equal(a[key], b[key]), f"{what}: {key} differs without a mass tensor"
    return a


@pytest.mark.parametrize("T,h,permille", [
    (301, 2, 300),      # rows not a multiple of 4: unaligned kept rows, a ragged last chunk
    (4352, 24, 165),    # the FLUX layer: 816 tiles, about 5.5 per CTA (the row buffer is reused)
    (12032, 3, 165),    # FLUX 2304x1280 rows: longer than the candidate buffer
])
def test_selection_is_exact_on_the_kernels_own_mass(cm, T, h, permille):
    q, k, v = inputs(T, h)
    check_both_forms(cm, q, k, v, O.k_from_density(T, permille), 1.0 / math.sqrt(128), f"T={T}")


@pytest.mark.parametrize("T", [4352, 12000])
def test_all_masses_tie(cm, T):
    """q = 0: every query attends uniformly, so every key of a block has the same mass (the block's
    query count / T) and the selection is keys 0 .. k-1. At T = 12000 every key is a candidate and
    the candidates overflow the buffer: the selection runs over the whole row."""
    import torch
    h = 2
    q, k, v = inputs(T, h)
    q = torch.zeros_like(q)
    kk = O.k_from_density(T, 165)
    r = check_both_forms(cm, q, k, v, kk, 1.0 / math.sqrt(128), f"ties, T={T}")
    nb = (T + 127) // 128
    want = np.broadcast_to(np.arange(kk, dtype=np.int32), (h, nb, kk))
    np.testing.assert_array_equal(r["idx"].cpu().numpy(), want)
    mass = r["mass"].cpu().numpy()
    for b in range(nb):
        n = min(128, T - 128 * b)
        np.testing.assert_allclose(mass[:, b], n / T, rtol=2e-5)


def test_sharp_softmax_many_zero_masses(cm):
    """A large logit scale: most keys get a mass that underflows to 0 (below the histogram's range),
    so the k-th mass sits in its lowest bin and ties at 0 go to the lower index."""
    T, h = 4352, 4
    q, k, v = inputs(T, h, seed=9)
    kk = O.k_from_density(T, 300)
    r = check_both_forms(cm, q, k, v, kk, 16.0, "sharp softmax")
    mass = r["mass"].cpu().numpy()
    kth = np.sort(mass.reshape(-1, T), axis=1)[:, T - kk]
    print(f"sharp softmax: {(mass == 0).mean():.3f} of the masses are 0; k-th mass 0 in {(kth == 0).mean():.3f} "
          "of the rows")
    assert (kth < 2.0 ** -24).mean() > 0.5, "the case should put the k-th mass below the histogram's range"


def test_all_keys_selected(cm):
    T, h = 300, 2
    q, k, v = inputs(T, h)
    r = check_both_forms(cm, q, k, v, T, 1.0 / math.sqrt(128), "k = T")
    np.testing.assert_array_equal(r["idx"].cpu().numpy(), np.broadcast_to(np.arange(T, dtype=np.int32), (h, 3, T)))
