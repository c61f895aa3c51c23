"""Standalone cache column gather / scatter: bit-exact data movement."""
import numpy as np
import pytest

from dynamic_column_sparse_b200 import synth
from helpers import bits_of, dev_bf16, dev_i32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cm():
    from dynamic_column_sparse_b200 import chipmunk
    chipmunk.load_library()
    return chipmunk


@pytest.mark.parametrize("nb,H,Bt,k", [(4, 512, 64, 128), (34, 12288, 128, 3686), (3, 100, 128, 1), (2, 77, 64, 77)])
def test_gather_scatter_roundtrip(cm, nb, H, Bt, k):
    cache = synth.normal_bf16(11, 31, (nb, H, Bt))
    g = np.random.default_rng(nb * H + k)
    idx = np.sort(np.stack([g.choice(H, k, replace=False) for _ in range(nb)]), axis=1).astype(np.int32)
    d_cache, d_idx = dev_bf16(cache), dev_i32(idx)
    packed = cm.gather_cols(d_cache, d_idx)
    want = np.stack([cache[b][idx[b]] for b in range(nb)])
    np.testing.assert_array_equal(bits_of(packed), want)
    newvals = synth.normal_bf16(12, 31, (nb, k, Bt))
    cm.scatter_cols(dev_bf16(newvals), d_idx, d_cache)
    exp = cache.copy()
    for b in range(nb):
        exp[b][idx[b]] = newvals[b]
    np.testing.assert_array_equal(bits_of(d_cache), exp)
