"""Top-k column selection on the GPU against the oracle: bit-exact indices on
the same fp32 score rows (ties to the lower index)."""
import numpy as np
import pytest

import oracle as O
from dynamic_column_sparse_b200 import synth
from helpers import dev_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cm():
    from dynamic_column_sparse_b200 import chipmunk
    chipmunk.load_library()
    return chipmunk


@pytest.mark.parametrize("rows,n,k,ties", [
    (4, 512, 128, False),        # tiny MLP: 4 blocks x 512 hidden, 25%
    (4, 512, 128, True),
    (34, 12288, 3686, True),     # FLUX MLP scores
    (816, 4352, 718, True),      # FLUX attention mass rows (24 heads x 34 blocks)
    (7, 40960, 4096, True),      # longest row staged in shared memory
    (7, 40961, 4096, True),      # shortest row read from global memory
    (300, 118800, 8316, True),   # HunyuanVideo attention row length, two waves of the grid
    (3, 1000, 1, False),
    (3, 1000, 999, True),
])
def test_topk_matches_oracle(cm, rows, n, k, ties):
    s = synth.score_rows(7, rows, n, ties=ties)
    got = cm.topk_cols(dev_f32(s), k).cpu().numpy()
    np.testing.assert_array_equal(got, O.topk_cols(s, k))


def test_topk_special_values(cm):
    n = 3000
    rows = []
    rows.append(np.full(n, 0.5, dtype=np.float32))                       # all equal
    r = np.zeros(n, dtype=np.float32); r[::2] = -0.0; rows.append(r)      # -0 ties +0
    r = synth.score_rows(3, 1, n)[0] - 1.0; rows.append(r)                # negatives
    r = synth.score_rows(4, 1, n)[0]; r[[5, 17, 2999]] = np.inf; r[[7, 8]] = -np.inf; rows.append(r)
    r = np.round(synth.score_rows(5, 1, n)[0] * 2) / 2; rows.append(r.astype(np.float32))  # few distinct values
    s = np.stack(rows).astype(np.float32)
    for k in (0, 1, 2, 100, 1500, 2999, 3000):
        got = cm.topk_cols(dev_f32(s), k).cpu().numpy()
        np.testing.assert_array_equal(got, O.topk_cols(s, k), err_msg=f"k={k}")


def test_topk_tiny_rows(cm):
    for n in (1, 2, 3, 31, 33):
        s = synth.score_rows(n, 5, n, ties=True)
        for k in range(0, n + 1, max(1, n // 3)):
            got = cm.topk_cols(dev_f32(s), k).cpu().numpy()
            np.testing.assert_array_equal(got, O.topk_cols(s, k))


@pytest.mark.parametrize("rows,n,k", [
    (9, 45001, 3000),     # n not a multiple of 4: rows alternate between 16-byte aligned and not
    (5, 118800, 8316),    # HunyuanVideo attention row
    (3, 60000, 59999),
    (3, 50000, 1),
    (4, 50000, 30000),    # more candidates than the shared-memory buffer holds
])
def test_topk_long_rows(cm, rows, n, k):
    s = synth.score_rows(11, rows, n, ties=True)
    got = cm.topk_cols(dev_f32(s), k).cpu().numpy()
    np.testing.assert_array_equal(got, O.topk_cols(s, k))


def test_topk_long_special_values(cm):
    n = 50000
    rows = []
    rows.append(np.full(n, 0.5, dtype=np.float32))                               # all equal
    r = np.zeros(n, dtype=np.float32); r[::3] = -0.0; r[5::7] = 1e-30; rows.append(r)
    r = synth.score_rows(13, 1, n)[0] - 1.0; r[[0, 17, n - 1]] = np.inf; r[[3, 9]] = -np.inf; rows.append(r)
    r = np.round(synth.score_rows(14, 1, n)[0] * 2) / 2; rows.append(r.astype(np.float32))   # few distinct values
    # 20000 distinct values inside one 12-bit key bucket ([1, 1.125)) above 30000 small ones
    r = synth.score_rows(15, 1, n)[0] * 1e-3
    r[::5] = 1.0 + 0.1 * synth.uniform_f64(15, 99, (n + 4) // 5)[: len(r[::5])]
    r[1::5] = 1.0 + 0.1 * synth.uniform_f64(16, 99, len(r[1::5]))
    rows.append(r.astype(np.float32))
    s = np.stack(rows).astype(np.float32)
    for k in (1, 100, 4000, 19999, 20000, 20001, 49999):
        got = cm.topk_cols(dev_f32(s), k).cpu().numpy()
        np.testing.assert_array_equal(got, O.topk_cols(s, k), err_msg=f"k={k}")


def test_topk_long_rows_clustered_candidates(cm):
    """The top scores crowd one part of the row: one warp's share of the candidates outgrows its
    region while the row's total still fits (the candidates are then laid end to end)."""
    rows, n, k = 4, 60000, 3000
    s = synth.score_rows(17, rows, n, ties=True) * 1e-3
    hot = synth.score_rows(18, rows, 4000, ties=True) + 1.0
    s[:, 1000:5000] = hot                                 # the 3000 largest all sit in 4000 consecutive columns
    s[2, 30000:34000] = hot[2]                            # and, on one row, in two such runs
    got = cm.topk_cols(dev_f32(s.astype(np.float32)), k).cpu().numpy()
    np.testing.assert_array_equal(got, O.topk_cols(s.astype(np.float32), k))


def test_topk_long_rows_crowded_and_adversarial_samples(cm):
    """Rows whose values crowd a few 12-bit key buckets, like attention-mass rows (all near
    128 / T), and rows built against the sampled threshold of the long-row path: the largest
    values only where the sample does not look (the threshold comes out too low: too many
    candidates) or only where it looks (too high: too few)."""
    n, k = 118800, 8316
    z = synth.normal_f64(19, 1, 4 * n).reshape(4, n)
    rows = [1e-3 * (1.0 + 0.1 * z[0]), 1e-3 * (1.0 + 0.01 * z[1])]
    sampled = (np.arange(n) // 4) % 16 == 0              # float4 elements 0, 16, 32, ... are sampled
    r = 1e-3 * (1.0 + 0.1 * np.abs(z[2])); r[~sampled] += 1.0; rows.append(r)
    r = 1e-3 * (1.0 + 0.1 * np.abs(z[3])); r[sampled] += 1.0; rows.append(r)
    s = np.stack(rows).astype(np.float32)
    for kk in (k, 1, 9216, 9217):
        got = cm.topk_cols(dev_f32(s), kk).cpu().numpy()
        np.testing.assert_array_equal(got, O.topk_cols(s, kk), err_msg=f"k={kk}")
