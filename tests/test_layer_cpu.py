"""Host logic of the per-layer objects (no kernel runs): the buffers they own, the selected counts,
the workspace each asks the library for, the dense/sparse schedule, and the refusal of a sparse step
before the first refresh."""
import math

import pytest
import torch

from dynamic_column_sparse_b200 import chipmunk as cm
from dynamic_column_sparse_b200.layer import Schedule, SparseDeltaAttention, SparseDeltaMLP, k_from_density


@pytest.fixture(scope="module", autouse=True)
def lib():
    cm.load_library()


def test_k_from_density_rounds_down():
    assert k_from_density(12288, 300) == 3686
    assert k_from_density(118800, 70) == 8316
    assert k_from_density(4352, 165) == 718
    assert k_from_density(7, 999) == 6 and k_from_density(5, 0) == 0


def test_mlp_layer_buffers_and_workspace():
    T, D, H, Bt = 300, 64, 700, 128
    w1t = torch.zeros((H, D), dtype=torch.bfloat16)
    w2 = torch.zeros((H, D), dtype=torch.bfloat16)
    layer = SparseDeltaMLP(w1t, torch.zeros(H, dtype=torch.bfloat16), w2, torch.zeros(D, dtype=torch.bfloat16), T, Bt,
                           430)
    nb = 3
    assert layer.k == 301 and layer.nb == nb
    assert layer.a_cache.shape == (nb, H, Bt) and layer.a_cache.dtype == torch.bfloat16
    assert layer.y_cache.shape == (T, D) and layer.y_cache.dtype == torch.float32
    assert layer.idx.shape == (nb, 301) and layer.scores.shape == (nb, H)
    # the delta workspace: nb blocks x round_up(k, 128) columns x Bt tokens of bf16
    assert layer.workspace.numel() == nb * 384 * Bt * 2 == cm.mlp_workspace_bytes(T, H, 301, Bt)
    with pytest.raises(RuntimeError, match="refresh first"):
        layer.step(torch.zeros((T, D), dtype=torch.bfloat16))


@pytest.mark.parametrize("keep_mass", [False, True])
@pytest.mark.parametrize("compact", [False, True])
def test_attention_layer_buffers_and_workspace(keep_mass, compact):
    T, h = 1001, 3
    layer = SparseDeltaAttention(T, h, "cpu", 300, compact=compact, keep_mass=keep_mass)
    nb = (T + 127) // 128
    assert layer.k == 300 and layer.nb == nb and math.isclose(layer.scale, 128 ** -0.5)
    assert layer.idx.shape == (h, nb, 300) and layer.o.shape == (T, h, 128)
    if compact:
        assert layer.lse_c.shape == (h, T) and layer.o_c.dtype == torch.bfloat16
        assert layer.m_c is None and layer.l_c is None and layer.acc_c is None
    else:
        assert layer.acc_c.shape == (h, T, 128) and layer.lse_c is None and layer.o_c is None
    if keep_mass:
        assert layer.scores.shape == (h, nb, T) and layer.scores.dtype == torch.float32
    else:
        assert layer.scores is None
    # the log-sum-exp rounded to 256 bytes, plus (mass not kept) the fused kernel's row buffers
    lse = (h * T * 4 + 255) // 256 * 256
    assert layer.workspace.numel() == cm.attn_refresh_workspace_bytes(T, h, 300, keep_mass)
    if keep_mass:
        assert layer.workspace.numel() == lse
    else:
        row = (T + 31) // 32 * 128
        extra = layer.workspace.numel() - lse - 128
        assert extra > 0 and extra % row == 0 and extra // row <= 2 * h * nb
    with pytest.raises(RuntimeError, match="refresh first"):
        z = torch.zeros((T, h, 128), dtype=torch.bfloat16)
        layer.step(z, z, z)


def test_schedule_picks_the_dense_steps():
    sched = Schedule((0, 5))
    assert [s for s in range(10) if sched.is_dense(s)] == [0, 5]
    calls = []

    class Probe:
        def refresh(self, *a, stream=None):
            calls.append(("refresh", a))
            return "dense"

        def step(self, *a, stream=None):
            calls.append(("step", a))
            return "sparse"

    assert [sched.run(Probe(), s, s) for s in range(7)] == ["dense"] + ["sparse"] * 4 + ["dense", "sparse"]
    assert [c[0] for c in calls][:2] == ["refresh", "step"] and calls[5] == ("refresh", (5,))
