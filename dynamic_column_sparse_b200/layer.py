"""Per-layer state for the column-sparse delta method: caches, selections, schedule.

A diffusion transformer calls each layer once per denoising step. On a dense
(refresh) step the layer runs fully, scores every intermediate column, picks
the columns to recompute per token block and rebuilds its caches; on the
sparse steps in between it recomputes only those columns against the caches
(Chipmunk blog post, "Activation Deltas Across Diffusion Steps are Very
Sparse"; the HunyuanVideo table footnote runs 6 of 50 steps denser).

These classes own the device buffers and call the C ABI through
``dynamic_column_sparse_b200.chipmunk``; all arithmetic runs in the library's
CUDA kernels.
"""
from __future__ import annotations

import math

import torch

from . import chipmunk as cm


def k_from_density(n: int, density_permille: int) -> int:
    """Selected count per block for a kept fraction in per mille, rounded down."""
    return (int(n) * int(density_permille)) // 1000


class SparseDeltaMLP:
    """MLP ``gelu(x W1 + b1) W2 + b2`` with an activation / output cache.

    Weights: ``w1t`` [H][D] (W1 transposed), ``b1`` [H], ``w2`` [H][D],
    ``b2`` [D], all bf16 on one CUDA device. ``density_permille`` is the
    kept fraction of hidden columns per ``Bt``-token block.
    """

    def __init__(self, w1t, b1, w2, b2, T: int, Bt: int = 128, density_permille: int = 300):
        H, D = w1t.shape
        dev = w1t.device
        self.w1t, self.b1, self.w2, self.b2 = w1t, b1, w2, b2
        self.T, self.D, self.H, self.Bt = T, D, H, Bt
        self.nb = (T + Bt - 1) // Bt
        self.k = k_from_density(H, density_permille)
        self.a_cache = torch.zeros((self.nb, H, Bt), dtype=torch.bfloat16, device=dev)
        self.y_cache = torch.zeros((T, D), dtype=torch.float32, device=dev)
        self.out = torch.empty((T, D), dtype=torch.bfloat16, device=dev)
        self.idx = torch.zeros((self.nb, self.k), dtype=torch.int32, device=dev)
        self.scores = torch.empty((self.nb, H), dtype=torch.float32, device=dev)
        self.workspace = torch.empty(cm.mlp_workspace_bytes(T, H, self.k, Bt), dtype=torch.uint8, device=dev)
        self.has_cache = False

    def refresh(self, x, stream=None):
        """Dense step: output, column scores, new selection, rebuilt caches."""
        cm.mlp_refresh(x, self.w1t, self.b1, self.w2, self.b2, self.a_cache, self.y_cache, self.idx, self.scores,
                       self.out, Bt=self.Bt, first_step=not self.has_cache, stream=stream)
        self.has_cache = True
        return self.out

    def step(self, x, stream=None):
        """Sparse step: recompute the selected columns against the caches."""
        if not self.has_cache:
            raise RuntimeError("a sparse step needs a refresh first")
        cm.mlp_delta(x, self.w1t, self.b1, self.w2, self.idx, self.a_cache, self.y_cache, self.out, Bt=self.Bt,
                     workspace=self.workspace, stream=stream)
        return self.out


class SparseDeltaAttention:
    """Attention ``softmax(scale q k^T) v`` per head with a cached complement partial.

    ``q, k, v`` are [T][h][128] bf16. ``density_permille`` is the kept
    fraction of keys per (head, 128-query block). With ``compact`` the
    complement is cached as ``lse_c`` (fp32) and the normalised ``o_c`` (bf16)
    instead of ``m_c``, ``l_c``, ``acc_c`` (fp32): half the bytes. With
    ``keep_mass`` the refresh also keeps the attention mass ``scores``
    [h][nb][T] (fp32); otherwise the mass never leaves the refresh kernel's
    row buffers.
    """

    def __init__(self, T: int, h: int, device, density_permille: int = 165, scale: float | None = None,
                 compact: bool = False, keep_mass: bool = False):
        d = 128
        self.T, self.h, self.d = T, h, d
        self.nb = (T + 127) // 128
        self.k = k_from_density(T, density_permille)
        self.scale = 1.0 / math.sqrt(d) if scale is None else scale
        f32 = torch.float32
        self.idx = torch.zeros((h, self.nb, self.k), dtype=torch.int32, device=device)
        self.compact = compact
        if compact:
            self.lse_c = torch.empty((h, T), dtype=f32, device=device)
            self.o_c = torch.empty((h, T, d), dtype=torch.bfloat16, device=device)
            self.m_c = self.l_c = self.acc_c = None
        else:
            self.m_c = torch.empty((h, T), dtype=f32, device=device)
            self.l_c = torch.empty((h, T), dtype=f32, device=device)
            self.acc_c = torch.empty((h, T, d), dtype=f32, device=device)
            self.lse_c = self.o_c = None
        self.o = torch.empty((T, h, d), dtype=torch.bfloat16, device=device)
        self.scores = torch.empty((h, self.nb, T), dtype=f32, device=device) if keep_mass else None
        self.workspace = torch.empty(cm.attn_refresh_workspace_bytes(T, h, self.k, keep_mass), dtype=torch.uint8,
                                     device=device)
        self.has_cache = False

    def refresh(self, q, k, v, stream=None):
        """Dense step: output, attention mass, new key selection, complement cache."""
        cm.attn_refresh(q, k, v, self.idx, self.m_c, self.l_c, self.acc_c, self.o, self.scores, scale=self.scale,
                        workspace=self.workspace, stream=stream, lse_c=self.lse_c, o_c=self.o_c)
        self.has_cache = True
        return self.o

    def step(self, q, k, v, stream=None):
        """Sparse step: selected keys with the current q, k, v, merged with the cached complement."""
        if not self.has_cache:
            raise RuntimeError("a sparse step needs a refresh first")
        if self.compact:
            cm.attn_delta_compact(q, k, v, self.idx, self.lse_c, self.o_c, self.o, scale=self.scale, stream=stream)
        else:
            cm.attn_delta(q, k, v, self.idx, self.m_c, self.l_c, self.acc_c, self.o, scale=self.scale, stream=stream)
        return self.o


class Schedule:
    """Which denoising steps run dense: ``dense_steps`` (e.g. {0, 5} of 10)."""

    def __init__(self, dense_steps=(0,)):
        self.dense_steps = frozenset(dense_steps)

    def is_dense(self, step: int) -> bool:
        return step in self.dense_steps

    def run(self, layer, step: int, *inputs, stream=None):
        return layer.refresh(*inputs, stream=stream) if self.is_dense(step) else layer.step(*inputs, stream=stream)
