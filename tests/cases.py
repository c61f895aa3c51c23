"""Seeded parity cases built from the generator and the oracle only.

Every array here comes from ``dynamic_column_sparse_b200.synth`` or from an
``oracle`` call on such arrays; nothing is read back from the GPU.
"""
from __future__ import annotations

import functools
import math

import numpy as np

import oracle as O
from dynamic_column_sparse_b200 import synth


@functools.lru_cache(maxsize=4)
def mlp_case(seed: int, T: int, D: int, H: int, Bt: int, permille: int, sigma: float):
    """One MLP layer: cache = dense activations / output at x_prev (stored as
    bf16 / fp32), selection = top-k of the column L1 change at x_t."""
    L = synth.mlp_layer(seed, T, D, H, sigma)
    x_prev = O.bf16_decode(L["x_prev"])
    x_t = O.bf16_decode(L["x_t"])
    W1 = np.ascontiguousarray(O.bf16_decode(L["w1t"]).T)
    b1 = O.bf16_decode(L["b1"])
    W2 = O.bf16_decode(L["w2"])
    b2 = O.bf16_decode(L["b2"])
    a_prev, y_prev = O.dense_mlp(x_prev, W1, b1, W2, b2)
    A_bits = O.bf16_round(a_prev)
    Y32 = O.f32(y_prev)
    A64 = O.bf16_decode(A_bits)
    a_t, y_t = O.dense_mlp(x_t, W1, b1, W2, b2)
    k = O.k_from_density(H, permille)
    scores = O.mlp_scores(a_t, A64, Bt, first_step=False)
    idx = O.topk_cols(O.f32(scores), k)
    return dict(L=L, x_t=x_t, W1=W1, b1=b1, W2=W2, b2=b2, A_bits=A_bits, A64=A64, Y32=Y32, idx=idx, k=k,
                a_t=a_t, y_t=y_t, Bt=Bt, T=T, D=D, H=H)


@functools.lru_cache(maxsize=4)
def attn_case(seed: int, T: int, h: int, permille: int, sigma: float):
    """One attention layer: selection by attention mass at the previous step,
    cached complement partial at the previous step (stored fp32), current
    q, k, v after one drift step. Arrays in [h][T][d] (oracle layout)."""
    L = synth.attn_layer(seed, T, h, 128, sigma)
    hf = lambda a: np.ascontiguousarray(O.bf16_decode(a).transpose(1, 0, 2))
    qp, kp, vp = hf(L["q_prev"]), hf(L["k_prev"]), hf(L["v_prev"])
    q, k, v = hf(L["q"]), hf(L["k"]), hf(L["v"])
    scale = 1.0 / math.sqrt(128)
    kk = O.k_from_density(T, permille)
    mass = O.attn_mass(qp, kp, scale, 128)
    nb = mass.shape[1]
    idx = O.topk_cols(O.f32(mass.reshape(h * nb, T)), kk).reshape(h, nb, kk)
    m_c, l_c, acc_c = O.complement_partial(qp, kp, vp, idx, scale, 128)
    return dict(L=L, q=q, k=k, v=v, idx=idx, kk=kk, scale=scale,
                m_c=O.f32(m_c), l_c=O.f32(l_c), acc_c=O.f32(acc_c), T=T, h=h)
