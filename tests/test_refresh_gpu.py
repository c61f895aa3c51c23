"""Dense refresh on the GPU against the fp64 oracle.

Scores, rebuilt caches and outputs are compared within the float tolerance.
The new selection is a decision taken on float scores computed on each side,
so it is checked as a valid top-k of the oracle's scores within a small band;
rows where both sides select the same set also get their complement cache
compared with the oracle's."""
import numpy as np
import pytest

import oracle as O
from dynamic_column_sparse_b200 import synth
from helpers import (assert_bf16_storage, assert_is_topk_of, check_selection, assert_parity, bits_of, dev_bf16, dev_f32, f64_of, f64_of_bf16, heads_first, to_block_major,
                     to_token_major)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cm():
    from dynamic_column_sparse_b200 import chipmunk
    chipmunk.load_library()
    return chipmunk


@pytest.mark.parametrize("T,D,H,Bt,permille,first", [
    (256, 128, 512, 64, 250, True),
    (300, 192, 700, 128, 430, False),
    (4352, 3072, 12288, 128, 300, False),
])
def test_mlp_refresh(cm, T, D, H, Bt, permille, first):
    import torch
    L = synth.mlp_layer(5, T, D, H, 0.03)
    x = O.bf16_decode(L["x_t"])
    W1 = np.ascontiguousarray(O.bf16_decode(L["w1t"]).T)
    b1, W2, b2 = O.bf16_decode(L["b1"]), O.bf16_decode(L["w2"]), O.bf16_decode(L["b2"])
    # an old activation cache (the dense activations at x_prev) to score against
    a_old, _ = O.dense_mlp(O.bf16_decode(L["x_prev"]), W1, b1, W2, b2)
    A_old_bits = O.bf16_round(a_old)
    k = O.k_from_density(H, permille)
    nb = (T + Bt - 1) // Bt
    a_cache = dev_bf16(to_block_major(A_old_bits, Bt))
    y_cache = torch.empty((T, D), dtype=torch.float32, device="cuda")
    out = torch.empty((T, D), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((nb, k), dtype=torch.int32, device="cuda")
    scores = torch.empty((nb, H), dtype=torch.float32, device="cuda")
    cm.mlp_refresh(dev_bf16(L["x_t"]), dev_bf16(L["w1t"]), dev_bf16(L["b1"]), dev_bf16(L["w2"]), dev_bf16(L["b2"]),
                   a_cache, y_cache, idx, scores, out, Bt=Bt, first_step=first)
    torch.cuda.synchronize()
    assert cm.read_device_status() == 0
    ref = O.mlp_refresh(x, W1, b1, W2, b2, O.bf16_decode(A_old_bits), Bt, k, first)
    assert_bf16_storage(O.bf16_decode(to_token_major(bits_of(a_cache), T)), ref["a"], "a_cache")
    assert_parity(f64_of(y_cache), ref["y"], "y_cache")
    assert_parity(f64_of_bf16(out), ref["y"], "out", bf16_out=True)
    assert_parity(f64_of(scores), ref["scores"], "scores", max_of_rms=5e-3, mean_rel=1e-3)
    check_selection(idx.cpu().numpy(), ref["scores"], k, band=2e-3)


@pytest.mark.parametrize("T,h,permille", [(300, 2, 165), (700, 3, 300), (4352, 24, 165)])
def test_attn_refresh(cm, T, h, permille):
    import torch
    L = synth.attn_layer(6, T, h, 128, 0.03)
    hf = lambda a: np.ascontiguousarray(O.bf16_decode(a).transpose(1, 0, 2))
    q, k, v = hf(L["q"]), hf(L["k"]), hf(L["v"])
    scale = 1.0 / np.sqrt(128)
    kk = O.k_from_density(T, permille)
    nb = (T + 127) // 128
    o = torch.empty((T, h, 128), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((h, nb, kk), dtype=torch.int32, device="cuda")
    m_c = torch.empty((h, T), dtype=torch.float32, device="cuda")
    l_c = torch.empty((h, T), dtype=torch.float32, device="cuda")
    acc_c = torch.empty((h, T, 128), dtype=torch.float32, device="cuda")
    scores = torch.empty((h, nb, T), dtype=torch.float32, device="cuda")
    cm.attn_refresh(dev_bf16(L["q"]), dev_bf16(L["k"]), dev_bf16(L["v"]), idx, m_c, l_c, acc_c, o, scores,
                    scale=scale)
    torch.cuda.synchronize()
    assert cm.read_device_status() == 0
    ref = O.attn_refresh(q, k, v, scale, 128, kk)
    assert_parity(heads_first(f64_of_bf16(o)), ref["O"], "o", bf16_out=True)
    assert_parity(f64_of(scores), ref["mass"], "mass", max_of_rms=5e-3, mean_rel=1e-3)
    g_idx = idx.cpu().numpy()
    assert_is_topk_of(g_idx.reshape(h * nb, kk), scores.cpu().numpy().reshape(h * nb, T), "selection vs its own mass")
    same = check_selection(g_idx.reshape(h * nb, kk), ref["mass"].reshape(h * nb, T), kk, band=2e-3)
    assert same >= 0.9 * h * nb
    # complement cache on rows whose selection matches the oracle's
    gm, gl, ga = f64_of(m_c), f64_of(l_c), f64_of(acc_c)
    rows = []
    for hh in range(h):
        for b, r0, r1 in O.blocks(T, 128):
            if np.array_equal(g_idx[hh, b], ref["idx"][hh, b]):
                rows.append((hh, r0, r1))
    got_o = np.concatenate([ga[hh, r0:r1] / gl[hh, r0:r1, None] for hh, r0, r1 in rows])
    ref_o = np.concatenate([ref["acc_c"][hh, r0:r1] / ref["l_c"][hh, r0:r1, None] for hh, r0, r1 in rows])
    assert_parity(got_o, ref_o, "complement acc/l")
    got_lse = np.concatenate([gm[hh, r0:r1] + np.log(gl[hh, r0:r1]) for hh, r0, r1 in rows])
    ref_lse = np.concatenate([ref["m_c"][hh, r0:r1] + np.log(ref["l_c"][hh, r0:r1]) for hh, r0, r1 in rows])
    assert np.max(np.abs(got_lse - ref_lse)) < 1e-3, "complement log-sum-exp"


@pytest.mark.parametrize("T,h,permille", [(700, 2, 300), (4352, 24, 165)])
def test_attn_refresh_compact_cache(cm, T, h, permille):
    """The refresh writes the complement as lse_c (fp32) and o_c (bf16) when asked."""
    import torch
    L = synth.attn_layer(6, T, h, 128, 0.03)
    hf = lambda a: np.ascontiguousarray(O.bf16_decode(a).transpose(1, 0, 2))
    q, k, v = hf(L["q"]), hf(L["k"]), hf(L["v"])
    scale = 1.0 / np.sqrt(128)
    kk = O.k_from_density(T, permille)
    nb = (T + 127) // 128
    o = torch.empty((T, h, 128), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((h, nb, kk), dtype=torch.int32, device="cuda")
    lse_c = torch.empty((h, T), dtype=torch.float32, device="cuda")
    o_c = torch.empty((h, T, 128), dtype=torch.bfloat16, device="cuda")
    scores = torch.empty((h, nb, T), dtype=torch.float32, device="cuda")
    cm.attn_refresh(dev_bf16(L["q"]), dev_bf16(L["k"]), dev_bf16(L["v"]), idx, None, None, None, o, scores,
                    scale=scale, lse_c=lse_c, o_c=o_c)
    torch.cuda.synchronize()
    assert cm.read_device_status() == 0
    ref = O.attn_refresh(q, k, v, scale, 128, kk)
    assert_parity(heads_first(f64_of_bf16(o)), ref["O"], "o", bf16_out=True)
    g_idx = idx.cpu().numpy()
    same = check_selection(g_idx.reshape(h * nb, kk), ref["mass"].reshape(h * nb, T), kk, band=2e-3)
    assert same >= 0.9 * h * nb
    ref_lse, ref_oc = O.compact_partial(ref["m_c"], ref["l_c"], ref["acc_c"])
    got_lse, got_oc = f64_of(lse_c), f64_of_bf16(o_c)
    rows = [(hh, r0, r1) for hh in range(h) for b, r0, r1 in O.blocks(T, 128)
            if np.array_equal(g_idx[hh, b], ref["idx"][hh, b])]
    cat = lambda a: np.concatenate([a[hh, r0:r1] for hh, r0, r1 in rows])
    assert np.max(np.abs(cat(got_lse) - cat(ref_lse))) < 1e-3, "complement log-sum-exp"
    # o_c is a normalised attention output over the complement (P enters the MMA as bf16, as for o):
    # the bf16-output bar of o applies
    assert_parity(cat(got_oc), cat(ref_oc), "complement o_c", bf16_out=True)

