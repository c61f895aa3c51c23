"""HunyuanVideo-shaped layer (720x1280x129 video -> 33x90x160 latent, 2x2 patches
-> T = 118800 tokens; d_model 3072, MLP hidden 12288, 24 heads x 128) at full
size on the GPU, checked by the oracle on a seeded sample of 64 token blocks
(MLP) and 64 (head, query-block) tiles (attention), the short last block
(118800 = 928 * 128 + 16) always included.

Only the sampled rows (and, for attention, the sampled heads' keys and
values) are drawn by the counter-based generator that the oracle also sees;
the rest of each device tensor is filled by a seeded device generator, since
the kernels must run over the whole layer but the oracle checks only the
sample.
"""
import math

import numpy as np
import pytest

import oracle as O
from dynamic_column_sparse_b200 import synth
from helpers import assert_bf16_storage, assert_parity, bits_of, dev_bf16, f64_of_bf16

pytestmark = pytest.mark.gpu

T, D, H, NH, BT = 118800, 3072, 12288, 24, 128
NB = (T + BT - 1) // BT
SEED = 21


def block_rows(blocks):
    return np.concatenate([np.arange(b * BT, min((b + 1) * BT, T)) for b in blocks])


def sample_blocks(n, seed):
    rng = np.random.default_rng(seed)
    return sorted(set(rng.choice(NB - 1, n - 1, replace=False).tolist()) | {NB - 1})


def to_dev_bf16(bits):
    return dev_bf16(bits)


def test_hunyuan_mlp_delta_sampled():
    import torch
    g = torch.Generator(device="cuda").manual_seed(SEED)
    k = O.k_from_density(H, 300)
    assert k == 3686
    blocks = sample_blocks(64, 1)
    rows = block_rows(blocks)
    w1t = synth.normal_bf16(SEED, synth.TID["w1t"], (H, D), std=1 / math.sqrt(D))
    b1 = synth.normal_bf16(SEED, synth.TID["b1"], (H,), std=0.02)
    w2 = synth.normal_bf16(SEED, synth.TID["w2"], (H, D), std=1 / math.sqrt(H))
    b2 = synth.normal_bf16(SEED, synth.TID["b2"], (D,), std=0.02)
    xp = synth.rows_bf16(SEED, synth.TID["x_prev"], D, rows)
    xt = synth.drift_rows_bf16(xp, SEED, synth.TID["x_drift"], D, rows, 0.03)
    W1 = np.ascontiguousarray(O.bf16_decode(w1t).T)
    B1, W2, B2 = O.bf16_decode(b1), O.bf16_decode(w2), O.bf16_decode(b2)
    # oracle: cache = dense layer at x_prev on the sampled rows, selection from |a_t - A_c|
    a_prev, y_prev = O.dense_mlp(O.bf16_decode(xp), W1, B1, W2, B2)
    A_bits, Y32 = O.bf16_round(a_prev), O.f32(y_prev)
    A64 = O.bf16_decode(A_bits)
    a_t, _ = O.dense_mlp(O.bf16_decode(xt), W1, B1, W2, B2)
    idx_s = O.topk_cols(O.f32(O.mlp_scores(a_t, A64, BT, False)), k)
    A_new, Y_new = O.mlp_delta(O.bf16_decode(xt), W1, B1, W2, idx_s, A64, Y32.astype(np.float64), BT)
    # device tensors over the whole layer; the sampled rows carry the oracle's inputs
    rows_t = torch.from_numpy(rows).cuda()
    x = (torch.randn((T, D), generator=g, device="cuda")).to(torch.bfloat16)
    x[rows_t] = to_dev_bf16(xt)
    a_cache = (torch.randn((NB, H, BT), generator=g, device="cuda").abs() * 0.5).to(torch.bfloat16)
    y_cache = torch.randn((T, D), generator=g, device="cuda")
    y_cache[rows_t] = torch.from_numpy(Y32).cuda()
    idx = torch.sort(torch.rand((NB, H), generator=g, device="cuda").argsort(dim=1)[:, :k], dim=1)[0].to(torch.int32)
    r0 = 0
    for j, b in enumerate(blocks):
        n = min(BT, T - b * BT)
        blk = np.zeros((H, BT), dtype=np.uint16)
        blk[:, :n] = A_bits[r0:r0 + n].T
        a_cache[b] = to_dev_bf16(blk)
        idx[b] = torch.from_numpy(idx_s[j]).cuda()
        r0 += n
    out = torch.empty((T, D), dtype=torch.bfloat16, device="cuda")
    from dynamic_column_sparse_b200 import chipmunk as cm
    cm.mlp_delta(x, to_dev_bf16(w1t), to_dev_bf16(b1), to_dev_bf16(w2), idx.contiguous(), a_cache, y_cache, out,
                 Bt=BT)
    torch.cuda.synchronize()
    assert cm.read_device_status() == 0
    assert_parity(f64_of_bf16(out[rows_t]), Y_new, "out (sampled blocks)", bf16_out=True)
    assert_parity(y_cache[rows_t].double().cpu().numpy(), Y_new, "y_cache (sampled blocks)")
    got = np.concatenate([bits_of(a_cache[b])[:, :min(BT, T - b * BT)].T for b in blocks])
    sel = np.zeros_like(A_new, dtype=bool)
    r0 = 0
    for j, b in enumerate(blocks):
        n = min(BT, T - b * BT)
        sel[r0:r0 + n, idx_s[j]] = True
        r0 += n
    assert_bf16_storage(O.bf16_decode(got)[sel], A_new[sel], "a_cache (sampled, selected)")


def test_hunyuan_attention_delta_sampled():
    import torch
    from dynamic_column_sparse_b200 import chipmunk as cm
    g = torch.Generator(device="cuda").manual_seed(SEED + 1)
    kk = O.k_from_density(T, 70)
    assert kk == 8316
    heads = [0, 7, 13, 23]
    blocks = sample_blocks(16, 2)
    qrows = block_rows(blocks)
    scale = 1.0 / math.sqrt(128)
    tt = np.arange(T)
    q = torch.randn((T, NH, 128), generator=g, device="cuda").to(torch.bfloat16)
    kt = torch.randn((T, NH, 128), generator=g, device="cuda").to(torch.bfloat16)
    vt = torch.randn((T, NH, 128), generator=g, device="cuda").to(torch.bfloat16)
    m_c = torch.randn((NH, T), generator=g, device="cuda")
    l_c = torch.rand((NH, T), generator=g, device="cuda") * 100 + 1
    acc_c = torch.randn((NH, T, 128), generator=g, device="cuda")
    # unsampled tiles: a strided key set (distinct, ascending, in range)
    stride = T // kk
    shift = (torch.arange(NH, device="cuda")[:, None] + torch.arange(NB, device="cuda")[None, :]) % stride
    idx = (torch.arange(kk, device="cuda")[None, None, :] * stride + shift[:, :, None]).to(torch.int32).contiguous()
    expected = {}
    qrows_t = torch.from_numpy(qrows).cuda()
    for hh in heads:
        # the sampled head: keys / values at every token, queries on the sampled blocks, prev and current step
        all_rows = tt * NH + hh
        t_rows = qrows * NH + hh
        kp = synth.rows_bf16(SEED, synth.TID["k_prev"], 128, all_rows)
        vp = synth.rows_bf16(SEED, synth.TID["v_prev"], 128, all_rows)
        qp = synth.rows_bf16(SEED, synth.TID["q_prev"], 128, t_rows)
        kc = synth.drift_rows_bf16(kp, SEED, synth.TID["k_drift"], 128, all_rows, 0.03)
        vc = synth.drift_rows_bf16(vp, SEED, synth.TID["v_drift"], 128, all_rows, 0.03)
        qc = synth.drift_rows_bf16(qp, SEED, synth.TID["q_drift"], 128, t_rows, 0.03)
        Kp, Vp, Qp = O.bf16_decode(kp), O.bf16_decode(vp), O.bf16_decode(qp)
        # selection by attention mass at the previous step, complement cache at the previous step
        sel, mc, lc, ac = [], [], [], []
        r0 = 0
        for b in blocks:
            n = min(BT, T - b * BT)
            qb = Qp[r0:r0 + n]
            s_idx = O.topk_cols(O.f32(O.attn_mass_rows(qb, Kp, scale))[None, :], kk)[0]
            keep = np.ones(T, dtype=bool)
            keep[s_idx] = False
            m, l, a = O.attn_partial(qb, Kp[keep], Vp[keep], scale)
            sel.append(s_idx)
            mc.append(O.f32(m)), lc.append(O.f32(l)), ac.append(O.f32(a))
            r0 += n
        mc, lc, ac = np.concatenate(mc), np.concatenate(lc), np.concatenate(ac)
        ref = O.attn_delta(O.bf16_decode(qc)[None], O.bf16_decode(kc)[None], O.bf16_decode(vc)[None],
                           np.stack(sel)[None], mc[None].astype(np.float64), lc[None].astype(np.float64),
                           ac[None].astype(np.float64), scale, BT)[0]
        expected[hh] = ref
        kt[:, hh, :] = dev_bf16(kc)
        vt[:, hh, :] = dev_bf16(vc)
        q[qrows_t, hh, :] = dev_bf16(qc)
        m_c[hh, qrows_t] = torch.from_numpy(mc).cuda()
        l_c[hh, qrows_t] = torch.from_numpy(lc).cuda()
        acc_c[hh, qrows_t] = torch.from_numpy(ac).cuda()
        for j, b in enumerate(blocks):
            idx[hh, b] = torch.from_numpy(sel[j]).cuda()
    o = torch.empty((T, NH, 128), dtype=torch.bfloat16, device="cuda")
    cm.attn_delta(q, kt, vt, idx, m_c, l_c, acc_c, o, scale=scale)
    torch.cuda.synchronize()
    assert cm.read_device_status() == 0
    got = np.stack([f64_of_bf16(o[qrows_t, hh, :]) for hh in heads])
    ref = np.stack([expected[hh] for hh in heads])
    assert_parity(got, ref, "o (sampled tiles)", bf16_out=True)
