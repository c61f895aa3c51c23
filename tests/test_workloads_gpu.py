"""The pages' two larger workloads at full size on the GPU, checked by the oracle
on seeded samples:

* HunyuanVideo (720x1280x129 video -> 33x90x160 latent, 2x2 patches ->
  T = 118800 tokens; d_model 3072, MLP hidden 12288, 24 heads x 128; MLP 70%
  and attention 93% sparse): the sparse step and the dense refresh.
* FLUX.1-dev at 2304x1280 (144x80 latent patches + 512 text tokens ->
  T = 12032; MLP 70% and attention 83.5% sparse, k = 3686 and 1985): the
  sparse step.

The kernels run over the whole layer; the oracle checks sampled token blocks
(MLP) and sampled (head, query-block) tiles (attention), the short last block
always included (118800 = 928 * 128 + 16; 12032 = 94 * 128). Only the sampled
rows (and, for attention, the sampled heads' keys and values) are drawn by
the counter-based generator the oracle also sees; the rest of each device
tensor is filled by a seeded device generator.
"""
import math

import numpy as np
import pytest

import oracle as O
from dynamic_column_sparse_b200 import synth
from helpers import (assert_bf16_storage, assert_is_topk_of, assert_parity, bits_of, check_selection, dev_bf16,
                     f64_of, f64_of_bf16)

pytestmark = pytest.mark.gpu

D, H, NH, BT = 3072, 12288, 24, 128
SEED = 21
# name: (T, MLP kept per mille, attention kept per mille, sampled MLP blocks, sampled attention heads / blocks)
WORKLOADS = {
    "hunyuan_720x1280x129": (118800, 300, 70, 64, ([0, 7, 13, 23], 16)),
    "flux_2304x1280": (144 * 80 + 512, 300, 165, 32, ([2, 11, 19], 12)),
}


def nblocks(T):
    return (T + BT - 1) // BT


def block_rows(T, blocks):
    return np.concatenate([np.arange(b * BT, min((b + 1) * BT, T)) for b in blocks])


def sample_blocks(T, n, seed):
    """n sampled blocks, sorted, the last block of the layer always among them (and last)."""
    nb = nblocks(T)
    rng = np.random.default_rng(seed)
    return sorted(set(rng.choice(nb - 1, n - 1, replace=False).tolist()) | {nb - 1})


def mlp_weights():
    w1t = synth.normal_bf16(SEED, synth.TID["w1t"], (H, D), std=1 / math.sqrt(D))
    b1 = synth.normal_bf16(SEED, synth.TID["b1"], (H,), std=0.02)
    w2 = synth.normal_bf16(SEED, synth.TID["w2"], (H, D), std=1 / math.sqrt(H))
    b2 = synth.normal_bf16(SEED, synth.TID["b2"], (D,), std=0.02)
    W1 = np.ascontiguousarray(O.bf16_decode(w1t).T)
    return (w1t, b1, w2, b2), (W1, O.bf16_decode(b1), O.bf16_decode(w2), O.bf16_decode(b2))


def scatter_block_cache(a_cache, T, blocks, A_bits):
    """Write the sampled blocks' [rows][H] bf16 activations into the device cache [nb][H][Bt]."""
    r0 = 0
    for b in blocks:
        n = min(BT, T - b * BT)
        blk = np.zeros((H, BT), dtype=np.uint16)
        blk[:, :n] = A_bits[r0:r0 + n].T
        a_cache[b] = dev_bf16(blk)
        r0 += n


def gather_block_cache(a_cache, T, blocks):
    return np.concatenate([bits_of(a_cache[b])[:, :min(BT, T - b * BT)].T for b in blocks])


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_mlp_delta_sampled(name):
    import torch
    from dynamic_column_sparse_b200 import chipmunk as cm
    T, mlp_pm, _, nsample, _ = WORKLOADS[name]
    NB = nblocks(T)
    g = torch.Generator(device="cuda").manual_seed(SEED)
    k = O.k_from_density(H, mlp_pm)
    assert k == 3686
    blocks = sample_blocks(T, nsample, 1)
    rows = block_rows(T, blocks)
    (w1t, b1, w2, b2), (W1, B1, W2, B2) = mlp_weights()
    xp = synth.rows_bf16(SEED, synth.TID["x_prev"], D, rows)
    xt = synth.drift_rows_bf16(xp, SEED, synth.TID["x_drift"], D, rows, 0.03)
    # oracle: cache = dense layer at x_prev on the sampled rows, selection from |a_t - A_c|
    a_prev, y_prev = O.dense_mlp(O.bf16_decode(xp), W1, B1, W2, B2)
    A_bits, Y32 = O.bf16_round(a_prev), O.f32(y_prev)
    A64 = O.bf16_decode(A_bits)
    a_t, _ = O.dense_mlp(O.bf16_decode(xt), W1, B1, W2, B2)
    idx_s = O.topk_cols(O.f32(O.mlp_scores(a_t, A64, BT, False)), k)
    A_new, Y_new = O.mlp_delta(O.bf16_decode(xt), W1, B1, W2, idx_s, A64, Y32.astype(np.float64), BT)
    # device tensors over the whole layer; the sampled rows carry the oracle's inputs
    rows_t = torch.from_numpy(rows).cuda()
    x = torch.randn((T, D), generator=g, device="cuda").to(torch.bfloat16)
    x[rows_t] = dev_bf16(xt)
    a_cache = (torch.randn((NB, H, BT), generator=g, device="cuda").abs() * 0.5).to(torch.bfloat16)
    y_cache = torch.randn((T, D), generator=g, device="cuda")
    y_cache[rows_t] = torch.from_numpy(Y32).cuda()
    idx = torch.sort(torch.rand((NB, H), generator=g, device="cuda").argsort(dim=1)[:, :k], dim=1)[0].to(torch.int32)
    scatter_block_cache(a_cache, T, blocks, A_bits)
    for j, b in enumerate(blocks):
        idx[b] = torch.from_numpy(idx_s[j]).cuda()
    out = torch.empty((T, D), dtype=torch.bfloat16, device="cuda")
    cm.mlp_delta(x, dev_bf16(w1t), dev_bf16(b1), dev_bf16(w2), idx.contiguous(), a_cache, y_cache, out, Bt=BT)
    torch.cuda.synchronize()
    assert cm.read_device_status() == 0
    r = assert_parity(f64_of_bf16(out[rows_t]), Y_new, "out (sampled blocks)", bf16_out=True)
    print(f"{name} MLP out: max|err|/rms {r[0]:.4f}")
    assert_parity(y_cache[rows_t].double().cpu().numpy(), Y_new, "y_cache (sampled blocks)")
    got = gather_block_cache(a_cache, T, blocks)
    sel = np.zeros_like(A_new, dtype=bool)
    r0 = 0
    for j, b in enumerate(blocks):
        n = min(BT, T - b * BT)
        sel[r0:r0 + n, idx_s[j]] = True
        r0 += n
    assert_bf16_storage(O.bf16_decode(got)[sel], A_new[sel], "a_cache (sampled, selected)")
    np.testing.assert_array_equal(got[~sel], A_bits[~sel])


def sampled_head_inputs(T, hh, qrows, step):
    """One head's keys / values at every token and queries at the sampled rows, at the previous step
    (step 0) or after one drift step (step 1), as bf16 bits."""
    all_rows = np.arange(T) * NH + hh
    t_rows = qrows * NH + hh
    kp = synth.rows_bf16(SEED, synth.TID["k_prev"], 128, all_rows)
    vp = synth.rows_bf16(SEED, synth.TID["v_prev"], 128, all_rows)
    qp = synth.rows_bf16(SEED, synth.TID["q_prev"], 128, t_rows)
    if step == 0:
        return qp, kp, vp
    kc = synth.drift_rows_bf16(kp, SEED, synth.TID["k_drift"], 128, all_rows, 0.03)
    vc = synth.drift_rows_bf16(vp, SEED, synth.TID["v_drift"], 128, all_rows, 0.03)
    qc = synth.drift_rows_bf16(qp, SEED, synth.TID["q_drift"], 128, t_rows, 0.03)
    return (qp, kp, vp), (qc, kc, vc)


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_attention_delta_sampled(name):
    import torch
    from dynamic_column_sparse_b200 import chipmunk as cm
    T, _, attn_pm, _, (heads, nsample) = WORKLOADS[name]
    NB = nblocks(T)
    g = torch.Generator(device="cuda").manual_seed(SEED + 1)
    kk = O.k_from_density(T, attn_pm)
    assert kk == {118800: 8316, 12032: 1985}[T]
    blocks = sample_blocks(T, nsample, 2)
    qrows = block_rows(T, blocks)
    scale = 1.0 / math.sqrt(128)
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
        (qp, kp, vp), (qc, kc, vc) = sampled_head_inputs(T, hh, qrows, 1)
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
    r = assert_parity(got, ref, "o (sampled tiles)", bf16_out=True)
    print(f"{name} attention o: max|err|/rms {r[0]:.4f}")


def test_mlp_refresh_sampled_hunyuan():
    """Dense MLP refresh at T = 118800: rebuilt caches, output, column scores against an old cache,
    and the new selection, on 8 sampled token blocks."""
    import torch
    from dynamic_column_sparse_b200 import chipmunk as cm
    T = 118800
    NB = nblocks(T)
    g = torch.Generator(device="cuda").manual_seed(SEED + 2)
    k = O.k_from_density(H, 300)
    blocks = sample_blocks(T, 8, 3)
    rows = block_rows(T, blocks)
    (w1t, b1, w2, b2), (W1, B1, W2, B2) = mlp_weights()
    xp = synth.rows_bf16(SEED, synth.TID["x_prev"], D, rows)
    xt = synth.drift_rows_bf16(xp, SEED, synth.TID["x_drift"], D, rows, 0.03)
    a_old, _ = O.dense_mlp(O.bf16_decode(xp), W1, B1, W2, B2)
    A_old_bits = O.bf16_round(a_old)
    ref = O.mlp_refresh(O.bf16_decode(xt), W1, B1, W2, B2, O.bf16_decode(A_old_bits), BT, k, first_step=False)
    rows_t = torch.from_numpy(rows).cuda()
    x = torch.randn((T, D), generator=g, device="cuda").to(torch.bfloat16)
    x[rows_t] = dev_bf16(xt)
    a_cache = (torch.randn((NB, H, BT), generator=g, device="cuda").abs() * 0.5).to(torch.bfloat16)
    scatter_block_cache(a_cache, T, blocks, A_old_bits)
    y_cache = torch.empty((T, D), dtype=torch.float32, device="cuda")
    out = torch.empty((T, D), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((NB, k), dtype=torch.int32, device="cuda")
    scores = torch.empty((NB, H), dtype=torch.float32, device="cuda")
    cm.mlp_refresh(x, dev_bf16(w1t), dev_bf16(b1), dev_bf16(w2), dev_bf16(b2), a_cache, y_cache, idx, scores, out,
                   Bt=BT, first_step=False)
    torch.cuda.synchronize()
    assert cm.read_device_status() == 0
    bl = torch.tensor(blocks, device="cuda")
    assert_bf16_storage(O.bf16_decode(gather_block_cache(a_cache, T, blocks)), ref["a"], "a_cache (sampled)")
    assert_parity(f64_of(y_cache[rows_t]), ref["y"], "y_cache (sampled)")
    assert_parity(f64_of_bf16(out[rows_t]), ref["y"], "out (sampled)", bf16_out=True)
    g_scores = scores[bl].cpu().numpy()
    assert_parity(g_scores.astype(np.float64), ref["scores"], "scores (sampled)", max_of_rms=5e-3, mean_rel=1e-3)
    g_idx = idx[bl].cpu().numpy()
    assert_is_topk_of(g_idx, g_scores, "MLP selection vs its own scores")
    same = check_selection(g_idx, ref["scores"], k, band=2e-3)
    print(f"hunyuan MLP refresh: {same} of {len(blocks)} sampled selections as the oracle's")


def test_attention_refresh_sampled_hunyuan():
    """Dense attention refresh at T = 118800 (dense pass, attention mass with the top-k over its 22296
    rows of 118800, complement pass): output, mass rows, selection and complement cache on 32 sampled
    (head, query-block) tiles; every row's selection against the standalone top-k of the kept mass;
    the refresh without a mass tensor against the one with."""
    import torch
    from dynamic_column_sparse_b200 import chipmunk as cm
    T = 118800
    NB = nblocks(T)
    g = torch.Generator(device="cuda").manual_seed(SEED + 3)
    kk = O.k_from_density(T, 70)
    heads = [3, 16]
    blocks = sample_blocks(T, 16, 4)
    qrows = block_rows(T, blocks)
    scale = 1.0 / math.sqrt(128)
    q = torch.randn((T, NH, 128), generator=g, device="cuda").to(torch.bfloat16)
    kt = torch.randn((T, NH, 128), generator=g, device="cuda").to(torch.bfloat16)
    vt = torch.randn((T, NH, 128), generator=g, device="cuda").to(torch.bfloat16)
    qrows_t = torch.from_numpy(qrows).cuda()
    host = {}
    for hh in heads:
        qp, kp, vp = sampled_head_inputs(T, hh, qrows, 0)
        host[hh] = (O.bf16_decode(qp), O.bf16_decode(kp), O.bf16_decode(vp))
        kt[:, hh, :] = dev_bf16(kp)
        vt[:, hh, :] = dev_bf16(vp)
        q[qrows_t, hh, :] = dev_bf16(qp)
    layer_idx = torch.empty((NH, NB, kk), dtype=torch.int32, device="cuda")
    m_c = torch.empty((NH, T), dtype=torch.float32, device="cuda")
    l_c = torch.empty((NH, T), dtype=torch.float32, device="cuda")
    acc_c = torch.empty((NH, T, 128), dtype=torch.float32, device="cuda")
    o = torch.empty((T, NH, 128), dtype=torch.bfloat16, device="cuda")
    mass = torch.empty((NH, NB, T), dtype=torch.float32, device="cuda")
    cm.attn_refresh(q, kt, vt, layer_idx, m_c, l_c, acc_c, o, mass, scale=scale)
    torch.cuda.synchronize()
    assert cm.read_device_status() == 0
    bl = torch.tensor(blocks, device="cuda")
    got_o, ref_o, got_mass, ref_mass, got_idx = [], [], [], [], []
    cmp_rows = []   # (head, sampled block j, oracle partial over the oracle's complement)
    for hh in heads:
        Q, K, V = host[hh]
        got_o.append(f64_of_bf16(o[qrows_t, hh, :]))
        got_mass.append(mass[hh, bl].cpu().numpy())
        got_idx.append(layer_idx[hh, bl].cpu().numpy())
        r0 = 0
        for j, b in enumerate(blocks):
            n = min(BT, T - b * BT)
            qb = Q[r0:r0 + n]
            ref_o.append(O.finish(O.attn_partial(qb, K, V, scale)))
            mrow = O.attn_mass_rows(qb, K, scale)
            ref_mass.append(mrow)
            s_idx = O.topk_cols(O.f32(mrow)[None, :], kk)[0]
            keep = np.ones(T, dtype=bool)
            keep[s_idx] = False
            cmp_rows.append((hh, j, r0, n, s_idx, O.attn_partial(qb, K[keep], V[keep], scale)))
            r0 += n
    assert_parity(np.concatenate(got_o), np.concatenate(ref_o), "o (sampled tiles)", bf16_out=True)
    got_mass = np.concatenate(got_mass)
    ref_mass = np.stack(ref_mass)
    assert_parity(got_mass.astype(np.float64), ref_mass, "mass (sampled rows)", max_of_rms=5e-3, mean_rel=1e-3)
    got_idx = np.concatenate(got_idx)
    assert_is_topk_of(got_idx, got_mass, "selection vs its own mass rows")
    same = check_selection(got_idx, ref_mass, kk, band=2e-3)
    print(f"hunyuan attention refresh: {same} of {len(got_idx)} sampled selections as the oracle's")
    # complement cache on the tiles whose selection matches the oracle's
    gm, gl, ga = (f64_of(t[:, qrows_t]) for t in (m_c, l_c, acc_c))
    got_c, ref_c, got_lse, ref_lse = [], [], [], []
    for t, (hh, j, r0, n, s_idx, (m, l, acc)) in enumerate(cmp_rows):
        if not np.array_equal(got_idx[t], s_idx):
            continue
        got_c.append(ga[hh, r0:r0 + n] / gl[hh, r0:r0 + n, None])
        ref_c.append(acc / l[:, None])
        got_lse.append(gm[hh, r0:r0 + n] + np.log(gl[hh, r0:r0 + n]))
        ref_lse.append(m + np.log(l))
    assert got_c, "no sampled tile selects as the oracle does"
    assert_parity(np.concatenate(got_c), np.concatenate(ref_c), "complement acc/l (matching tiles)")
    assert np.max(np.abs(np.concatenate(got_lse) - np.concatenate(ref_lse))) < 1e-3, "complement log-sum-exp"
    # every row's in-kernel selection equals the standalone top-k kernel's on the same kept mass rows
    # (that kernel is bit-exact against the oracle's top-k in the top-k tests)
    alone = cm.topk_cols(mass.view(NH * NB, T), kk)
    assert torch.equal(alone, layer_idx.view(NH * NB, kk)), "fused selection vs standalone top-k"
    # without a mass tensor the mass stays in the kernel's row buffers: the same selection, output and cache
    del mass, alone
    kept = [t.clone() for t in (layer_idx, o, m_c, l_c, acc_c)]
    cm.attn_refresh(q, kt, vt, layer_idx, m_c, l_c, acc_c, o, None, scale=scale)
    torch.cuda.synchronize()
    assert cm.read_device_status() == 0
    for a, b, what in zip((layer_idx, o, m_c, l_c, acc_c), kept, ("idx", "o", "m_c", "l_c", "acc_c")):
        assert torch.equal(a, b), f"refresh without a mass tensor: {what} differs"
