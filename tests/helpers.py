"""Test glue: tensor conversions, layout changes and the parity tolerance.

Nothing here computes any part of the method; it moves bits between numpy,
torch and the library's storage layouts, and measures differences.
"""
from __future__ import annotations

import math

import numpy as np

import oracle as O

# Parity bar for floating-point outputs (bf16 inputs, fp32 accumulation):
# max |err| <= 2e-2 * RMS(reference) and mean relative error <= 5e-3.
MAX_ERR_OF_RMS = 2e-2
MEAN_REL_ERR = 5e-3


def dev_bf16(bits: np.ndarray, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def dev_f32(a: np.ndarray, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def dev_i32(a: np.ndarray, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


def bits_of(t) -> np.ndarray:
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f64_of_bf16(t) -> np.ndarray:
    return O.bf16_decode(bits_of(t))


def f64_of(t) -> np.ndarray:
    return t.detach().double().cpu().numpy()


def to_block_major(a_tok: np.ndarray, Bt: int, fill=0) -> np.ndarray:
    """[T][H] token-major -> [nb][H][Bt] block-column-major (slots past T get ``fill``)."""
    T, H = a_tok.shape
    nb = (T + Bt - 1) // Bt
    pad = np.full((nb * Bt, H), fill, dtype=a_tok.dtype)
    pad[:T] = a_tok
    return np.ascontiguousarray(pad.reshape(nb, Bt, H).transpose(0, 2, 1))


def to_token_major(a_blk: np.ndarray, T: int) -> np.ndarray:
    nb, H, Bt = a_blk.shape
    return np.ascontiguousarray(a_blk.transpose(0, 2, 1).reshape(nb * Bt, H)[:T])


def heads_first(a: np.ndarray) -> np.ndarray:
    """[T][h][d] -> [h][T][d]."""
    return np.ascontiguousarray(a.transpose(1, 0, 2))


def tokens_first(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a.transpose(1, 0, 2))


def err_stats(got: np.ndarray, ref: np.ndarray):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    d = np.abs(got - ref)
    rms = math.sqrt(float(np.mean(ref * ref))) if ref.size else 0.0
    mx = float(d.max()) if d.size else 0.0
    rel = float(d.sum() / max(np.abs(ref).sum(), 1e-300)) if d.size else 0.0
    return mx, rms, rel


def assert_bf16_storage(got, ref, what: str, mean_rel=MEAN_REL_ERR):
    """A cache stored as bf16: each value within one bf16 ulp of the reference
    (round-to-nearest storage plus the fp32 arithmetic before it), and the
    mean relative error bound of the output tolerance."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    rms = math.sqrt(float(np.mean(ref * ref))) if ref.size else 0.0
    d = np.abs(got - ref)
    bound = 2.0 ** -7 * np.abs(ref) + 1e-3 * rms
    bad = int(np.count_nonzero(d > bound))
    assert bad == 0, f"{what}: {bad} values beyond one bf16 ulp (worst {float((d - bound).max()):.3e})"
    rel = float(d.sum() / max(np.abs(ref).sum(), 1e-300))
    assert rel <= mean_rel, f"{what}: mean rel err {rel:.3e} > {mean_rel}"


def assert_parity(got, ref, what: str, max_of_rms=MAX_ERR_OF_RMS, mean_rel=MEAN_REL_ERR, bf16_out=False):
    """max |err| <= max_of_rms * RMS(ref) and mean relative error <= mean_rel.

    With ``bf16_out`` the result is stored as bf16 and each element may also
    carry its own storage rounding, at most half a bf16 ulp = 2^-8 |ref|: an
    output whose largest values exceed 5 RMS (attention outputs reach about
    6 RMS) cannot meet the bare bound whatever the arithmetic before it.
    """
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    mx, rms, rel = err_stats(got, ref)
    if bf16_out:
        excess = float(np.max(np.abs(got - ref) - 2.0 ** -8 * np.abs(ref))) if got.size else 0.0
        assert excess <= max_of_rms * rms + 1e-30, (
            f"{what}: max(|err| - 2^-8|ref|) {excess:.3e} > {max_of_rms} * RMS {rms:.3e}")
    else:
        assert mx <= max_of_rms * rms + 1e-30, f"{what}: max|err| {mx:.3e} > {max_of_rms} * RMS {rms:.3e}"
    assert rel <= mean_rel, f"{what}: mean rel err {rel:.3e} > {mean_rel}"
    return mx / max(rms, 1e-300), rel


def check_selection(idx, ref_scores, k, band):
    """idx rows: strictly ascending, k distinct; every kept score >= every dropped score - band * scale."""
    rows, n = ref_scores.shape
    assert idx.shape == (rows, k)
    same = 0
    ref_idx = O.topk_cols(O.f32(ref_scores), k)
    for r in range(rows):
        sel = idx[r]
        assert np.all(np.diff(sel) > 0) and sel.min() >= 0 and sel.max() < n
        if np.array_equal(sel, ref_idx[r]):
            same += 1
            continue
        mask = np.zeros(n, dtype=bool)
        mask[sel] = True
        scale = max(np.abs(ref_scores[r]).max(), 1e-30)
        if k and k < n:
            assert ref_scores[r][mask].min() >= ref_scores[r][~mask].max() - band * scale, f"row {r}"
    return same


def assert_is_topk_of(idx, scores, what: str):
    """Each row of ``idx`` is the exact top-k of the same row of ``scores`` (fp32 values, compared as
    numbers, so -0 equals +0), ties to the lower index, strictly ascending. A property check of a
    result against its own input: every kept score is >= every dropped one, and where the k-th value
    ties, the kept copies are the lowest-indexed ones."""
    idx = np.asarray(idx)
    scores = np.asarray(scores, dtype=np.float32)
    rows, k = idx.shape
    n = scores.shape[1]
    assert scores.shape[0] == rows
    if k == 0:
        return
    assert np.all(np.diff(idx, axis=1) > 0) if k > 1 else True, f"{what}: not strictly ascending"
    assert idx.min() >= 0 and idx.max() < n, f"{what}: index out of range"
    for r in range(rows):
        kept = np.zeros(n, dtype=bool)
        kept[idx[r]] = True
        tau = scores[r][kept].min()
        if k < n:
            dropped = scores[r][~kept]
            assert dropped.max() <= tau, f"{what}: row {r} drops a score above a kept one"
            tie_dropped = np.flatnonzero(~kept & (scores[r] == tau))
            tie_kept = np.flatnonzero(kept & (scores[r] == tau))
            if tie_dropped.size:
                assert tie_kept.max() < tie_dropped.min(), f"{what}: row {r} breaks a tie toward a higher index"
