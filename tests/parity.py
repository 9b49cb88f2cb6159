"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (bf16 inputs, fp64 reference): attention outputs max-abs <= 2e-2 and
mean-abs <= 2e-3; masks bit-exact except on rows whose k-th and (k+1)-th block
scores differ by less than 1e-6 relative, where several masks are correct.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import bsa_oracle as O

MAX_ABS = 2e-2
MEAN_ABS = 2e-3
TIE_REL = 1e-6


def compare_masks(mask_gpu: torch.Tensor, mask_ref: np.ndarray, P_ref: np.ndarray, k: int):
    """Returns (number of non-exempt mismatching rows, exempt rows, mismatching exempt rows).

    On exempt rows the GPU mask must still be a valid top-k: exactly k ones, and
    each kept score no smaller than the reference k-th score by more than the
    tie tolerance.
    """
    mg = mask_gpu.cpu().numpy().astype(np.uint8)
    assert mg.shape == mask_ref.shape
    assert set(np.unique(mg).tolist()) <= {0, 1}
    assert np.all(mg.sum(-1) == k), "every row must keep exactly k blocks"
    diff_rows = np.any(mg != mask_ref, axis=-1)
    exempt = O.tie_exempt_rows(P_ref, k, TIE_REL)
    bad = diff_rows & ~exempt
    if np.any(diff_rows & exempt):
        kth = -np.sort(-P_ref, axis=-1)[..., k - 1]
        kept_min = np.where(mg == 1, P_ref, np.inf).min(-1)
        ok = kept_min >= kth * (1 - 2 * TIE_REL)
        assert np.all(ok[diff_rows & exempt]), "an exempt row kept a block outside the tie band"
    return int(bad.sum()), int(exempt.sum()), int((diff_rows & exempt).sum())


def attn_errors(out_gpu_rows: np.ndarray, ref_rows: np.ndarray):
    err = np.abs(out_gpu_rows.astype(np.float64) - ref_rows)
    return float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0


def assert_close(out_gpu_rows: np.ndarray, ref_rows: np.ndarray, what: str = ""):
    assert np.all(np.isfinite(out_gpu_rows)), f"{what}: non-finite output"
    mx, mn = attn_errors(out_gpu_rows, ref_rows)
    assert mx <= MAX_ABS and mn <= MEAN_ABS, f"{what}: max-abs {mx:.3e} mean-abs {mn:.3e}"
    return mx, mn


def sampled_blocks(Qb: int, n_random: int, seed: int):
    """Query blocks {0, 1, Qb/2, Qb-1} plus seeded random ones (sorted, unique)."""
    rng = np.random.default_rng(seed)
    s = {0, min(1, Qb - 1), Qb // 2, Qb - 1}
    s |= set(rng.integers(0, Qb, size=n_random).tolist())
    return sorted(s)


def oracle_rows(q, k, v, mask_np: np.ndarray, b: int, h: int, blocks, cache=None):
    """Oracle output rows of the listed query blocks of head (b, h), concatenated."""
    qh, kh, vh = O.to_f64(q[b, h]), O.to_f64(k[b, h]), O.to_f64(v[b, h])
    return [O.attention_rows(qh, kh, vh, mask_np[b, h, i], i) for i in blocks]


def gpu_rows(out: torch.Tensor, b: int, h: int, blocks, N: int):
    o = out[b, h].float().cpu().numpy()
    return [o[i * 128:min(N, (i + 1) * 128)] for i in blocks]


def compare_cdf_masks(mask_gpu: torch.Tensor, mask_ref: np.ndarray, P_ref: np.ndarray, tau: float):
    """cdfthreshd masks: rows may differ only where the decision is not determined
    at the inputs' precision (O.cdf_exempt_rows).  Every GPU row keeps at least one
    block.  Returns (non-exempt mismatching rows, exempt rows)."""
    mg = mask_gpu.cpu().numpy().astype(np.uint8)
    assert mg.shape == mask_ref.shape
    assert np.all(mg.sum(-1) >= 1)
    diff = np.any(mg != mask_ref, axis=-1)
    ex = O.cdf_exempt_rows(P_ref, tau)
    return int((diff & ~ex).sum()), int(ex.sum())


def workspace_lists(ws: torch.Tensor, BH: int, Qb: int, Kb: int, d: int):
    """The compacted (idx, cnt) lists from a workspace, at the offsets of the
    layout include/bsa.h documents: status 256 | qbar | kbar | block scores (rows
    padded to 4 floats) | idx int16 | cnt int32, each rounded up to 256 bytes."""
    r = lambda x: (x + 255) // 256 * 256
    Kp = (Kb + 3) // 4 * 4
    o_idx = 256 + r(BH * Qb * d * 4) + r(BH * Kb * d * 4) + r(BH * Qb * Kp * 4)
    o_cnt = o_idx + r(BH * Qb * Kb * 2)
    idx = ws[o_idx:o_idx + BH * Qb * Kb * 2].view(torch.int16).view(BH * Qb, Kb).cpu().numpy()
    cnt = ws[o_cnt:o_cnt + BH * Qb * 4].view(torch.int32).cpu().numpy()
    return idx, cnt
