"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (bf16 inputs, fp64 reference): attention outputs max-abs <= 2e-2 and
mean-abs <= 2e-3; masks bit-exact except on rows whose k-th and (k+1)-th block
scores differ by less than 1e-6 relative, where several masks are correct.

How a selection call is checked: the GPU mask is first validated against the
oracle's (bit-exact outside the tie band; inside it, the same kept count and
every kept block within the band), and the number of rows where it differs is
bounded.  The attention output is then compared on EVERY row -- the rows whose
masks differ included -- with the oracle's attention over the validated GPU mask,
which on all other rows is the oracle's own mask.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

from oracle import bsa_oracle as O

MAX_ABS = 2e-2
MEAN_ABS = 2e-3
TIE_REL = 1e-6
# Rows allowed to differ inside the tie band: at most 0.1% of the rows, and at
# least 2 (a tie of two equal-to-1e-6 scores is rare, but a small case may hit one).
DIFF_ROW_FRACTION = 1e-3


def max_diff_rows(n_rows: int) -> int:
    return max(2, math.ceil(DIFF_ROW_FRACTION * n_rows))


@dataclass
class MaskCheck:
    """A validated GPU mask (uint8 ndarray) and how it relates to the oracle's."""
    mask: np.ndarray
    rows: int
    exempt: int
    differing: int

    def __str__(self):
        return f"{self.differing} of {self.rows} rows differ (all inside the tie band; {self.exempt} rows in it)"


def _np(mask) -> np.ndarray:
    if isinstance(mask, torch.Tensor):
        mask = mask.cpu().numpy()
    return np.asarray(mask).astype(np.uint8)


def _bound(n_diff: int, rows: int, what: str):
    lim = max_diff_rows(rows)
    assert n_diff <= lim, f"{what}: {n_diff} of {rows} rows differ inside the tie band (allowed {lim})"


def compare_masks(mask_gpu, mask_ref: np.ndarray, P_ref: np.ndarray, k: int):
    """Returns (number of non-exempt mismatching rows, exempt rows, mismatching exempt rows).

    On exempt rows the GPU mask must still be a valid top-k: exactly k ones, and
    each kept score no smaller than the reference k-th score by more than the
    tie tolerance.
    """
    mg = _np(mask_gpu)
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


def check_topk_mask(mask_gpu, mask_ref: np.ndarray, P_ref: np.ndarray, topk: float,
                    causal: bool = False, what: str = "") -> MaskCheck:
    """Validates a top-k selection mask (non-causal or causal) and bounds the rows
    that differ from the oracle's inside the tie band."""
    mg = _np(mask_gpu)
    assert mg.shape == mask_ref.shape
    rows = int(np.prod(mg.shape[:-1]))
    if not causal:
        bad, n_ex, n_diff = compare_masks(mg, mask_ref, P_ref, O.keep_count(topk, mg.shape[-1]))
        assert bad == 0, f"{what}: {bad} mask rows differ outside the tie band"
    else:
        Kb = mg.shape[-1]
        n_ex = n_diff = 0
        for i in range(mg.shape[2]):
            E = O.causal_block_limit(i, Kb)
            assert np.all(mg[:, :, i, E:] == 0), f"{what}: row {i} keeps an ineligible block"
            bad, ex, diff = compare_masks(mg[:, :, i:i + 1, :E], mask_ref[:, :, i:i + 1, :E],
                                          P_ref[:, :, i:i + 1, :E], O.keep_count(topk, E))
            assert bad == 0, f"{what}: causal row {i} differs outside the tie band"
            n_ex += ex
            n_diff += diff
    _bound(n_diff, rows, what)
    return MaskCheck(mg, rows, n_ex, n_diff)


def compare_cdf_masks(mask_gpu, mask_ref: np.ndarray, P_ref: np.ndarray, tau: float):
    """cdfthreshd masks: rows may differ only where the decision is not determined
    at the inputs' precision (O.cdf_exempt_rows).  Every GPU row keeps at least one
    block, and on a differing exempt row the kept blocks are still a score-ordered
    prefix whose mass lies at the threshold to within the exemption's tolerance.
    Returns (non-exempt mismatching rows, exempt rows, mismatching exempt rows)."""
    mg = _np(mask_gpu)
    assert mg.shape == mask_ref.shape
    assert np.all(mg.sum(-1) >= 1)
    diff = np.any(mg != mask_ref, axis=-1)
    ex = O.cdf_exempt_rows(P_ref, tau)
    t32 = float(np.float32(tau))
    Kb = mg.shape[-1]
    flat_m, flat_p = mg.reshape(-1, Kb), P_ref.reshape(-1, Kb)
    for r in np.flatnonzero((diff & ex).reshape(-1)):
        p = flat_p[r]
        kept = np.flatnonzero(flat_m[r])
        order = np.lexsort((np.arange(Kb), -p))
        m = kept.size
        # a prefix of the score order, up to ties at its boundary
        assert p[kept].min() >= p[order[m - 1]] * (1 - 2 * TIE_REL), "cdf row kept a block off the prefix"
        cum = np.cumsum(p[order])
        assert m == Kb or cum[m - 1] >= t32 - 1e-4, "cdf row stops below the threshold"
        assert m == 1 or cum[m - 2] < t32 + 1e-4, "cdf row runs past the threshold"
    return int((diff & ~ex).sum()), int(ex.sum()), int((diff & ex).sum())


def check_cdf_mask(mask_gpu, mask_ref: np.ndarray, P_ref: np.ndarray, tau: float,
                   what: str = "") -> MaskCheck:
    mg = _np(mask_gpu)
    bad, n_ex, n_diff = compare_cdf_masks(mg, mask_ref, P_ref, tau)
    assert bad == 0, f"{what}: {bad} cdf mask rows differ outside the exemption"
    rows = int(np.prod(mg.shape[:-1]))
    _bound(n_diff, rows, what)
    return MaskCheck(mg, rows, n_ex, n_diff)


def differing_blocks(mc: MaskCheck, mask_ref: np.ndarray, b: int, h: int):
    """Query blocks of head (b, h) whose GPU mask differs from the oracle's."""
    return np.flatnonzero(np.any(mc.mask[b, h] != mask_ref[b, h], axis=-1)).tolist()


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
