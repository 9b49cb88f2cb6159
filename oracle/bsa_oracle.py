"""Plain, slow fp64 CPU oracle for mean-pooled top-k block selection and
block-sparse (128 x 64 tile) attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports this module; only the
tests, the smoke check and the benchmark's CPU-baseline leg call it.  It shares
no code with the CUDA path: everything below is numpy in float64, written as
the plain definition, with no blocking, fusion or reordering beyond what the
definition states.

What it computes, and where that comes from:

* The call pattern and tensor layout: ``spas_sage2_attn_meansim_topk_cuda(q, k,
  v, topk, is_causal=False)`` is a drop-in for scaled-dot-product attention on
  [B, H, N, d] tensors; ``block_sparse_sage2_attn_cuda(q, k, v, mask_id)`` takes
  a caller mask instead (SpargeAttention Documentation, the recommended-API
  paragraph and the block-sparse-mask paragraph).
* The mask: shape (B, H, ceil(N/128), ceil(N/64)), values 0/1, fixed block size
  128 x 64 (SpargeAttention Documentation, "Mask Requirements").
* ``topk`` trades accuracy (larger) for sparsity (smaller) (same page, the
  paragraph after the recommended API).
* Selection: mean-pool q over 128-row blocks and k over 64-row blocks, score
  the blocks with softmax(Qbar Kbar^T / sqrt(d)) per head, keep the top-k
  fraction of key blocks per query block ("meansim" and "topk" in the API
  name).  The pages name these steps but print no formula; the readings taken
  where they are silent are listed next to each function.
* Attention restricted to the kept tiles, non-causal, bf16 inputs (Attention
  Mechanisms, "Sol-Attn on Wan2.1": forward-only, non-causal, BF16).

Every function has a pin in tests/test_oracle_pins.py that checks it against
something other than itself (closed forms, brute force, library routines).
"""
from __future__ import annotations

import math

import numpy as np

# SpargeAttention Documentation, "Mask Requirements": the block is 128 x 64.
BLOCK_Q = 128
BLOCK_K = 64


def to_f64(t) -> np.ndarray:
    """bf16/fp32 torch tensor or array -> float64 ndarray (exact upcast)."""
    try:
        import torch

        if isinstance(t, torch.Tensor):
            return t.detach().to("cpu").to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(t, dtype=np.float64)


def block_counts(N: int) -> tuple[int, int]:
    """(ceil(N/128), ceil(N/64)).

    "Mask Requirements" prints the key count once as a mix of ceil and floor
    division and once as ceil(seq_len / 64); the ceiling is taken, so a partial
    last key block is its own block.
    """
    return -(-N // BLOCK_Q), -(-N // BLOCK_K)


def keep_count(topk: float, Kb: int) -> int:
    """Number of key blocks kept per query block for a top-k fraction.

    Reading (the pages are silent): k = ceil(topk * Kb) evaluated in float64
    on the float32 value of topk, clamped to [1, Kb], so topk = 1.0 is exactly
    dense and no row is ever empty.
    """
    t = float(np.float32(topk))
    k = int(math.ceil(t * Kb))
    return max(1, min(Kb, k))


def pool_mean(x: np.ndarray, block: int) -> np.ndarray:
    """Mean of x [B, H, N, d] over consecutive row blocks -> [B, H, ceil(N/block), d].

    Reading: a partial last block is averaged over its valid rows only.
    """
    B, H, N, d = x.shape
    nb = -(-N // block)
    out = np.empty((B, H, nb, d), dtype=np.float64)
    for i in range(nb):
        lo, hi = i * block, min((i + 1) * block, N)
        out[:, :, i, :] = x[:, :, lo:hi, :].sum(axis=2) / (hi - lo)
    return out


def block_scores(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """P = softmax_j(Qbar_i . Kbar_j / sqrt(d)) per (b, h, i) -> [B, H, Qb, Kb]."""
    d = qbar.shape[-1]
    S = np.matmul(qbar, np.swapaxes(kbar, -1, -2)) / math.sqrt(d)
    S = S - S.max(axis=-1, keepdims=True)
    E = np.exp(S)
    return E / E.sum(axis=-1, keepdims=True)


def topk_mask(P: np.ndarray, k: int) -> np.ndarray:
    """Keep the k largest entries of every row of P; equal scores go to the lower index.

    Returns uint8 [B, H, Qb, Kb] with exactly k ones per row.
    """
    Kb = P.shape[-1]
    rows = P.reshape(-1, Kb)
    mask = np.zeros(rows.shape, dtype=np.uint8)
    j = np.arange(Kb)
    for r in range(rows.shape[0]):
        order = np.lexsort((j, -rows[r]))  # primary: P descending, secondary: j ascending
        mask[r, order[:k]] = 1
    return mask.reshape(P.shape)


def cdf_mask(P: np.ndarray, threshold: float) -> np.ndarray:
    """cdfthreshd selection ("SpargeAttention Documentation", the --mode
    cdfthreshd flag of the inference scripts; the pages print no formula).

    Reading: order each row by P descending (equal scores: lower index first)
    and keep the shortest prefix whose cumulative mass reaches the threshold,
    at least one block.  If rounding leaves the total mass below the threshold,
    the whole row is kept.  threshold is taken as its float32 value.
    """
    tau = float(np.float32(threshold))
    Kb = P.shape[-1]
    rows = P.reshape(-1, Kb)
    mask = np.zeros(rows.shape, dtype=np.uint8)
    j = np.arange(Kb)
    for r in range(rows.shape[0]):
        order = np.lexsort((j, -rows[r]))
        cum = np.cumsum(rows[r][order])
        m = int(np.searchsorted(cum, tau, side="left"))  # first prefix whose sum >= tau
        mask[r, order[:min(m, Kb - 1) + 1]] = 1
    return mask.reshape(P.shape)


def select_cdf(q, k, threshold: float):
    """Mean-pool, score and cdfthreshd-select.  Returns (mask uint8, P float64)."""
    _, P = select(q, k, 1.0)
    return cdf_mask(P, threshold), P


def cdf_exempt_rows(P: np.ndarray, threshold: float, tol: float = 1e-4, tie_rel: float = 1e-6) -> np.ndarray:
    """Rows whose cdfthreshd decision is not determined at the precision of the
    inputs: the threshold lies within `tol` of a cumulative sum next to the cut,
    or the scores around the cut tie to within `tie_rel`."""
    tau = float(np.float32(threshold))
    Kb = P.shape[-1]
    rows = P.reshape(-1, Kb)
    ex = np.zeros(rows.shape[0], dtype=bool)
    j = np.arange(Kb)
    for r in range(rows.shape[0]):
        order = np.lexsort((j, -rows[r]))
        ps = rows[r][order]
        cum = np.cumsum(ps)
        m = min(int(np.searchsorted(cum, tau, side="left")), Kb - 1)
        near = abs(cum[m] - tau) < tol or (m > 0 and abs(cum[m - 1] - tau) < tol)
        tie = m + 1 < Kb and (ps[m] - ps[m + 1]) < tie_rel * ps[m]
        ex[r] = near or tie
    return ex.reshape(P.shape[:-1])


def causal_block_limit(i: int, Kb: int) -> int:
    """Number of key blocks that query block i may use under causal attention.

    Reading (is_causal is exposed by the recommended API on "SpargeAttention
    Documentation" but not described): key block j holds keys 64 j .. 64 j + 63
    and query block i rows 128 i .. 128 i + 127, so a key of block j precedes
    some row of block i exactly when j <= 2 i + 1.
    """
    return min(2 * i + 2, Kb)


def causal_topk_mask(P: np.ndarray, topk: float) -> np.ndarray:
    """Top-k among each row's causally eligible key blocks: row i keeps
    keep_count(topk, E_i) of its E_i = causal_block_limit(i, Kb) eligible blocks,
    equal scores to the lower index; ineligible blocks are never kept."""
    B, H, Qb, Kb = P.shape
    mask = np.zeros(P.shape, dtype=np.uint8)
    for i in range(Qb):
        E = causal_block_limit(i, Kb)
        mask[:, :, i, :E] = topk_mask(P[:, :, i:i + 1, :E], keep_count(topk, E))[:, :, 0]
    return mask


def select(q, k, topk: float, causal: bool = False):
    """Mean-pool, score and top-k select.  Returns (mask uint8, P float64).

    q and k may be bf16 torch tensors; they are upcast one (b, h) slice at a
    time so that full-size inputs fit in host memory.  With causal=True the
    top-k runs over each row's eligible key blocks (causal_topk_mask).
    """
    B, H, N, d = q.shape
    Qb, Kb = block_counts(N)
    qbar = np.empty((B, H, Qb, d))
    kbar = np.empty((B, H, Kb, d))
    for b in range(B):
        for h in range(H):
            qbar[b, h] = pool_mean(to_f64(q[b, h])[None, None], BLOCK_Q)[0, 0]
            kbar[b, h] = pool_mean(to_f64(k[b, h])[None, None], BLOCK_K)[0, 0]
    P = block_scores(qbar, kbar)
    if causal:
        return causal_topk_mask(P, topk), P
    return topk_mask(P, keep_count(topk, Kb)), P


def kept_key_columns(mask_row: np.ndarray, N: int) -> np.ndarray:
    """Token columns c < N covered by the kept key blocks of one mask row, ascending."""
    cols = [np.arange(j * BLOCK_K, min((j + 1) * BLOCK_K, N)) for j in np.flatnonzero(mask_row)]
    return np.concatenate(cols) if cols else np.zeros(0, dtype=np.int64)


def attention_rows(qh: np.ndarray, kh: np.ndarray, vh: np.ndarray, mask_row: np.ndarray,
                   i: int, causal: bool = False) -> np.ndarray:
    """Output rows [128 i, min(128 i + 128, N)) of one head -> [rows, d] float64.

    qh, kh, vh are that head's [N, d] float64 arrays and mask_row its Kb mask
    entries for query block i.  Softmax over the union of the kept key blocks
    (nonzero entries), scale 1/sqrt(d) as in scaled-dot-product attention,
    taken in two passes (row max, then exponentials and their sum).  Reading: a
    query block with no kept key block produces zeros.  With causal=True only
    keys at or before the row's own position count, and a row left with no
    such key produces zeros too.
    """
    N, d = qh.shape
    lo, hi = i * BLOCK_Q, min((i + 1) * BLOCK_Q, N)
    cols = kept_key_columns(mask_row, N)
    if cols.size == 0:
        return np.zeros((hi - lo, d), dtype=np.float64)
    S = qh[lo:hi] @ kh[cols].T / math.sqrt(d)
    if causal:
        S = np.where(cols[None, :] <= np.arange(lo, hi)[:, None], S, -np.inf)
    m = S.max(axis=1, keepdims=True)
    out = np.zeros((hi - lo, d), dtype=np.float64)
    live = np.isfinite(m[:, 0])
    if live.any():
        E = np.exp(S[live] - m[live])
        out[live] = (E @ vh[cols]) / E.sum(axis=1, keepdims=True)
    return out


def block_sparse_attention(q, k, v, mask, causal: bool = False) -> np.ndarray:
    """Full output [B, H, N, d] float64 of attention restricted to the kept tiles
    (and, with causal=True, to keys at or before each row)."""
    mask = np.asarray(mask)
    B, H, N, d = q.shape
    Qb, Kb = block_counts(N)
    assert mask.shape == (B, H, Qb, Kb), (mask.shape, (B, H, Qb, Kb))
    out = np.empty((B, H, N, d), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            qh, kh, vh = to_f64(q[b, h]), to_f64(k[b, h]), to_f64(v[b, h])
            for i in range(Qb):
                out[b, h, i * BLOCK_Q:min((i + 1) * BLOCK_Q, N)] = attention_rows(qh, kh, vh, mask[b, h, i], i,
                                                                                  causal)
    return out


def sparse_attention_topk(q, k, v, topk: float):
    """Selection followed by block-sparse attention.  Returns (O float64, mask)."""
    mask, _ = select(q, k, topk)
    return block_sparse_attention(q, k, v, mask), mask


def dense_attention(q, k, v) -> np.ndarray:
    """Textbook softmax(q k^T / sqrt(d)) v over all keys, per (b, h), float64."""
    q, k, v = to_f64(q), to_f64(k), to_f64(v)
    d = q.shape[-1]
    S = np.einsum("bhnd,bhmd->bhnm", q, k) / math.sqrt(d)
    S = S - S.max(axis=-1, keepdims=True)
    E = np.exp(S)
    return np.einsum("bhnm,bhmd->bhnd", E, v) / E.sum(axis=-1, keepdims=True)


def tie_exempt_rows(P: np.ndarray, k: int, rel: float = 1e-6) -> np.ndarray:
    """Rows whose k-th and (k+1)-th largest scores differ by less than `rel` relative.

    On such rows more than one mask is correct to the precision of the inputs,
    so a selection computed in another precision may legitimately differ there.
    Returns a bool array of shape P.shape[:-1].
    """
    Kb = P.shape[-1]
    if k >= Kb:
        return np.zeros(P.shape[:-1], dtype=bool)
    s = -np.sort(-P, axis=-1)
    pk, pk1 = s[..., k - 1], s[..., k]
    return (pk - pk1) < rel * pk


# ------------------------------------------------------------ token reordering
def token_permutation(T: int, Hg: int, Wg: int, text: int, mode: str) -> np.ndarray:
    """perm[new_position] = old_position for a [text | T x Hg x Wg video] sequence.

    The AB-Attention README ("Optional cube layout") groups video tokens into
    4 x 4 x 4 spatiotemporal cubes; the LightX2V page ("Sol-Attn on Wan2.1")
    applies a Morton3D ordering.  Readings: text tokens stay first and in place;
    "cube" orders video tokens by (t//4, h//4, w//4, t%4, h%4, w%4), cubes
    clipped at the grid edges; "morton" orders them by the Z-order key that
    interleaves the bits of (t, h, w) (t highest in each bit triple), ties
    impossible; "raster" is the identity.
    """
    nv = T * Hg * Wg
    m = np.arange(nv)
    t, h, w = m // (Hg * Wg), (m // Wg) % Hg, m % Wg
    if mode == "raster":
        order = m
    elif mode == "cube":
        order = np.lexsort((w % 4, h % 4, t % 4, w // 4, h // 4, t // 4))
    elif mode == "morton":
        key = np.zeros(nv, dtype=np.int64)
        for b in range(21):
            key |= ((t >> b) & 1) << (3 * b + 2)
            key |= ((h >> b) & 1) << (3 * b + 1)
            key |= ((w >> b) & 1) << (3 * b)
        order = np.argsort(key, kind="stable")
    else:
        raise ValueError(mode)
    return np.concatenate([np.arange(text), text + order]).astype(np.int64)


def kept_mass(q, k, mask, b: int, h: int, blocks) -> np.ndarray:
    """Share of each sampled row's dense softmax mass that falls in its kept key
    blocks (1.0 = the selection loses nothing), for the listed query blocks."""
    qh, kh = to_f64(q[b, h]), to_f64(k[b, h])
    N, d = qh.shape
    out = []
    for i in blocks:
        lo, hi = i * BLOCK_Q, min((i + 1) * BLOCK_Q, N)
        S = qh[lo:hi] @ kh.T / math.sqrt(d)
        E = np.exp(S - S.max(axis=1, keepdims=True))
        cols = kept_key_columns(mask[b, h, i], N)
        out.append(E[:, cols].sum(axis=1) / E.sum(axis=1))
    return np.concatenate(out)
