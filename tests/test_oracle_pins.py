"""Pins for the fp64 oracle: every function is checked against something other
than itself (hand-worked shapes, closed forms, brute force over all subsets,
torch's scaled_dot_product_attention and scipy's softmax as library routines,
and invariants of attention).  No GPU."""
import itertools
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import softmax as scipy_softmax

from oracle import bsa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- block counts
def test_block_counts_match_hand_worked_shapes():
    rows = []
    with open(os.path.join(GOLDEN, "mask_shapes.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                rows.append(tuple(int(x) for x in line.split()))
    assert len(rows) >= 9
    for N, qb, kb in rows:
        assert O.block_counts(N) == (qb, kb), N


def test_keep_count_values():
    # k = ceil(topk * Kb), at least 1, at most Kb (hand-worked).
    assert O.keep_count(1.0, 1182) == 1182
    assert O.keep_count(0.5, 1182) == 591
    assert O.keep_count(0.3, 1182) == 355  # 354.6 -> 355
    assert O.keep_count(0.1, 1182) == 119  # 118.2 -> 119
    assert O.keep_count(0.1, 1857) == 186  # 185.7 -> 186
    assert O.keep_count(0.5, 278) == 139
    assert O.keep_count(0.5, 16) == 8
    assert O.keep_count(1e-6, 10) == 1
    assert O.keep_count(0.25, 4) == 1
    assert O.keep_count(0.26, 4) == 2


# --------------------------------------------------------------------- pooling
@pytest.mark.parametrize("block", [128, 64])
def test_pool_mean_closed_form_all_ragged_lengths(block):
    # x[n, c] = n + 1000 c: the mean over rows [lo, hi) is (lo + hi - 1) / 2 + 1000 c.
    for N in range(1, 301):
        d = 3
        x = (np.arange(N)[:, None] + 1000.0 * np.arange(d)[None, :])[None, None]
        got = O.pool_mean(x, block)
        nb = -(-N // block)
        assert got.shape == (1, 1, nb, d)
        for i in range(nb):
            lo, hi = i * block, min(N, (i + 1) * block)
            want = (lo + hi - 1) / 2.0 + 1000.0 * np.arange(d)
            np.testing.assert_allclose(got[0, 0, i], want, rtol=0, atol=1e-9)


def test_pool_mean_constant_blocks():
    rng = _rng(1)
    consts = rng.normal(size=(2, 3, 5, 7))
    x = np.repeat(consts, 64, axis=2)[:, :, :300]  # blocks of 64 identical rows, ragged end
    got = O.pool_mean(x, 64)
    np.testing.assert_allclose(got, consts, rtol=0, atol=1e-12)


# -------------------------------------------------------------- block scores
def test_block_scores_closed_form_and_scale():
    # Qbar_i = a_i e_0 and Kbar_j = b_j e_0, so S_ij = a_i b_j / sqrt(d).
    for d in (16, 64, 128):
        a = np.array([0.5, -1.0, 2.0])
        b = np.array([1.0, 0.25, -3.0, 0.0, 7.0])
        qbar = np.zeros((1, 1, 3, d)); qbar[0, 0, :, 0] = a
        kbar = np.zeros((1, 1, 5, d)); kbar[0, 0, :, 0] = b
        got = O.block_scores(qbar, kbar)[0, 0]
        want = scipy_softmax(np.outer(a, b) / math.sqrt(d), axis=1)
        np.testing.assert_allclose(got, want, rtol=1e-13, atol=0)


def test_block_scores_rows_are_distributions():
    rng = _rng(2)
    P = O.block_scores(rng.normal(size=(2, 3, 4, 64)) * 5, rng.normal(size=(2, 3, 9, 64)) * 5)
    assert np.all(P > 0)
    np.testing.assert_allclose(P.sum(-1), 1.0, rtol=0, atol=1e-12)
    # Order of P within a row equals the order of the raw dot products.
    qbar = rng.normal(size=(1, 1, 1, 8)); kbar = rng.normal(size=(1, 1, 20, 8))
    P = O.block_scores(qbar, kbar)[0, 0, 0]
    dots = kbar[0, 0] @ qbar[0, 0, 0]
    assert list(np.argsort(P)) == list(np.argsort(dots))


# ------------------------------------------------------------------------ top-k
def _brute_topk(row, k):
    """Max-sum subset of size k; among equal sums the lexicographically smallest index set."""
    best, best_set = None, None
    for sub in itertools.combinations(range(len(row)), k):  # lexicographic order
        s = sum(row[j] for j in sub)
        if best is None or s > best:
            best, best_set = s, sub
    return best_set


def test_topk_matches_brute_force_on_random_rows():
    rng = _rng(3)
    for trial in range(60):
        Kb = int(rng.integers(1, 11))
        k = int(rng.integers(1, Kb + 1))
        row = rng.random(Kb)
        got = np.flatnonzero(O.topk_mask(row[None, None, None], k)[0, 0, 0])
        assert tuple(got) == _brute_topk(list(row), k), (row, k)


def test_topk_ties_go_to_lower_index():
    row = np.array([0.1, 0.3, 0.2, 0.3, 0.3, 0.05])
    for k, want in [(1, [1]), (2, [1, 3]), (3, [1, 3, 4]), (4, [1, 2, 3, 4])]:
        got = np.flatnonzero(O.topk_mask(row[None, None, None], k)[0, 0, 0])
        assert list(got) == want
        assert tuple(got) == _brute_topk(list(row), k)
    # all equal: the first k
    got = np.flatnonzero(O.topk_mask(np.ones((1, 1, 1, 9)), 4)[0, 0, 0])
    assert list(got) == [0, 1, 2, 3]


def test_select_ties_from_duplicated_key_blocks():
    # Key blocks 1 and 3 are identical copies, so their scores tie exactly; with
    # k = 1 and block 1/3 the best, block 1 must win.
    rng = _rng(4)
    d, N = 8, 256
    q = np.tile(rng.normal(size=(1, d)), (N, 1))[None, None]
    k = rng.normal(size=(1, 1, N, d)) * 0.01
    best = q[0, 0, 0] * 3.0
    k[0, 0, 64:128] = best
    k[0, 0, 192:256] = best
    mask, P = O.select(q, k, 0.25)  # Kb = 4 -> k = 1
    assert P[0, 0, 0, 1] == P[0, 0, 0, 3]
    assert list(np.flatnonzero(mask[0, 0, 0])) == [1]
    mask, _ = O.select(q, k, 0.5)  # k = 2
    assert list(np.flatnonzero(mask[0, 0, 0])) == [1, 3]


def test_select_brute_force_pure_python():
    """Whole selection recomputed with Python loops and math.exp, then all subsets."""
    rng = _rng(5)
    B, H, N, d = 1, 2, 300, 4
    q = rng.normal(size=(B, H, N, d)); k = rng.normal(size=(B, H, N, d))
    for topk in (0.2, 0.5, 0.8, 1.0):
        mask, P = O.select(q, k, topk)
        Qb, Kb = 3, 5
        kk = max(1, min(Kb, math.ceil(float(np.float32(topk)) * Kb)))
        for h in range(H):
            means_q = []
            for i in range(Qb):
                rows = range(128 * i, min(N, 128 * i + 128))
                means_q.append([sum(q[0, h, r, c] for r in rows) / len(rows) for c in range(d)])
            means_k = []
            for j in range(Kb):
                rows = range(64 * j, min(N, 64 * j + 64))
                means_k.append([sum(k[0, h, r, c] for r in rows) / len(rows) for c in range(d)])
            for i in range(Qb):
                s = [sum(means_q[i][c] * means_k[j][c] for c in range(d)) / math.sqrt(d) for j in range(Kb)]
                z = sum(math.exp(x) for x in s)
                p = [math.exp(x) / z for x in s]
                np.testing.assert_allclose(P[0, h, i], p, rtol=1e-12)
                want = _brute_topk(p, kk)
                assert tuple(np.flatnonzero(mask[0, h, i])) == want


def test_tie_exempt_rows():
    P = np.array([[[[0.4, 0.3, 0.3]], [[0.5, 0.3, 0.2]], [[0.3, 0.3 * (1 - 1e-8), 0.4]]]])
    ex = O.tie_exempt_rows(P, 2)
    assert ex.tolist() == [[[True], [False], [True]]]
    assert not O.tie_exempt_rows(P, 3).any()


# -------------------------------------------------------------------- attention
def _sdpa(q, k, v, attn_mask=None):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    m = None if attn_mask is None else t(attn_mask)
    return torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=m).numpy()


def _expand(mask, N):
    return np.repeat(np.repeat(mask, 128, axis=2), 64, axis=3)[:, :, :N, :N].astype(bool)


@pytest.mark.parametrize("N,d", [(256, 64), (300, 64), (200, 128), (1, 64), (65, 128)])
def test_all_ones_mask_equals_library_sdpa(N, d):
    rng = _rng(6)
    q, k, v = (rng.normal(size=(2, 2, N, d)) for _ in range(3))
    Qb, Kb = O.block_counts(N)
    ones = np.ones((2, 2, Qb, Kb), dtype=np.uint8)
    want = _sdpa(q, k, v)
    np.testing.assert_allclose(O.block_sparse_attention(q, k, v, ones), want, rtol=0, atol=1e-12)
    np.testing.assert_allclose(O.dense_attention(q, k, v), want, rtol=0, atol=1e-12)
    out, mask = O.sparse_attention_topk(q, k, v, 1.0)  # topk = 1 keeps every block
    assert mask.all()
    np.testing.assert_allclose(out, want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("N", [384, 300, 129])
def test_block_mask_equals_sdpa_with_expanded_token_mask(N):
    rng = _rng(7)
    d = 32
    q, k, v = (rng.normal(size=(1, 3, N, d)) * 2 for _ in range(3))
    Qb, Kb = O.block_counts(N)
    mask = (rng.random((1, 3, Qb, Kb)) < 0.5).astype(np.uint8)
    mask[0, 0, 0] = 0  # one empty row
    mask[0, 1, -1] = 0
    mask[0, 1, -1, -1] = 1  # last query block keeps only the ragged last key block
    got = O.block_sparse_attention(q, k, v, mask)
    tok = _expand(mask, N)
    nonempty = tok.any(-1)
    want = _sdpa(q, k, v, attn_mask=tok)
    np.testing.assert_allclose(got[nonempty], want[nonempty], rtol=0, atol=1e-12)
    assert np.all(got[~nonempty] == 0.0)  # empty rows are defined as zero


def test_constant_v_gives_constant_output():
    rng = _rng(8)
    N, d = 300, 64
    q, k = rng.normal(size=(1, 2, N, d)) * 3, rng.normal(size=(1, 2, N, d)) * 3
    v = np.full((1, 2, N, d), -1.75)
    mask = (rng.random((1, 2, 3, 5)) < 0.6).astype(np.uint8)
    mask[0, 0, 1] = 0
    out = O.block_sparse_attention(q, k, v, mask)
    for h in range(2):
        for i in range(3):
            rows = out[0, h, 128 * i:min(N, 128 * i + 128)]
            if mask[0, h, i].any():
                np.testing.assert_allclose(rows, -1.75, rtol=0, atol=1e-12)
            else:
                assert np.all(rows == 0)


def test_single_kept_tile_is_softmax_over_its_keys():
    rng = _rng(9)
    N, d = 300, 16
    q, k, v = (rng.normal(size=(1, 1, N, d)) for _ in range(3))
    for j in range(5):
        mask = np.zeros((1, 1, 3, 5), dtype=np.uint8)
        mask[0, 0, :, j] = 1
        out = O.block_sparse_attention(q, k, v, mask)
        keys = slice(64 * j, min(N, 64 * j + 64))
        w = scipy_softmax(q[0, 0] @ k[0, 0, keys].T / math.sqrt(d), axis=1)
        np.testing.assert_allclose(out[0, 0], w @ v[0, 0, keys], rtol=0, atol=1e-12)


def test_permuting_keys_inside_a_kept_block_changes_nothing():
    rng = _rng(10)
    N, d = 256, 32
    q, k, v = (rng.normal(size=(1, 1, N, d)) for _ in range(3))
    mask = np.array([[[[1, 0, 1, 1], [0, 1, 1, 0]]]], dtype=np.uint8)
    base = O.block_sparse_attention(q, k, v, mask)
    perm = np.arange(N)
    perm[128:192] = 128 + rng.permutation(64)
    perm[0:64] = rng.permutation(64)
    out = O.block_sparse_attention(q, k[:, :, perm], v[:, :, perm], mask)
    np.testing.assert_allclose(out, base, rtol=0, atol=1e-12)
    # Moving a key into a dropped block does change the result.
    perm2 = np.arange(N); perm2[[0, 64]] = [64, 0]
    out2 = O.block_sparse_attention(q, k[:, :, perm2], v[:, :, perm2], mask)
    assert np.abs(out2 - base).max() > 1e-3


def test_topk_selection_keeps_highest_scoring_blocks_end_to_end():
    # A query field aligned with two specific key blocks: those must be kept.
    rng = _rng(11)
    N, d = 512, 16
    q = np.zeros((1, 1, N, d)); q[..., 0] = 1.0
    k = rng.normal(size=(1, 1, N, d)) * 0.1
    k[0, 0, 64 * 2:64 * 3, 0] += 5.0
    k[0, 0, 64 * 6:64 * 7, 0] += 4.0
    mask, P = O.select(q, k, 0.25)  # Kb = 8 -> k = 2
    for i in range(4):
        assert list(np.flatnonzero(mask[0, 0, i])) == [2, 6]


# ------------------------------------------------------- planted mistakes fail
def test_planted_mistakes_are_caught(monkeypatch):
    """Each plausible slip in the oracle must fail at least one pin above."""
    import oracle.bsa_oracle as mod

    def fails(fn):
        try:
            fn()
        except AssertionError:
            return True
        return False

    good_pool = mod.pool_mean

    def pool_full_divisor(x, block):  # divides a ragged block by the full size
        B, H, N, d = x.shape
        nb = -(-N // block)
        out = np.empty((B, H, nb, d))
        for i in range(nb):
            out[:, :, i] = x[:, :, i * block:(i + 1) * block].sum(axis=2) / block
        return out

    monkeypatch.setattr(mod, "pool_mean", pool_full_divisor)
    assert fails(lambda: test_pool_mean_closed_form_all_ragged_lengths(64))
    monkeypatch.setattr(mod, "pool_mean", good_pool)

    good_scores = mod.block_scores
    monkeypatch.setattr(mod, "block_scores", lambda a, b: good_scores(a * math.sqrt(a.shape[-1]), b))
    assert fails(test_block_scores_closed_form_and_scale)  # missing 1/sqrt(d)
    monkeypatch.setattr(mod, "block_scores", good_scores)

    good_topk = mod.topk_mask

    def topk_high_index_ties(P, k):
        Kb = P.shape[-1]
        rows = P.reshape(-1, Kb)
        m = np.zeros(rows.shape, np.uint8)
        for r in range(rows.shape[0]):
            order = np.lexsort((-np.arange(Kb), -rows[r]))
            m[r, order[:k]] = 1
        return m.reshape(P.shape)

    monkeypatch.setattr(mod, "topk_mask", topk_high_index_ties)
    assert fails(test_topk_ties_go_to_lower_index)
    monkeypatch.setattr(mod, "topk_mask", good_topk)

    good_rows = mod.attention_rows

    def rows_transposed_mask(qh, kh, vh, mask_row, i, causal=False):  # uses the complement of the mask
        return good_rows(qh, kh, vh, (np.asarray(mask_row) == 0).astype(np.uint8), i, causal)

    monkeypatch.setattr(mod, "attention_rows", rows_transposed_mask)
    assert fails(lambda: test_block_mask_equals_sdpa_with_expanded_token_mask(300))
    monkeypatch.setattr(mod, "attention_rows", good_rows)

    def rows_off_by_one_causal(qh, kh, vh, mask_row, i, causal=False):  # excludes the diagonal key
        if not causal:
            return good_rows(qh, kh, vh, mask_row, i)
        N, d = qh.shape
        lo, hi = i * 128, min((i + 1) * 128, N)
        cols = mod.kept_key_columns(mask_row, N)
        S = qh[lo:hi] @ kh[cols].T / math.sqrt(d)
        S = np.where(cols[None, :] < np.arange(lo, hi)[:, None], S, -np.inf)
        m = S.max(axis=1, keepdims=True)
        out = np.zeros((hi - lo, d))
        live = np.isfinite(m[:, 0])
        E = np.exp(S[live] - m[live])
        out[live] = (E @ vh[cols]) / E.sum(axis=1, keepdims=True)
        return out

    monkeypatch.setattr(mod, "attention_rows", rows_off_by_one_causal)
    assert fails(lambda: test_causal_all_ones_equals_library_causal_sdpa(300))
    monkeypatch.setattr(mod, "attention_rows", good_rows)


# ---------------------------------------------------------------- cdfthreshd
def _brute_cdf(row, tau):
    """Smallest subset reaching mass tau; among those the largest mass, then the
    lexicographically smallest index set."""
    n = len(row)
    for size in range(1, n + 1):
        best, best_set = None, None
        for sub in itertools.combinations(range(n), size):
            s = sum(row[j] for j in sub)
            if s >= tau and (best is None or s > best):
                best, best_set = s, sub
        if best_set is not None:
            return best_set
    return tuple(range(n))


def test_cdf_mask_matches_brute_force():
    rng = _rng(21)
    for trial in range(60):
        Kb = int(rng.integers(1, 10))
        row = rng.random(Kb) ** 3
        row = row / row.sum()
        tau = float(np.float32(rng.uniform(0.05, 0.999)))
        got = tuple(np.flatnonzero(O.cdf_mask(row[None, None, None], tau)[0, 0, 0]))
        assert got == _brute_cdf(list(row), tau), (row, tau)


def test_cdf_mask_closed_forms():
    # Values exactly representable in float32, so the float32 threshold equals its
    # decimal value.
    row = np.array([0.125, 0.375, 0.25, 0.25])[None, None, None]
    assert list(np.flatnonzero(O.cdf_mask(row, 0.375)[0, 0, 0])) == [1]        # 0.375 reaches 0.375
    assert list(np.flatnonzero(O.cdf_mask(row, 0.5)[0, 0, 0])) == [1, 2]       # 0.625, tie -> lower index
    assert list(np.flatnonzero(O.cdf_mask(row, 0.625)[0, 0, 0])) == [1, 2]
    assert list(np.flatnonzero(O.cdf_mask(row, 0.75)[0, 0, 0])) == [1, 2, 3]   # 0.875
    assert O.cdf_mask(row, 1.0)[0, 0, 0].sum() == 4
    assert O.cdf_mask(row, 1e-6)[0, 0, 0].sum() == 1                           # at least one
    # the threshold is read as float32: 0.4f > 0.4, so 0.4 alone no longer reaches it
    row2 = np.array([0.1, 0.4, 0.2, 0.3])[None, None, None]
    assert list(np.flatnonzero(O.cdf_mask(row2, 0.4)[0, 0, 0])) == [1, 3]


def test_cdf_exempt_rows_flags_boundaries():
    P = np.array([[[[0.5, 0.3, 0.2]], [[0.5, 0.25, 0.25 * (1 - 1e-9)]]]])
    assert O.cdf_exempt_rows(P, 0.8)[0, 0, 0]       # 0.5 + 0.3 sits on the threshold
    assert O.cdf_exempt_rows(P, 0.7)[0, 1, 0]       # kept and first dropped score tie
    assert not O.cdf_exempt_rows(P, 0.6)[0, 0, 0]


# -------------------------------------------------------------------- causal
def test_causal_block_limit_hand_worked():
    # query block i covers rows 128i..128i+127, so key blocks 0..2i+1 hold earlier keys
    assert [O.causal_block_limit(i, 100) for i in range(4)] == [2, 4, 6, 8]
    assert O.causal_block_limit(3, 5) == 5


@pytest.mark.parametrize("N", [256, 300, 129, 1])
def test_causal_all_ones_equals_library_causal_sdpa(N):
    rng = _rng(31)
    q, k, v = (rng.normal(size=(1, 2, N, 32)) for _ in range(3))
    Qb, Kb = O.block_counts(N)
    ones = np.ones((1, 2, Qb, Kb), dtype=np.uint8)
    want = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), is_causal=True).numpy()
    np.testing.assert_allclose(O.block_sparse_attention(q, k, v, ones, causal=True), want, rtol=0, atol=1e-12)


def test_causal_block_mask_equals_sdpa_with_combined_mask():
    rng = _rng(32)
    N = 400
    q, k, v = (rng.normal(size=(1, 3, N, 16)) * 2 for _ in range(3))
    Qb, Kb = O.block_counts(N)
    mask = (rng.random((1, 3, Qb, Kb)) < 0.5).astype(np.uint8)
    mask[0, 0, 1] = 0
    mask[0, 0, 1, 3] = 1          # only the second diagonal block: rows 128..191 see nothing
    got = O.block_sparse_attention(q, k, v, mask, causal=True)
    tok = _expand(mask, N) & np.tril(np.ones((N, N), dtype=bool))[None, None]
    live = tok.any(-1)
    want = _sdpa(q, k, v, attn_mask=tok)
    np.testing.assert_allclose(got[live], want[live], rtol=0, atol=1e-12)
    assert np.all(got[~live] == 0.0) and (~live).sum() >= 64


def test_causal_topk_matches_brute_force_over_eligible_blocks():
    rng = _rng(33)
    for trial in range(20):
        Qb = 3
        Kb = int(rng.integers(2, 7))
        P = rng.random((1, 1, Qb, Kb))
        topk = float(rng.uniform(0.05, 1.0))
        m = O.causal_topk_mask(P, topk)
        for i in range(Qb):
            E = O.causal_block_limit(i, Kb)
            kk = O.keep_count(topk, E)
            assert m[0, 0, i, E:].sum() == 0
            assert tuple(np.flatnonzero(m[0, 0, i])) == _brute_topk(list(P[0, 0, i, :E]), kk)


# --------------------------------------------------------- token reordering
def test_token_permutations_hand_worked():
    # 1 x 2 x 8 grid, no text: cubes of 4 x 4 x 4 clip to 1 x 2 x 4, so the cube
    # order takes columns 0-3 of both rows, then columns 4-7 of both rows.
    p = O.token_permutation(1, 2, 8, 0, "cube")
    assert list(p) == [0, 1, 2, 3, 8, 9, 10, 11, 4, 5, 6, 7, 12, 13, 14, 15]
    # Morton on a 1 x 2 x 4 grid: key interleaves (h, w) bits -> (0,0)(0,1)(1,0)(1,1)(0,2)(0,3)(1,2)(1,3)
    p = O.token_permutation(1, 2, 4, 0, "morton")
    assert list(p) == [0, 1, 4, 5, 2, 3, 6, 7]
    p = O.token_permutation(2, 3, 5, 4, "raster")
    assert list(p) == list(range(34))


@pytest.mark.parametrize("mode", ["cube", "morton"])
def test_token_permutation_is_a_bijection_keeping_text_first(mode):
    for T, Hg, Wg, text in [(21, 45, 80, 0), (13, 30, 45, 226), (1, 1, 7, 3), (5, 9, 6, 0)]:
        p = O.token_permutation(T, Hg, Wg, text, mode)
        assert sorted(p.tolist()) == list(range(text + T * Hg * Wg))
        assert list(p[:text]) == list(range(text))


def test_cube_blocks_are_spatially_compact():
    # every aligned run of 64 tokens inside full cubes spans a 4 x 4 x 4 box
    T, Hg, Wg = 8, 8, 8
    p = O.token_permutation(T, Hg, Wg, 0, "cube")
    for s0 in range(0, T * Hg * Wg, 64):
        m = p[s0:s0 + 64]
        t, h, w = m // 64, (m // 8) % 8, m % 8
        assert np.ptp(t) == 3 and np.ptp(h) == 3 and np.ptp(w) == 3


def test_kept_mass_is_one_for_dense_and_below_one_for_sparse():
    rng = _rng(41)
    q, k = rng.normal(size=(1, 1, 300, 16)) * 2, rng.normal(size=(1, 1, 300, 16)) * 2
    ones = np.ones((1, 1, 3, 5), np.uint8)
    np.testing.assert_allclose(O.kept_mass(q, k, ones, 0, 0, [0, 2]), 1.0, atol=1e-12)
    half = ones.copy(); half[..., 1::2] = 0
    km = O.kept_mass(q, k, half, 0, 0, [0, 1, 2])
    assert np.all(km < 1) and np.all(km > 0)


def test_kept_mass_hand_worked():
    """d = 1 and N = 130 (query blocks of 128 and 2 rows; key blocks of 64, 64 and 2
    keys).  k is ln 3 on keys 0-63, 0 on keys 64-127 and ln 5 on keys 128-129, so a
    row with q = 1 gives each key weight 3, 1 or 5 (total 64*3 + 64*1 + 2*5 = 266)
    and a row with q = 2 weights 9, 1 or 25 (total 576 + 64 + 50 = 690)."""
    N = 130
    k = np.zeros((1, 1, N, 1))
    k[0, 0, :64, 0] = math.log(3.0)
    k[0, 0, 128:, 0] = math.log(5.0)
    q = np.ones((1, 1, N, 1))
    q[0, 0, 128:, 0] = 2.0
    mask = np.array([[[[1, 0, 1], [1, 1, 0]]]], dtype=np.uint8)
    km = O.kept_mass(q, k, mask, 0, 0, [0, 1])
    assert km.shape == (130,)
    np.testing.assert_allclose(km[:128], 202.0 / 266.0, rtol=1e-13)
    np.testing.assert_allclose(km[128:], 640.0 / 690.0, rtol=1e-13)
    # the listed blocks select the rows: block 1 alone gives its two rows only
    np.testing.assert_allclose(O.kept_mass(q, k, mask, 0, 0, [1]), 640.0 / 690.0, rtol=1e-13)
    # and the mask row of each block is its own
    swapped = mask[:, :, ::-1].copy()
    np.testing.assert_allclose(O.kept_mass(q, k, swapped, 0, 0, [0])[0], 256.0 / 266.0, rtol=1e-13)
