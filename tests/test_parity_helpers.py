"""The parity helpers the GPU tests rely on, on CPU: a mask that differs from the
oracle's only inside the tie band is accepted (and counted); one that differs
outside it, keeps the wrong count, keeps a block outside the band, or differs on
too many rows is rejected.  The same for causal rows and cdfthreshd prefixes."""
import numpy as np
import pytest

from oracle import bsa_oracle as O
from tests import parity as P


def _rows(n, Kb, seed):
    rng = np.random.default_rng(seed)
    S = rng.normal(size=(1, 1, n, Kb))
    E = np.exp(S)
    return E / E.sum(-1, keepdims=True)


def test_topk_mask_tie_band():
    Pr = _rows(20, 16, 0)
    k = 4  # topk 0.25 of 16 key blocks
    # row 3: make the 4th and 5th largest equal to within 1e-9 relative
    order = np.argsort(-Pr[0, 0, 3])
    Pr[0, 0, 3, order[4]] = Pr[0, 0, 3, order[3]] * (1 - 1e-9)
    mref = O.topk_mask(Pr, k)
    mg = mref.copy()
    mg[0, 0, 3, order[3]], mg[0, 0, 3, order[4]] = 0, 1  # the other member of the tie
    mc = P.check_topk_mask(mg, mref, Pr, 0.25)
    assert (mc.differing, mc.rows) == (1, 20) and mc.exempt >= 1
    assert P.differing_blocks(mc, mref, 0, 0) == [3]
    # the same swap on a row without a tie fails
    bad = mref.copy()
    o5 = np.argsort(-Pr[0, 0, 5])
    bad[0, 0, 5, o5[3]], bad[0, 0, 5, o5[4]] = 0, 1
    with pytest.raises(AssertionError):
        P.check_topk_mask(bad, mref, Pr, 0.25)
    # a row keeping one block too many fails
    extra = mref.copy()
    extra[0, 0, 7, np.argsort(-Pr[0, 0, 7])[k]] = 1
    with pytest.raises(AssertionError):
        P.check_topk_mask(extra, mref, Pr, 0.25)
    # a tie row that swaps in a block far outside the band fails
    far = mref.copy()
    far[0, 0, 3, order[3]], far[0, 0, 3, order[-1]] = 0, 1
    with pytest.raises(AssertionError):
        P.check_topk_mask(far, mref, Pr, 0.25)


def test_differing_rows_are_bounded():
    n, Kb, k = 40, 8, 2
    Pr = np.full((1, 1, n, Kb), 1.0 / Kb)  # every row a full tie
    mref = O.topk_mask(Pr, k)
    mg = mref.copy()
    mg[0, 0, :3] = 0
    mg[0, 0, :3, -k:] = 1  # three rows differ, all in the tie band
    with pytest.raises(AssertionError, match="allowed 2"):
        P.check_topk_mask(mg, mref, Pr, k / Kb)
    mg[0, 0, 2] = mref[0, 0, 2]
    assert P.check_topk_mask(mg, mref, Pr, k / Kb).differing == 2


def test_causal_rows_keep_only_eligible_blocks():
    Pr = _rows(4, 8, 1)
    mref = O.causal_topk_mask(Pr, 0.5)
    assert P.check_topk_mask(mref, mref, Pr, 0.5, causal=True).differing == 0
    bad = mref.copy()
    bad[0, 0, 0, 5] = 1  # query block 0 may use key blocks 0 and 1 only
    bad[0, 0, 0, np.flatnonzero(bad[0, 0, 0, :2])[0]] = 0
    with pytest.raises(AssertionError):
        P.check_topk_mask(bad, mref, Pr, 0.5, causal=True)


def test_cdf_prefix_rules():
    Pr = np.array([[[[0.5, 0.3, 0.15, 0.05]]]])
    tau = 0.79995
    mref = O.cdf_mask(Pr, tau)                # keeps 0, 1 (0.8 reaches tau)
    assert mref[0, 0, 0].tolist() == [1, 1, 0, 0]
    assert O.cdf_exempt_rows(Pr, tau)[0, 0, 0]  # 0.8 lies within 1e-4 of tau: an exempt row
    longer = mref.copy(); longer[0, 0, 0, 2] = 1  # one block more: still at the threshold
    bad, ex, diff = P.compare_cdf_masks(longer, mref, Pr, tau)
    assert (bad, diff) == (0, 1)
    gap = mref.copy(); gap[0, 0, 0] = [1, 0, 1, 0]  # not a prefix of the score order
    with pytest.raises(AssertionError):
        P.compare_cdf_masks(gap, mref, Pr, tau)
    far = mref.copy(); far[0, 0, 0] = [1, 1, 1, 1]  # runs past the threshold
    with pytest.raises(AssertionError):
        P.compare_cdf_masks(far, mref, Pr, tau)
