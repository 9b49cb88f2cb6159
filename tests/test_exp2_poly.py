"""The attention kernel's software exp2 (Cody-Waite split + Remez polynomial),
emulated step by step in float32 with the coefficients read from the CUDA
header, against numpy's exp2 over the range the softmax feeds it.  No GPU."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _coeffs():
    src = open(os.path.join(ROOT, "block_sparse_attention_14_b200", "csrc", "bsa_common.cuh")).read()
    body = src[src.index("uint64_t exp2_poly2("):]
    body = body[:body.index("\n}\n")]
    c = [float(x) for x in re.findall(r"f2_pack\(([-+0-9.e]+)f,", body)]
    # order in the source: shifter, -shifter, -1 (x - n), then c4, c3, c2, c1, c0
    return [np.float32(v) for v in c[3:]]


def _exp2_poly_f32(x):
    c4, c3, c2, c1, c0 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    n = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = (c4 * f + c3).astype(np.float32)
    p = (p * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_coefficients_are_parsed():
    c = _coeffs()
    assert len(c) == 5 and abs(float(c[-1]) - 1.0) < 1e-5 and abs(float(c[-2]) - np.log(2)) < 1e-3


def test_relative_error_over_softmax_range():
    x = np.concatenate([np.linspace(-126.0, 8.0, 2_000_001, dtype=np.float32),
                        np.float32(np.arange(-126, 9))])  # exact integers
    got = _exp2_poly_f32(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 3e-6, rel.max()


def test_clamps_below_minus_126_and_minus_inf():
    x = np.array([-np.inf, -1000.0, -127.5, -126.0], dtype=np.float32)
    got = _exp2_poly_f32(x)
    assert np.all(np.isfinite(got)) and np.all(got > 0) and np.all(got < 1.2e-38)


def test_fit_script_reproduces_the_coefficients():
    import importlib.util

    spec = importlib.util.spec_from_file_location(
        "fit", os.path.join(ROOT, "block_sparse_attention_14_b200", "csrc", "exp2_poly_fit.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    c, err = m.remez_rel(4)
    assert err < 3e-6
    np.testing.assert_allclose(np.float32(c[::-1]), _coeffs(), rtol=1e-6)
