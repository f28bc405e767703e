"""The forward kernel's FMA-pipe exp2 (exp2_poly2 in fm_common.cuh): its
coefficients are the ones the committed Remez fit produces, and its fp32
evaluation (argument reduction by the 1.5*2^23 rounding constant, Horner
steps, exponent-field scaling), mirrored here in numpy fp32, stays within the
polynomial's error bound of the true 2^x over the range the softmax uses."""
import os
import re

import numpy as np

from mask_aware_flash_b200 import exp2_poly

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_coeffs():
    src = open(os.path.join(ROOT, "mask_aware_flash_b200", "csrc", "fm_common.cuh")).read()
    return [float(re.search(rf"kExp2C{k} = ([0-9.e+-]+)f", src).group(1)) for k in range(4)]


def test_coefficients_match_remez_fit():
    coef, err = exp2_poly.remez_exp2(3)
    assert err < 8e-5
    np.testing.assert_allclose(_header_coeffs(), exp2_poly.as_f32(coef), rtol=2e-7)


def _emulate(x):
    f32 = np.float32
    c0, c1, c2, c3 = (f32(v) for v in _header_coeffs())
    xc = np.maximum(x.astype(f32), f32(-125.0))
    t = (xc + f32(12582912.0)).astype(f32)
    r = (t - f32(12582912.0)).astype(f32)
    fr = (xc - r).astype(f32)
    q = (fr * c3 + c2).astype(f32)
    q = (q * fr + c1).astype(f32)
    q = (q * fr + c0).astype(f32)
    bits = q.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32)


def test_fp32_evaluation_error_bound():
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float64),
                        np.arange(-125, 9, dtype=np.float64) + 0.5]).astype(np.float32)
    got = _emulate(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 1e-4, rel.max()


def test_masked_scores_become_negligible():
    got = _emulate(np.array([-np.inf, -1e30, -200.0, -125.0], dtype=np.float32))
    assert np.all(got > 0) and np.all(got < 1e-37)
