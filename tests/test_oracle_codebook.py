"""Pins for the NF4 codebook.

Pages: automatone "QLoRA paper explained", paragraph "4-bit NormalFloat (NF4)"
(levels at the quantiles of a standard normal); creativeworksofknowledge
"QLoRA: Fine-Tune 70B on One GPU", section "1. NF4 (NormalFloat4)
quantization" (levels allocated in proportion to the Gaussian, denser near
zero).  Exact zero and monotone levels are fixed by the hot path's statement.
The closed-form check uses scipy's ndtri / ndtr, an independent routine from
the oracle's erfc bisection.
"""
import numpy as np
from scipy.special import ndtr, ndtri

import oracle


def test_codebook_shape_and_invariants(L):
    assert L.dtype == np.float32 and L.shape == (16,)
    assert np.all(np.diff(L) > 0), "levels must be strictly increasing"
    assert L[0] == -1.0 and L[15] == 1.0
    assert L[7] == 0.0 and np.count_nonzero(L == 0.0) == 1
    assert np.count_nonzero(L < 0) == 7 and np.count_nonzero(L > 0) == 8


def test_normal_quantile_matches_scipy():
    for p in [0.5, 0.51, 0.6, 0.75, 0.9, 0.95, 0.9677083333333334, 0.99, 0.001, 0.3]:
        assert abs(oracle.normal_quantile(p) - ndtri(p)) <= 4e-15 * max(1.0, abs(ndtri(p)))


def test_codebook_equals_closed_form_quantiles(L):
    delta = 1.0 - 0.5 * (1.0 / 30.0 + 1.0 / 32.0)
    assert oracle.default_delta() == delta
    top = ndtri(delta)
    pos = [ndtri(0.5 + (delta - 0.5) * j / 8.0) / top for j in range(1, 9)]
    neg = [-ndtri(0.5 + (delta - 0.5) * j / 7.0) / top for j in range(1, 8)]
    ref = np.array(sorted(neg) + [0.0] + pos, dtype=np.float64)
    # one float rounding of the double value: the two routines agree to a few 1e-16,
    # far inside half a float ulp, so the rounded tables are identical
    assert np.array_equal(ref.astype(np.float32), L)


def test_levels_split_the_normal_into_equal_mass_steps(L):
    # the levels are quantiles: on each side the normal mass between neighbours is constant
    delta = oracle.default_delta()
    top = ndtri(delta)
    pos_cdf = ndtr(L[7:].astype(np.float64) * top)      # 0, v1..v8
    neg_cdf = ndtr(-L[:8][::-1].astype(np.float64) * top)   # 0, w1..w7 mirrored
    dpos, dneg = np.diff(pos_cdf), np.diff(neg_cdf)
    assert np.allclose(dpos, (delta - 0.5) / 8, atol=1e-7)
    assert np.allclose(dneg, (delta - 0.5) / 7, atol=1e-7)


def test_levels_denser_near_zero(L):
    gaps = np.diff(L.astype(np.float64))
    # gaps shrink toward the zero level on both sides (Gaussian allocation)
    assert np.all(np.diff(gaps[:7]) < 0)
    assert np.all(np.diff(gaps[7:]) > 0)
