"""The parity harness itself (tests/_parity.py), on CPU.

The GPU tests trust these helpers to measure errors and to apply the stated
and derived tolerances, so they are checked here by hand cases; the derived
lse bound is checked both ways: fp32 arithmetic of the kind the kernels do
stays inside it, and plausible mistakes fall far outside it.
"""

import math

import numpy as np
import pytest

from _parity import BF16_O, assert_close, assert_lse_close, errors, lse_tolerance


def test_error_metrics_by_hand():
    ma, rf = errors([1.0, 2.0, 2.0], [1.0, 0.0, 0.0])
    assert ma == 2.0
    assert rf == pytest.approx(math.sqrt(8.0) / 1.0)
    ma, rf = errors([3.0, 4.0], [0.0, 0.0])     # zero reference: the plain norm of the difference
    assert (ma, rf) == (4.0, 5.0)
    assert errors(np.zeros((0, 3)), np.zeros((0, 3))) == (0.0, 0.0)
    with pytest.raises(AssertionError):
        errors([1.0], [1.0, 2.0])


def test_assert_close_applies_both_bounds():
    ref = np.ones(100)
    assert_close(ref + 0.004, ref, *BF16_O)                      # inside both
    with pytest.raises(AssertionError):
        assert_close(ref + 0.021, ref, *BF16_O)                  # max-abs exceeded
    g = ref.copy()
    g[:50] += 0.015                                               # max-abs fine, rel-Frob 1.06e-2 > 5e-3
    with pytest.raises(AssertionError):
        assert_close(g, ref, *BF16_O)
    with pytest.raises(AssertionError):
        assert_close(np.array([np.nan, 1.0]), np.array([1.0, 1.0]), 1.0)


def test_large_output_widening():
    ref = np.array([32.0, 1.0])
    # max|ref| = 32: the absolute bound 2e-2 scales to 2e-2 * 32 / 4 = 0.16, on every element
    assert_close(ref + np.array([0.15, 0.0]), ref, 2e-2, large_outputs=True)
    assert_close(ref + np.array([0.0, 0.15]), ref, 2e-2, large_outputs=True)
    with pytest.raises(AssertionError):
        assert_close(ref + np.array([0.1, 0.0]), ref, 2e-2)
    with pytest.raises(AssertionError):
        assert_close(ref + np.array([0.17, 0.0]), ref, 2e-2, large_outputs=True)
    # the relative Frobenius bound is not widened
    with pytest.raises(AssertionError):
        assert_close(ref + np.array([0.15, 0.15]), ref, 2e-2, 1e-3, large_outputs=True)


def test_large_output_flag_refused_on_order_one_reference():
    ref = np.array([3.9, -1.0])
    with pytest.raises(AssertionError, match="order-one"):
        assert_close(ref, ref, 2e-2, large_outputs=True)


def _lse_fp32(q, k, scale):
    """lse as fp32 kernels form it: fp32 dot products accumulated over d in
    order, the maximum, fp32 exponentials summed key by key, m + ln l."""
    q32, k32 = q.astype(np.float32), k.astype(np.float32)
    s = np.zeros((q.shape[0], k.shape[0]), dtype=np.float32)
    for d in range(q.shape[1]):
        s = s + np.outer(q32[:, d], k32[:, d]).astype(np.float32)
    s = (s * np.float32(scale)).astype(np.float32)
    m = s.max(axis=1)
    l = np.zeros(q.shape[0], dtype=np.float32)
    for j in range(k.shape[0]):
        l = (l + np.exp(s[:, j] - m).astype(np.float32)).astype(np.float32)
    return (m + np.log(l)).astype(np.float32).astype(np.float64)


def _lse64(q, k, scale):
    s = scale * (q @ k.T)
    m = s.max(axis=1)
    return m + np.log(np.exp(s - m[:, None]).sum(axis=1))


@pytest.mark.parametrize("mult,Nk,D", [(1.0, 700, 64), (40.0, 512, 64), (1.0, 300, 128)])
def test_lse_bound_covers_fp32_arithmetic(mult, Nk, D):
    rng = np.random.default_rng(Nk + D)
    q = (rng.standard_normal((6, D)) * mult).astype(np.float32).astype(np.float64)
    k = (rng.standard_normal((Nk, D)) * mult).astype(np.float32).astype(np.float64)
    scale = 1.0 / math.sqrt(D)
    ref = _lse64(q, k, scale)
    assert_lse_close(_lse_fp32(q, k, scale), ref, q, k, scale)


def test_lse_bound_catches_plausible_mistakes():
    rng = np.random.default_rng(5)
    q = rng.standard_normal((6, 64))
    k = rng.standard_normal((400, 64))
    scale = 0.125
    ref = _lse64(q, k, scale)
    tol = lse_tolerance(q, k, scale, ref)
    assert np.all(tol < 2e-3)
    with pytest.raises(AssertionError):
        assert_lse_close(ref / math.log(2.0), ref, q, k, scale)          # base-2 lse
    with pytest.raises(AssertionError):
        assert_lse_close(_lse64(q, k, 1.0), ref, q, k, scale)            # scale not applied
    with pytest.raises(AssertionError):
        assert_lse_close(ref - np.log(400.0), ref, q, k, scale)          # mean instead of sum
