"""Shared parity helpers: error metrics and the tolerances the tests enforce.

Tolerances
----------
* bf16 paths: O within max-abs 2e-2 and relative Frobenius 5e-3 of the fp64
  oracle; dQ, dK, dV within max-abs 3e-2 and relative Frobenius 1e-2.
* fp32 path: O within max-abs 1e-4.
* The stated absolute bounds presume outputs of order one (N(0,1) inputs,
  |ref| <= ORDER_ONE = 4), and every order-one tensor is held to them.  Only a
  construction that makes a tensor large -- few keys shared by many query
  rows, so that dV and dK sum many rows (a single key: dV_0 = sum_i dO_i,
  |dV| ~ 30-80) -- may pass ``large_outputs=True``.  The helper then asserts
  that the reference really exceeds ORDER_ONE, and scales the absolute bound
  of that tensor by max|ref| / ORDER_ONE: the rounding errors of these sums
  (bf16 P and dS, half an ulp of bf16 being 2^-9 relative) grow with the
  magnitude of the summed terms, which is that of the largest outputs, and
  half an ulp of a bf16 value of 8 (2^-5) already exceeds 3e-2.  The relative
  Frobenius bound is never widened.
* lse (no tolerance is stated for it; derived from the arithmetic): the
  kernels evaluate lse_i = m_i + ln l_i in fp32 from scores s_ij = scale * q_i.k_j
  accumulated in fp32 and from Nk exponentials summed in fp32.  The error is
  bounded by the dot-product error scale * gamma_D * max_j sum_d |q_id k_jd|
  (gamma_D = D u / (1 - D u), u = 2^-24), plus the relative error of the exp-sum
  (< (Nk + 16) u for sequential fp32 summation with approximate exp2 of
  relative error < 2^-21), plus two roundings of |lse| itself (2 u |lse|), plus
  1e-4 absolute slack for the log evaluation.
"""

from __future__ import annotations

import numpy as np
import torch

U32 = 2.0 ** -24

BF16_O = (2e-2, 5e-3)
BF16_GRAD = (3e-2, 1e-2)
F32_O_MAX_ABS = 1e-4
ORDER_ONE = 4.0


def errors(gpu, ref):
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    if g.size == 0:
        return 0.0, 0.0
    diff = g - r
    max_abs = float(np.abs(diff).max())
    nr = float(np.linalg.norm(r))
    rel = float(np.linalg.norm(diff) / nr) if nr > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def assert_close(gpu, ref, max_abs_tol, rel_tol=None, what="", large_outputs=False):
    ma, rf = errors(gpu, ref)
    g = np.asarray(gpu, dtype=np.float64)
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    if large_outputs:
        top = float(np.abs(np.asarray(ref, dtype=np.float64)).max())
        assert top > ORDER_ONE, f"{what}: large_outputs given for an order-one reference (max |ref| {top:.2f})"
        bound = max_abs_tol * top / ORDER_ONE
        assert ma <= bound, f"{what}: max-abs {ma:.3e} > {bound:.3e} ({max_abs_tol:.1e} x max|ref| {top:.1f} / " \
                            f"{ORDER_ONE}) (rel-Frob {rf:.3e})"
    else:
        assert ma <= max_abs_tol, f"{what}: max-abs {ma:.3e} > {max_abs_tol:.1e} (rel-Frob {rf:.3e})"
    if rel_tol is not None:
        assert rf <= rel_tol, f"{what}: rel-Frob {rf:.3e} > {rel_tol:.1e} (max-abs {ma:.3e})"
    return ma, rf


def lse_tolerance(q64, k64, scale, lse_ref):
    """Per-row lse bound (see module docstring); q64 [..., Nq, D], k64 [..., Nk, D]."""
    D = q64.shape[-1]
    Nk = k64.shape[-2]
    gamma = D * U32 / (1 - D * U32)
    absdot = np.abs(q64) @ np.abs(np.swapaxes(k64, -1, -2))  # [..., Nq, Nk]
    dot_err = abs(scale) * gamma * absdot.max(axis=-1)
    sum_err = (Nk + 16) * U32 * 2.0
    return 1e-4 + dot_err + sum_err + 2 * U32 * np.abs(lse_ref)


def assert_lse_close(gpu_lse, ref_lse, q64, k64, scale, what="lse"):
    tol = lse_tolerance(q64, k64, scale, ref_lse)
    err = np.abs(np.asarray(gpu_lse, dtype=np.float64) - ref_lse)
    assert np.isfinite(err).all(), f"{what}: non-finite"
    bad = err > tol
    assert not bad.any(), f"{what}: {bad.sum()} rows exceed the derived bound; worst err {err.max():.3e}, " \
                          f"tol there {tol.reshape(-1)[np.argmax(err)]:.3e}"
    return float(err.max())


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy()
