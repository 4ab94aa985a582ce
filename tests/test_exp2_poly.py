"""The prefill kernel computes one weight pair in eight as 2^y on the FMA pipe
(prefill.cu, exp2_poly2): Cody-Waite range reduction, a polynomial fit of 2^f
on |f| <= 1/2, and the integer part added to the exponent field.  These tests
pin the coefficients in the kernel source to the fitting script beside it,
and the whole float32 evaluation, step by step as the kernel does it, to
exp2 within the fit's error bound."""
import importlib.util
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "paged_kv_cache_419_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("exp2_poly_fit", os.path.join(CSRC, "exp2_poly_fit.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def kernel_coefficients(degree: int) -> np.ndarray:
    text = open(os.path.join(CSRC, "prefill.cu")).read()
    m = re.search(r"kExp2Deg%d\[%d\]\s*=\s*\{([^}]*)\}" % (degree, degree + 1), text)
    assert m, f"kExp2Deg{degree} not found"
    return np.array([float(x.strip().rstrip("f")) for x in m.group(1).split(",")], dtype=np.float32)


def fma32(a, b, c):
    """float32 fused multiply-add: the float64 product of two float32 values is
    exact, so one rounding of a * b + c to float64 and then to float32 differs
    from a true fused operation only in double-rounding ties."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly_like_kernel(y: np.ndarray, coeffs: np.ndarray) -> np.ndarray:
    y = np.maximum(y.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)                     # 1.5 * 2^23: y + magic rounds y to an integer
    t = (y + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    f = fma32(j, np.full_like(j, -1.0), y)             # y - j, exact
    p = np.full_like(f, coeffs[-1])
    for c in coeffs[-2::-1]:
        p = fma32(p, f, np.full_like(f, c))
    bits = p.view(np.int32) + (t.view(np.int32) << np.int32(23))
    return bits.view(np.float32)


@pytest.mark.parametrize("degree", [3, 4])
def test_kernel_coefficients_are_the_fit(degree):
    c_fit, _ = _fit_module().fit(degree)
    c_src = kernel_coefficients(degree)
    assert c_src.shape == c_fit.shape
    np.testing.assert_allclose(c_src, c_fit, rtol=0, atol=1e-6)


@pytest.mark.parametrize("degree,bound", [(3, 2.0 ** -13.6), (4, 2.0 ** -18.4)])
def test_polynomial_error_bound(degree, bound):
    """Relative error of p(f) against 2^f on |f| <= 1/2, with the source's
    float32 coefficients: the fit's equal-ripple bound."""
    c = kernel_coefficients(degree).astype(np.float64)
    f = np.linspace(-0.5, 0.5, 400001)
    p = np.polyval(c[::-1], f)
    err = np.abs(p / np.exp2(f) - 1.0)
    assert err.max() < bound
    # equal ripple: the error comes within 10 % of its peak at both ends and inside
    assert err[0] > 0.9 * err.max() and err[-1] > 0.9 * err.max()


@pytest.mark.parametrize("degree,bound", [(3, 2.0 ** -13.6), (4, 2.0 ** -18.4)])
def test_emulated_exp2_matches_exp2(degree, bound):
    """The float32 evaluation as the kernel does it, over every exponent the
    kernel's weights can have (y <= 8 + the lag of the running max) and down to
    the clamp at -125: relative error within the polynomial's bound plus a few float32
    roundings."""
    rng = np.random.default_rng(7)
    y = np.concatenate([np.linspace(-125.0, 12.0, 1_000_001), rng.uniform(-125.0, 12.0, 200_000),
                        np.arange(-125, 13, dtype=np.float64), np.arange(-125, 12) + 0.5]).astype(np.float32)
    got = exp2_poly_like_kernel(y, kernel_coefficients(degree)).astype(np.float64)
    want = np.exp2(y.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < bound + 8 * 2.0 ** -24


def test_emulated_exp2_clamps_tiny_and_masked_inputs():
    """Inputs below -125, -inf included (a masked key's score), give the clamped
    weight ~2^-125: positive, normal and negligible against a row's largest
    weight (at least 1); the kernel zeroes masked keys by a select after it."""
    c = kernel_coefficients(3)
    y = np.array([-np.inf, -1e30, -300.0, -127.0, -126.0, -125.0], dtype=np.float32)
    got = exp2_poly_like_kernel(y, c).astype(np.float64)
    assert np.all(np.abs(got / 2.0 ** -125 - 1.0) < 2.0 ** -13.6)
    assert np.all(got >= np.finfo(np.float32).tiny)     # normal, not a subnormal encoding
