"""The FMA-pipe base-2 exponential of the split-ex2 soft kernel (ex2_fma in
bcjr_l16.cuh), pinned on the CPU: its polynomial is the one ex2_poly.py fits,
and the whole device formula (range reduction through 1.5 * 2^23, degree-5
Horner in fp32 fused multiply-adds, exponent-field scaling), emulated bit for
bit in NumPy, stays within 2.5e-7 relative of 2^x over the range the kernel
uses (ex2.approx, which it replaces, is specified to 2 ulp = 2.4e-7)."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "bcjr_sum_product_b200", "csrc")


def _poly_module():
    spec = importlib.util.spec_from_file_location("ex2_poly", os.path.join(CSRC, "ex2_poly.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _kernel_coefficients():
    src = open(os.path.join(CSRC, "bcjr_l16.cuh")).read()
    body = src[src.index("float ex2_fma(float x)"):]
    body = body[:body.index("\n}\n")]
    return [float(x) for x in re.findall(r"([0-9]+\.[0-9]+)f", body) if float(x) < 2.0 and float(x) != 1.5]


def _ex2_fma(x):
    """The device formula on float32 arrays, rounding as the GPU does."""
    f32 = np.float32
    x = np.minimum(np.maximum(x.astype(f32), f32(-126.0)), f32(127.0))
    t = (x + f32(12582912.0)).astype(f32)
    f = (x - (t - f32(12582912.0)).astype(f32)).astype(f32)
    c = [f32(v) for v in _kernel_coefficients()]
    p = np.full_like(f, c[0])
    for ci in c[1:]:
        p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(ci)).astype(f32)   # one fused rounding
    n = (t.view(np.int32) - np.int32(0x4B400000)).astype(np.uint32)
    return (p.view(np.uint32) + (n << np.uint32(23))).view(f32)


def test_kernel_uses_the_fitted_polynomial():
    m = _poly_module()
    fitted = m.fit().astype(np.float32)
    used = np.array(_kernel_coefficients(), np.float32)
    assert len(used) == m.DEGREE + 1
    np.testing.assert_array_equal(used, fitted)
    assert m.max_rel_error(m.fit()) < 2.5e-7


def test_device_formula_relative_error():
    x = np.concatenate([np.linspace(-126.0, 1.0, 2_000_001), -np.abs(np.random.default_rng(0).normal(0, 3, 200_000))])
    x = x.astype(np.float32)
    y = _ex2_fma(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 2.5e-7, rel.max()
    # below the clamp the result stays a tiny non-negative number (ex2.approx.ftz gives 0)
    low = _ex2_fma(np.array([-127.0, -200.0, -1e30], np.float32))
    assert np.all(low >= 0) and np.all(low < 2.0 ** -125)
    # integers are exact powers of two
    k = np.arange(-120, 20).astype(np.float32)
    np.testing.assert_allclose(_ex2_fma(k), np.exp2(k), rtol=2e-7)
