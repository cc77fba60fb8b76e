"""The FMA-pipe exp2 of the prefill softmax (exp2_poly2 in plx_device.cuh):
its coefficients are the ones exp2_poly_fit.py produces, and its fp32
evaluation (Cody-Waite style reduction, degree-4 polynomial, exponent add),
emulated step by step in numpy, stays within the stated 2.7e-6 of 2^x."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "covariance_corrected_softmax_b200", "csrc")


def _header_coeffs():
    with open(os.path.join(CSRC, "plx_device.cuh")) as f:
        src = f.read()
    body = src[src.index("float2 exp2_poly2(float2 x)"):]
    body = body[:body.index("\n}\n")]
    # r starts at c4 ("r = make_float2(c4, c4)"), then the Horner steps
    # "r = __ffma2_rn(r, f, make_float2(ck, ck))" add c3, c2, c1, c0
    vals = re.findall(r"r = make_float2\(([-0-9.e+]+)f, \1f\)", body)
    vals += re.findall(r"r = __ffma2_rn\(r, f, make_float2\(([-0-9.e+]+)f, \1f\)\)", body)
    vals = [float(v) for v in vals]
    return np.array(vals[::-1], dtype=np.float32)  # c0 .. c4


def _fit_module():
    spec = importlib.util.spec_from_file_location("exp2_poly_fit",
                                                  os.path.join(CSRC, "exp2_poly_fit.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _emulate(x, c):
    """The kernel's steps in fp32: clamp, round via the 1.5*2^23 bias, f = x - n,
    Horner, then add n to the exponent field."""
    x = np.maximum(x.astype(np.float32), np.float32(-32.0))
    bias = np.float32(12582912.0)
    y = (x + bias).astype(np.float32)
    n = (y - bias).astype(np.float32)
    f = (x - n).astype(np.float32)
    r = np.full_like(f, c[4])
    for k in (3, 2, 1, 0):
        r = (r * f + c[k]).astype(np.float32)
    bits = r.view(np.int32) + (y.view(np.int32) << 23)
    return bits.view(np.float32)


def test_header_coefficients_are_the_fit():
    c_hdr = _header_coeffs()
    c_fit = _fit_module().fit(4)
    assert c_hdr.shape == (5,)
    np.testing.assert_array_equal(c_hdr, c_fit)


def test_emulated_exp2_error_bound():
    c = _header_coeffs()
    x = np.linspace(-30.0, 8.0, 400001).astype(np.float32)
    got = _emulate(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 3e-6, rel.max()
    # far below fp16's rounding of P (2^-11), which is what the kernel keeps
    assert rel.max() < 2.0 ** -11 / 100


def test_emulated_exp2_clamps_below_minus_32():
    c = _header_coeffs()
    got = _emulate(np.array([-40.0, -1000.0, -32.0], dtype=np.float32), c)
    assert np.all(got > 0) and np.all(np.abs(got / np.float32(2.0 ** -32) - 1) < 3e-6)
    # 2^-32 rounds to zero in fp16, like the true value would
    assert np.all(got.astype(np.float16) == 0)
