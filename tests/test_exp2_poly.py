"""The softmax's FMA-pipe 2^x (ptx.cuh exp2_poly2), checked on the CPU.

The kernels evaluate part of their exponentials as 2^x = 2^j 2^f with
j = round(x) and a degree-3 polynomial for 2^f on [-1/2, 1/2] (Cody-Waite
range reduction).  This test repeats the same float32 steps in numpy --
rounding by adding 1.5 * 2^23, the Horner polynomial with the coefficients
compiled into ptx.cuh, and j added to the exponent field -- and checks the
relative error against the exact 2^x over every x the kernels feed it
(-120 <= x <= 0 under the fixed softmax reference), and that the constants
in ptx.cuh are the ones the fit script produces."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "global_causal_attention_b200", "csrc")


def coefficients_in_source():
    text = open(os.path.join(CSRC, "ptx.cuh")).read()
    body = text[text.index("uint64_t exp2_poly2("):]
    body = body[:body.index("return r;")]
    vals = [float(v) for v in re.findall(r"f2_pack\(([0-9.]+)f, \1f\)", body) if float(v) != 12582912.0]
    # Horner order in the source: c3, c2, c1, c0 (the rounding constant 1.5 * 2^23 set aside)
    assert len(vals) == 4, vals
    c3, c2, c1, c0 = vals
    return np.array([c0, c1, c2, c3], np.float32)


def emulate(x):
    """The kernel's steps, in float32 with round-to-nearest."""
    x = np.asarray(x, np.float32)
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic).astype(np.float32)).astype(np.float32)
    c = coefficients_in_source()
    p = (f * c[3] + c[2]).astype(np.float32)
    p = (p * f + c[1]).astype(np.float32)
    p = (p * f + c[0]).astype(np.float32)
    bits = (p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))).astype(np.uint32)
    return bits.view(np.float32)


def test_relative_error_over_the_softmax_range():
    x = np.concatenate([np.linspace(-120.0, 0.0, 2_000_001, dtype=np.float32),
                        np.float32(-np.arange(0, 121, dtype=np.float32)),          # integers (f = 0)
                        np.float32(-np.arange(0, 120, dtype=np.float32) - 0.5)])   # ties of the rounding
    got = emulate(x).astype(np.float64)
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(got / exact - 1.0)
    assert rel.max() < 1e-4, rel.max()
    # far below the bf16 rounding of P (relative 2^-9)
    assert rel.max() < 2.0 ** -9 / 20


def test_constants_match_the_fit():
    import importlib.util
    spec = importlib.util.spec_from_file_location("exp2_poly_fit", os.path.join(CSRC, "exp2_poly_fit.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    c, err = mod.fit()
    assert err < 1e-4
    np.testing.assert_allclose(coefficients_in_source(), c, rtol=1e-6)
