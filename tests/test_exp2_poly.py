"""The FMA-pipe exp2 (packed pairs) used for part of the forward's
exponentials (CPU).

Simulates the kernel's fp32 operation sequence in numpy (clamp, rounding by
the 1.5 * 2^23 constant, cubic in Horner form, exponent-field add) and checks
it against 2^x in fp64 over the whole range the kernel feeds it, and that the
fp32 coefficients in sm100.cuh are the ones the Remez fit produces."""
import os
import re

import numpy as np

from exact_io_aware_67_b200 import fit_exp2

HDR = os.path.join(os.path.dirname(fit_exp2.__file__), "csrc", "sm100.cuh")


def _coeffs_in_header():
    """The cubic's coefficients as the packed kernel function states them
    (each literal appears twice there, once per lane of the pair)."""
    txt = open(HDR).read()
    body = txt[txt.index("float2 ex2_poly2"):txt.index("return make_float2(__int_as_float")]
    vals = [float(v.rstrip("f")) for v in re.findall(r"[0-9]\.[0-9]+e[-+][0-9]+f", body)]
    assert len(vals) == 8 and vals[0::2] == vals[1::2], vals
    return vals[0::2]


def _ex2_poly(x, c):
    """The kernel's per-lane fp32 sequence: clamp, t = x + 1.5 2^23,
    n = t - 1.5 2^23, f = fma(n, -1, x), cubic by three fmas, n added to the
    exponent field."""
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-125.0))
    t = (x + f32(12582912.0)).astype(f32)
    n = (t - f32(12582912.0)).astype(f32)
    f = (x.astype(np.float64) - n.astype(np.float64)).astype(f32)
    # fused multiply-adds, rounded once each (evaluate in fp64, round to fp32)
    p = (f.astype(np.float64) * c[3] + c[2]).astype(f32)
    p = (p.astype(np.float64) * f + c[1]).astype(f32)
    p = (p.astype(np.float64) * f + c[0]).astype(f32)
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xffffffff).astype(np.uint32).view(f32)


def test_header_coefficients_match_fit():
    c, err = fit_exp2.remez()
    got = _coeffs_in_header()
    # header order: c3, c2, c1, c0
    np.testing.assert_allclose(got, [c[3], c[2], c[1], c[0]], rtol=2e-7)
    assert err < 1e-4


def test_relative_error_over_kernel_range():
    c = np.array(_coeffs_in_header()[::-1], dtype=np.float64)
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001), -np.random.default_rng(0).random(100000) * 20])
    y = _ex2_poly(x.astype(np.float32), c).astype(np.float64)
    ref = np.exp2(x.astype(np.float32).astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 1.2e-4, rel.max()


def test_masked_and_underflow_inputs_are_negligible():
    c = np.array(_coeffs_in_header()[::-1], dtype=np.float64)
    x = np.array([-np.inf, -1e30, -200.0, -125.0], dtype=np.float32)
    y = _ex2_poly(x, c)
    assert np.all(np.isfinite(y)) and np.all(y >= 0) and np.all(y <= 2.0 ** -124)
