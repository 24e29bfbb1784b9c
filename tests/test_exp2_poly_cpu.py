"""The FMA-pipe exponential of the attention kernel (exp2_poly_x2 in
csrc/sm100.cuh): its coefficients are the ones the committed fit
(csrc/fit_exp2_poly.py, Lawson's reweighted least squares for the minimax
relative error) produces, and the whole routine -- clamp at -125, rounding
range reduction with the 1.5 * 2^23 shift, Horner steps rounded to fp32 as
fused multiply-adds, exponent inserted by an integer add -- emulated in fp32
stays within its error bound of 2^x on the range the softmax uses."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "vision_transformer_encoder_layernorm_b200", "csrc")


def _kernel_coefficients():
    src = open(os.path.join(CSRC, "sm100.cuh")).read()
    body = src[src.index("void exp2_poly_x2("):]
    body = body[:body.index("\n}\n")]
    # Horner order in the kernel: c3 * f + c2, then * f + c1, then * f + c0
    vals = [float(v) for v in re.findall(r"f2_pack\(([0-9.]+)f, \1f\)", body)]
    shift = [v for v in vals if v > 1e6]
    coef = [v for v in vals if v < 2.0]
    assert shift == [12582912.0] and len(coef) == 4, vals
    c3, c2, c1, c0 = coef
    return np.array([c0, c1, c2, c3])


def _fit_module():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_coefficients_come_from_the_committed_fit():
    m = _fit_module()
    c = m.fit()
    k = _kernel_coefficients()
    assert np.allclose(c, k, rtol=2e-8, atol=0), (c, k)
    assert m.max_rel_error(k) < 7.5e-5


def _f32(a):
    return np.asarray(a, dtype=np.float64).astype(np.float32)


def _fma32(a, b, c):
    # a single rounding of a*b + c to fp32 (the fp64 product of two fp32
    # values is exact; the sum rounds once more only in rare double-rounding
    # cases, far below the bound checked here)
    return _f32(a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64))


def _emulate(x):
    c0, c1, c2, c3 = (np.float32(v) for v in _kernel_coefficients())
    x = np.maximum(_f32(x), np.float32(-125.0))
    t = _f32(x.astype(np.float64) + 12582912.0)
    j = _f32(t.astype(np.float64) - 12582912.0)
    f = _fma32(j, np.full_like(j, -1.0), x)
    p = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    p = _fma32(p, f, np.full_like(f, c1))
    p = _fma32(p, f, np.full_like(f, c0))
    bits = (p.view(np.uint32).astype(np.int64) + (t.view(np.uint32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_emulated_routine_within_bound():
    # the softmax feeds s * scale * log2(e) - m: at most 8 above the stale max
    x = np.concatenate([np.linspace(-125.0, 8.0, 400001), -np.arange(0, 125.01, 0.125)])
    y = _emulate(x).astype(np.float64)
    ref = np.exp2(_f32(x).astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 7.5e-5 + 4 * 2.0 ** -24, rel.max()
    # below the clamp the result is that of -125, within the bound of 2^-125
    # (masked keys: negligible against a row sum of at least 1)
    lo = _emulate(np.array([-125.0]))[0]
    assert np.all(_emulate(np.array([-126.0, -1e9, -np.inf])) == lo)
    assert abs(float(lo) / 2.0 ** -125 - 1.0) < 7.5e-5 + 4 * 2.0 ** -24
