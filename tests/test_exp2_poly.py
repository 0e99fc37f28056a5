"""The FMA-pipe exp2 of the attention and mass kernels, checked on the host.

The kernels compute 2^x for one score pair in four with a degree-3
polynomial instead of the MUFU ex2 unit (mcs_ptx.cuh, exp2_poly2). This test
reads the polynomial's coefficients from that header and replays the same
float32 steps in numpy (the 1.5 * 2^23 shifter splits x = n + f with
|f| <= 1/2, Horner's rule with fused multiply-adds, n added to the exponent
field, arguments below -125 flushed to 0), then checks the relative error
against 2^x in double precision over the range the softmax produces.
"""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "free_sparse_attention_pddp_b200", "csrc", "mcs_ptx.cuh")


def _coefficients():
    src = open(HEADER).read()
    body = src[src.index("void exp2_poly2("):]
    body = body[:body.index("\n}\n")]
    # the three Horner steps, highest degree first: f2_fma(c3, f, c2), then + c1, then + c0
    coeffs = [float(v) for v in re.findall(r"f2_pack\(([0-9.]+)f, \1f\)", body)]
    assert len(coeffs) == 4, coeffs  # the shifter is a named constant, not matched here
    c3, c2, c1, c0 = coeffs
    return np.float32(c0), np.float32(c1), np.float32(c2), np.float32(c3)


def _fma32(a, b, c):
    # a fused multiply-add rounds once: exact product and sum in double, one float32 rounding
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly(x):
    c0, c1, c2, c3 = _coefficients()
    x = np.asarray(x, dtype=np.float32)
    xc = np.maximum(x, np.float32(-125.0))
    shift = np.float32(12582912.0)
    t = (xc + shift).astype(np.float32)
    f = (xc - (t - shift).astype(np.float32)).astype(np.float32)
    p = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    p = _fma32(p, f, np.full_like(f, c1))
    p = _fma32(p, f, np.full_like(f, c0))
    bits = (p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))).astype(np.uint32)
    r = bits.view(np.float32)
    return np.where(x < np.float32(-125.0), np.float32(0.0), r)


def test_relative_error_bound():
    # softmax arguments: s * scale * log2 e - m, at most +1 (lazy rescale threshold) and
    # down to far below the flush threshold
    x = np.linspace(-125.0, 1.5, 1_000_001).astype(np.float32)
    got = exp2_poly(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() < 8e-5, rel.max()  # far below bf16's 2^-9 relative rounding of P


def test_integers_and_flush():
    x = np.arange(-125, 2, dtype=np.float32)
    rel = np.abs(exp2_poly(x).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 8e-5
    assert np.all(exp2_poly(np.array([-125.5, -200.0, -np.inf], dtype=np.float32)) == 0.0)
    assert np.all(np.isfinite(exp2_poly(np.linspace(-130, 2, 10001).astype(np.float32))))


def test_monotone_on_a_fine_grid():
    # P must not invert the order of two close scores by more than its error bound
    x = np.linspace(-20.0, 1.0, 200_001).astype(np.float32)
    y = exp2_poly(x).astype(np.float64)
    dips = np.diff(y) / y[:-1]
    assert dips.min() > -2e-4
