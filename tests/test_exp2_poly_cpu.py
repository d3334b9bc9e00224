"""The causal-attention kernel takes part of its 2^x from a cubic on the FMA pipes
(`exp2_poly2` in csrc/sm100.cuh) instead of the special-function unit.  These tests read
the coefficients out of that source, replay its fp32 steps here (range reduction by the
1.5 * 2^23 rounding constant, the cubic by fused multiply-adds, 2^j added into the exponent
field) and hold the result to the relative error bound its comment states, over the whole
range the kernel can feed it."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(__file__), "..", "gated_linear_attention_liger_b200", "csrc", "sm100.cuh")


def _coefficients():
    text = open(SRC).read()
    body = text[text.index("float2 exp2_poly2(float2 x)"):]
    body = body[:body.index("\n}\n")]
    consts = [float(c) for c in re.findall(r"make_float2\(([0-9.]+)f, \1f\)", body)]
    consts = [c for c in consts if c < 1.0]   # drop the rounding constant 1.5 * 2^23
    # Horner order in the source: c3, c2, then c1, then c0
    assert len(consts) == 4, consts
    return [np.float32(c) for c in consts]


def _fma32(a, b, c):
    """fp32 fused multiply-add: the float32 product is exact in float64, one rounding to float32."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly(x):
    c3, c2, c1, c0 = _coefficients()
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    rnd = np.float32(12582912.0)
    t = (x + rnd).astype(np.float32)
    j = (t - rnd).astype(np.float32)
    f = _fma32(j, np.full_like(j, -1.0), x)
    p = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    p = _fma32(p, f, np.full_like(f, c1))
    p = _fma32(p, f, np.full_like(f, c0))
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_reduction_is_exact_and_fraction_in_half_interval():
    x = np.linspace(-125.0, 127.0, 200001, dtype=np.float32)
    rnd = np.float32(12582912.0)
    j = ((x + rnd).astype(np.float32) - rnd).astype(np.float32)
    assert np.array_equal(j, np.rint(x.astype(np.float64)).astype(np.float32))
    f = x.astype(np.float64) - j.astype(np.float64)
    assert np.abs(f).max() <= 0.5


def test_relative_error_within_stated_bound():
    x = np.concatenate([np.linspace(-125.0, 127.0, 400001, dtype=np.float32),
                        np.linspace(-1.0, 1.0, 100001, dtype=np.float32)])
    got = exp2_poly(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() < 8e-5, rel.max()
    assert np.all(np.isfinite(got)) and np.all(got > 0)


def test_below_range_reads_as_two_to_minus_125():
    got = exp2_poly(np.array([-125.0, -200.0, -1e30, -np.inf], np.float32)).astype(np.float64)
    assert np.allclose(got, 2.0 ** -125, rtol=1e-4)


def test_integers_are_near_exact_powers_of_two():
    k = np.arange(-125, 128, dtype=np.float32)
    got = exp2_poly(k).astype(np.float64)
    # at f = 0 the cubic gives its constant term: 2^k scaled by c0
    c0 = float(_coefficients()[3])
    assert np.allclose(got, np.exp2(k.astype(np.float64)) * c0, rtol=1e-7)
