"""The FMA-pipe exp2 used for part of the softmax exponentials.

The coefficients in attn_fwd.cuh must be the ones the committed Remez fit
produces, and a float32 simulation of the kernel's sequence (range
reduction by the 1.5*2^23 rounding trick, Horner with fused multiply-adds,
exponent-field add) must track 2^x within the fit's bound over the whole
input range the softmax produces (x <= 14; clamped at -126).
"""
import os
import re
import sys

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "long_context_bidirectional_b200", "csrc")
sys.path.insert(0, CSRC)
import fit_exp2_poly as F  # noqa: E402


def kernel_coefficients():
    src = open(os.path.join(CSRC, "attn_fwd.cuh")).read()
    body = src[src.index("float exp2_poly(float x)"):]
    body = body[:body.index("return")]
    nums = [float(x) for x in re.findall(r"(-?\d+\.\d+(?:e-?\d+)?)f", body)]
    # constants in order: clamp, 2 x rounding magic, c3, c2, c1, c0
    return nums[-4:][::-1]          # -> c0, c1, c2, c3


def fma32(a, b, c):
    return (np.float64(a) * np.float64(b) + np.float64(c)).astype(np.float32)


def exp2_poly_sim(x):
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    c0, c1, c2, c3 = (np.float32(v) for v in kernel_coefficients())
    p = np.full_like(f, c3)
    p = fma32(p, f, c2)
    p = fma32(p, f, c1)
    p = fma32(p, f, c0)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_kernel_coefficients_are_the_fit():
    c, err = F.remez_rel(3)
    np.testing.assert_allclose(kernel_coefficients(), c.astype(np.float32), rtol=1e-6)
    assert err < 8e-5


def test_fit_equioscillates():
    c, err = F.remez_rel(3)
    g = np.linspace(-0.5, 0.5, 20001)
    e = F.rel_err(c, g)
    # a minimax fit of degree 3 touches +-err at 5 alternating points
    assert np.isclose(np.max(np.abs(e)), err)
    ext = np.sum(np.abs(e) > 0.999 * err)
    assert ext >= 5


def test_simulated_kernel_exp2_accuracy():
    # results are normal floats for x >= -125; below that they are < 2^-125
    # and round to 0 in fp16 (checked separately)
    x = np.concatenate([np.linspace(-125, 14, 200001), np.linspace(-2, 2, 50001),
                        np.arange(-125, 15)]).astype(np.float32)
    got = exp2_poly_sim(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert np.max(rel) < 8e-5, float(np.max(rel))
    # clamped region: tiny non-negative values that round to 0 in fp16
    tiny = exp2_poly_sim(np.array([-125.5, -126.0, -200.0, -np.inf], dtype=np.float32))
    assert np.all(tiny >= 0) and np.all(tiny < 2.0 ** -124)
    assert np.all(tiny.astype(np.float16) == 0)
