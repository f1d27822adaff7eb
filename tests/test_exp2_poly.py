"""The softmax kernels' software exp2 (exp2_poly2 in tc.cuh), emulated bit
for bit in numpy float32 with the coefficients read from the kernel source,
against numpy's exp2 in float64 over the whole input range the softmax
produces (x <= 8; x < -120 clamped).  The kernel moves part of the softmax
exponentials from the MUFU unit to the FMA pipes with it; its error must stay
far below the bf16 rounding (2^-9) that P receives right after."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "step_reuse_b200", "csrc", "tc.cuh")


def kernel_coefficients():
    text = open(SRC).read()
    vals = dict(re.findall(r"\b(kExpP[0-3]) = ([-0-9.e]+)f", text))
    return [np.float32(vals[f"kExpP{i}"]) for i in range(4)]


def test_kernels_share_one_polynomial():
    # one definition (tc.cuh); the kernels that use it define no copy of their own
    csrc = os.path.dirname(SRC)
    for name in os.listdir(csrc):
        if name.endswith(".cu"):
            text = open(os.path.join(csrc, name)).read()
            assert "void exp2_poly2" not in text and "kExpP0 =" not in text, name


def exp2_poly_emulated(x):
    c0, c1, c2, c3 = kernel_coefficients()
    x = np.maximum(np.asarray(x, np.float32), np.float32(-120.0))
    magic = np.float32(12582912.0)
    y = (x + magic).astype(np.float32)
    n = (y - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    # fmaf is fused: emulate each step in float64 then round to float32
    p = np.float32(np.float64(c3) * f + np.float64(c2))
    p = np.float32(np.float64(p) * f + np.float64(c1))
    p = np.float32(np.float64(p) * f + np.float64(c0))
    bits = (p.view(np.uint32).astype(np.uint64) + (y.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_exp2_poly_relative_error():
    x = np.concatenate([np.linspace(-120.0, 8.0, 2_000_001, dtype=np.float64),
                        np.arange(-120, 9, dtype=np.float64) + 0.5,
                        np.arange(-120, 9, dtype=np.float64)]).astype(np.float32)
    got = exp2_poly_emulated(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 1.05e-4, rel.max()
    assert rel.max() < 2.0 ** -9 / 18
    # integers (the row maximum among them) are exact powers of two
    xi = np.arange(-120, 9, dtype=np.float32)
    assert (exp2_poly_emulated(xi).astype(np.float64) == np.exp2(xi.astype(np.float64))).all()


def test_exp2_poly_clamps_and_orders():
    v = exp2_poly_emulated(np.array([-np.inf, -1000.0, -121.0, -120.0, 0.0, 8.0], np.float32))
    assert np.isfinite(v).all() and (v >= 0).all()
    assert v[0] == v[1] == v[2] == v[3] and v[3] < 1e-35
    assert v[4] == 1.0 and v[5] == 256.0
    # monotone on a fine grid (no jumps at the integer boundaries of the reduction)
    x = np.linspace(-20.0, 8.0, 200_001, dtype=np.float32)
    y = exp2_poly_emulated(x)
    assert (np.diff(y.astype(np.float64)) >= -1e-6 * y[1:]).all()
