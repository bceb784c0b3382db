"""The software exp2 used for part of the softmax exponentials: its
polynomial coefficients (read from the kernel source) meet the stated
relative-error bounds for 2^f on [-1/2, 1/2], and the range reduction keeps
the error bound for the inputs the softmax produces (x in [-126, 8])."""
import os
import re

import numpy as np
import pytest

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "flash_attention_fwd_b200", "csrc", "fwd_common.cuh")


def coefficients():
    src = open(SRC).read()
    body = src[src.index("exp2_poly2(uint64_t x2)"):src.index("uint32_t t0 = (uint32_t)t")]
    deg3 = body[body.index("DEG == 3"):body.index("} else {")]
    deg4 = body[body.index("} else {"):]

    def ordered(block):
        vals = [float(v) for v in re.findall(r"f2_pack\(([0-9.e-]+)f,", block)]
        # Horner order: highest coefficient first
        return vals[::-1]

    return {3: ordered(deg3), 4: ordered(deg4)}


def horner32(coefs, f):
    f = f.astype(np.float32)
    p = np.full_like(f, np.float32(coefs[-1]))
    for c in coefs[-2::-1]:
        p = (p.astype(np.float64) * f + np.float64(np.float32(c))).astype(np.float32)
    return p


@pytest.mark.parametrize("deg,bound", [(3, 8e-5), (4, 3e-6)])
def test_polynomial_bound(deg, bound):
    c = coefficients()[deg]
    assert len(c) == deg + 1
    f = np.linspace(-0.5, 0.5, 200001)
    rel = np.abs(horner32(c, f).astype(np.float64) / np.exp2(f) - 1.0)
    assert rel.max() <= bound


@pytest.mark.parametrize("deg,bound", [(3, 8e-5), (4, 3e-6)])
def test_range_reduction(deg, bound):
    c = coefficients()[deg]
    x = np.concatenate([np.linspace(-126.0, 8.0, 400001),
                        np.array([-126.0, -0.5, 0.5, 0.0, 7.9999])]).astype(np.float32)
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    assert np.all(np.abs(f) <= 0.5)
    p = horner32(c, f)
    bits = p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))
    y = (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32).astype(np.float64)
    exact = np.exp2(x.astype(np.float64))
    normal = x > -125.0
    assert np.all(np.abs(y[normal] / exact[normal] - 1.0) <= bound)
    assert np.all(y[~normal] < 1e-37)   # masked scores: vanishingly small
