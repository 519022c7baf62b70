"""The polynomial 2^x used for part of the softmax exponentials, checked on the CPU.

The kernel's constants are read from the CUDA header and the same float32 steps (round by the
1.5*2^23 trick, reduced argument in [-1/2, 1/2], degree-3 polynomial, exponent added to the bit
pattern) are replayed in numpy; the result must stay within 1e-4 relative of 2^x, well below the
bf16 rounding (2^-9) that P receives next, and masked scores (-inf) must give a value too small to
move a finite row sum."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(__file__), "..", "block_sparse_spatio_flash_b200", "csrc", "svg_common.cuh")


def constants():
    src = open(HDR).read()
    vals = dict(re.findall(r"kExpC(\d) = ([0-9.e+-]+)f", src))
    return [np.float32(float(vals[str(i)])) for i in range(4)]


def poly_exp2(x):
    c0, c1, c2, c3 = constants()
    x = np.asarray(x, dtype=np.float32)
    xc = np.maximum(x, np.float32(-125.0))
    magic = np.float32(12582912.0)
    r = (xc + magic).astype(np.float32)
    n = (r - magic).astype(np.float32)
    f = (xc - n).astype(np.float32)
    p = (((c3 * f + c2) * f + c1) * f + c0).astype(np.float32)
    bits = (r.view(np.uint32) << np.uint32(23)) + p.view(np.uint32)
    return bits.astype(np.uint32).view(np.float32)


def test_reduced_range_error():
    f = np.linspace(-0.5, 0.5, 200001)
    c0, c1, c2, c3 = (float(c) for c in constants())
    p = ((c3 * f + c2) * f + c1) * f + c0
    assert np.max(np.abs(p / np.exp2(f) - 1.0)) < 8e-5


def test_full_range_relative_error():
    x = np.concatenate([np.linspace(-124.0, 0.0, 400001), -np.logspace(-6, 0, 1001), [0.0]]).astype(np.float32)
    got = poly_exp2(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got / want - 1.0)) < 1e-4


def test_integers_and_masked():
    x = np.arange(-120, 1, dtype=np.float32)
    got = poly_exp2(x).astype(np.float64)
    assert np.allclose(got, np.exp2(x.astype(np.float64)), rtol=1e-4, atol=0)
    tiny = poly_exp2(np.array([-np.inf, -1e30, -200.0], dtype=np.float32))
    assert np.all(tiny > 0) and np.all(tiny < 1e-37)
