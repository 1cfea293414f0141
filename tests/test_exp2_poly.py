"""Error bound of the FMA-pipe 2^x the kernel uses on tiles without masked
entries (Cody-Waite reduction + degree-3 minimax polynomial).

The kernel's float32 steps are replayed in numpy with its constants (read
from the CUDA source) and compared with exp2 over the whole input range the
softmax feeds it (x <= 8 after the lazy-rescale threshold, clamped at -126).
The bound, 1e-4 relative, is far below the 2^-9 relative rounding of the
bf16 P that follows.
"""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "masked_attention_fa_b200", "csrc", "fa_kernel_sm100.cu")


def _coeffs():
    src = open(SRC).read()
    body = src[src.index("void ex2_poly_x2"):]
    body = body[:body.index("\n}\n")]
    nums = re.findall(r"([0-9]+\.[0-9]+)f", body)
    # order of appearance: shift constant, -126 clamp, c3, c3, c2, c2, c1, c1, c0, c0
    vals = [float(x) for x in nums if float(x) < 1.0]
    c3, c2, c1, c0 = vals[0], vals[2], vals[4], vals[6]
    return np.float32(c0), np.float32(c1), np.float32(c2), np.float32(c3)


def _fma32(a, b, c):
    return (a.astype(np.float64) * b + c).astype(np.float32)


def ex2_poly_replay(x):
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    shift = np.float32(12582912.0)
    t = (x + shift).astype(np.float32)
    n = (t - shift).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = _fma32(np.full_like(f, c3), f, c2)
    p = _fma32(p, f, c1)
    p = _fma32(p, f, c0)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_poly_exp2_relative_error_bound():
    x = np.linspace(-125.0, 9.0, 2_000_001).astype(np.float32)
    got = ex2_poly_replay(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1e-4, rel.max()


def test_poly_exp2_integers_and_clamp():
    ks = np.arange(-120, 9).astype(np.float32)
    got = ex2_poly_replay(ks).astype(np.float64)
    np.testing.assert_allclose(got, np.exp2(ks.astype(np.float64)), rtol=1e-4)
    tiny = ex2_poly_replay(np.array([-1e9, -300.0, -126.0], np.float32))
    assert np.all(tiny >= 0) and np.all(tiny < 1e-37)
