"""The kernels' FMA-pipe exp2 (exp2_fma2 in sm100_ptx.cuh), checked on the CPU
by emulating its fp32 operation sequence step by step against 2^x in fp64:
the coefficients match a fresh Remez fit, the relative error stays within the
fit's bound, integers come out exact, and very negative inputs flush towards 0.
"""
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_attention_109_b200", "csrc")
sys.path.insert(0, CSRC)
import exp2_poly_fit  # noqa: E402

f32 = np.float32


def kernel_coefficients():
    text = open(os.path.join(CSRC, "sm100_ptx.cuh")).read()
    return [f32(float(re.search(rf"kExp2A{k} = ([-0-9.e]+)f;", text).group(1)))
            for k in (1, 2, 3)]


def fma32(a, b, c):
    # a*b is exact in fp64 for fp32 operands; one rounding to fp32 after the add
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(f32)


def emulate(x):
    a1, a2, a3 = kernel_coefficients()
    x = np.maximum(x.astype(f32), f32(-126.0))
    sh = f32(12582912.0)
    t = (x + sh).astype(f32)
    f = (x - (t - sh).astype(f32)).astype(f32)
    p = fma32(f, np.full_like(f, a3), np.full_like(f, a2))
    p = fma32(p, f, np.full_like(f, a1))
    p = fma32(p, f, np.full_like(f, f32(1.0)))
    bits = (p.view(np.uint32).astype(np.uint64) +
            (t.view(np.uint32).astype(np.uint64) << np.uint64(23))) & np.uint64(0xFFFFFFFF)
    return bits.astype(np.uint32).view(f32)


def test_coefficients_match_the_fit():
    coef, err = exp2_poly_fit.fit(3)
    assert err < 4.4e-4
    assert [f32(c) for c in coef] == kernel_coefficients()


def test_relative_error_bound():
    x = np.linspace(-125.9, 8.5, 2_000_003).astype(f32)
    y = emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 4.5e-4, rel.max()


def test_integers_exact_and_underflow():
    n = np.arange(-126, 9, dtype=np.int64)
    assert np.array_equal(emulate(n.astype(f32)).astype(np.float64), np.exp2(n.astype(np.float64)))
    tiny = emulate(np.array([-126.4, -130.0, -1e9, -np.inf], dtype=f32))
    assert np.all(tiny >= 0) and np.all(tiny <= 2.0 ** -125)
