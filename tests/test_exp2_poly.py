"""The polynomial 2^x that the forward kernel runs on the FMA pipe.

Checks (on the CPU, emulating the kernel's fp32 steps with numpy):
  - the constants in sa_common.cuh are the ones gen_exp2_poly.py fits (degree 4);
  - over x in [-125, 0] the result is within 4e-6 relative of 2^x in fp64, including
    the range reduction x = n + f (n = round(x) via 1.5 * 2^23) and the exponent add;
  - integer x gives powers of two to within the same bound, and x below -125 clamps.
"""
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "prototype_sketch_attention_b200", "csrc")
sys.path.insert(0, CSRC)


def kernel_constants():
    src = open(os.path.join(CSRC, "sa_common.cuh")).read()
    body = src[src.index("exp2_poly2(uint64_t x2)"):]
    return np.array([float(re.search(rf"kC{i} = ([0-9.e+-]+)f;", body).group(1)) for i in range(5)],
                    dtype=np.float32)


def f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def fma32(a, b, c):
    return f32(np.asarray(a, np.float64) * np.asarray(b, np.float64) + np.asarray(c, np.float64))


def emulate(x):
    c = kernel_constants()
    magic = np.float32(12582912.0)
    x = np.maximum(f32(x), np.float32(-125.0))
    t = f32(x.astype(np.float64) + np.float64(magic))       # add.rn
    n = f32(t.astype(np.float64) - np.float64(magic))
    f = fma32(n, np.float32(-1.0), x)
    p = fma32(c[4], f, c[3])
    p = fma32(p, f, c[2])
    p = fma32(p, f, c[1])
    p = fma32(p, f, c[0])
    bits = (p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_constants_match_generator():
    import gen_exp2_poly
    c = gen_exp2_poly.fit(4)
    np.testing.assert_array_equal(c, kernel_constants())
    assert gen_exp2_poly.max_rel_error(c) < 4e-6


def test_error_bound_over_range():
    x = np.concatenate([np.linspace(-125.0, 0.0, 2_000_001), -np.logspace(-8, 0, 10001)])
    y = emulate(x).astype(np.float64)
    ref = np.exp2(f32(x).astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 4e-6, rel.max()


def test_integers_and_clamp():
    x = np.arange(-125, 1, dtype=np.float64)
    y = emulate(x).astype(np.float64)
    np.testing.assert_allclose(y, np.exp2(x), rtol=4e-6)
    assert emulate(np.array([-1e30]))[0] == emulate(np.array([-125.0]))[0]
    assert 0 < emulate(np.array([-np.inf]))[0] < 1e-37
