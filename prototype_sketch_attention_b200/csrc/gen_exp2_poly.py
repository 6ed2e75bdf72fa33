"""Fits the polynomial used for 2^f, f in [-1/2, 1/2], on the FMA pipe of the forward kernel.

Method: weighted least squares in relative error (weights 1 / 2^f) at 512 Chebyshev
nodes of [-1/2, 1/2], then a few iterations of the Lawson reweighting scheme (IRLS)
that move the least-squares fit toward the minimax (equioscillating) fit. The
coefficients are rounded to fp32, and the printed error is that of the fp32
Horner evaluation with fused multiply-adds.

The kernel splits x <= 0 into n + f with n = round-to-nearest(x) (by adding and
subtracting 1.5 * 2^23), evaluates p(f) with fp32 FMAs, and adds n to the exponent
field of p(f). Run this script to regenerate the
constants; tests/test_exp2_poly.py checks the committed constants against the bound.

    python prototype_sketch_attention_b200/csrc/gen_exp2_poly.py [degree]
"""
from __future__ import annotations

import sys

import numpy as np


def fit(degree: int = 4, nodes: int = 512, iters: int = 60) -> np.ndarray:
    k = np.arange(nodes)
    f = -0.5 * np.cos(np.pi * (k + 0.5) / nodes)  # Chebyshev nodes on [-1/2, 1/2]
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True) / y[:, None]  # relative-error rows
    w = np.ones(nodes)
    c = None
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(V * sw[:, None], np.ones(nodes) * sw, rcond=None)
        err = np.abs(V @ c - 1.0)
        w = w * (err + 1e-300)
        w /= w.sum()
    return c.astype(np.float32)


def horner_fp32(c: np.ndarray, f: np.ndarray) -> np.ndarray:
    """fp32 Horner with fused multiply-add (each step rounded once to fp32)."""
    f64 = f.astype(np.float64)
    acc = np.float32(c[-1])
    acc = np.full(f.shape, acc, dtype=np.float32)
    for ci in c[-2::-1]:
        acc = (acc.astype(np.float64) * f64 + np.float64(ci)).astype(np.float32)
    return acc


def max_rel_error(c: np.ndarray, n: int = 1 << 20) -> float:
    f = np.linspace(-0.5, 0.5, n, dtype=np.float32)
    p = horner_fp32(c, f).astype(np.float64)
    return float(np.max(np.abs(p / np.exp2(f.astype(np.float64)) - 1.0)))


def main() -> int:
    degree = int(sys.argv[1]) if len(sys.argv) > 1 else 4
    c = fit(degree)
    print(f"// degree {degree}, max relative error {max_rel_error(c):.3e} (fp32 Horner, FMA)")
    for i, ci in enumerate(c):
        print(f"constexpr float kExp2C{i} = {float(ci)!r}f;  // {np.float32(ci).view(np.uint32):#010x}")
    return 0


if __name__ == "__main__":
    sys.exit(main())
