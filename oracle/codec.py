"""Sketch cache codec, plain numpy reference. TEST INFRASTRUCTURE ONLY (like the rest of
this package): only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline leg may
use it, and the CUDA library shares nothing with it.

What it computes. A cached sketch (k rows of length d, fp32) is stored compactly
between requests, since the sketch is user-only and is reused across candidates and
requests ("100,000 videos in your pocket" blog, section "3. The system makes it cheap
enough to matter", low-rank caching). The pages name no storage format; the plainest
readings, taken here, are:

  bf16: every value rounded to the nearest bfloat16 (ties to even); decode widens.
  fp8:  per row j a scale s_j = max_e |S_je| / 448 (1 for an all-zero row); every value
        S_je / s_j rounded to the nearest FP8 E4M3 value (ties to even; the OCP "fn"
        variant: finite only, largest magnitude 448); decode = code * s_j.

The scale and the quotient S_je / s_j are computed in fp32 (IEEE division, rounded to
nearest), since the quotient decides an integer code and a GPU encoder takes that
decision in fp32; decode's product is rounded to fp32 once. Zeros are written as +0.

E4M3 here is built from its definition (1 sign bit, 4 exponent bits with bias 7,
3 mantissa bits; exponent field 0 holds the subnormals k * 2^-9), not from a library,
so that a library's conversion can serve as an independent check.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def _round_half_even(x: np.ndarray) -> np.ndarray:
    return np.round(x)  # numpy rounds halves to even


def bf16_bits(x) -> np.ndarray:
    """fp32 -> bfloat16 bit patterns (uint16), round to nearest even; finite inputs."""
    u = np.ascontiguousarray(np.asarray(x, dtype=np.float32)).view(np.uint32).astype(np.uint64)
    lower = u & 0xFFFF
    upper = u >> 16
    round_up = (lower > 0x8000) | ((lower == 0x8000) & ((upper & 1) == 1))
    return (upper + round_up).astype(np.uint16)


def bf16_decode(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


def e4m3_round(a) -> np.ndarray:
    """Nearest E4M3 value to each |a| <= 448 (ties to even), as float64 magnitudes."""
    a = np.abs(np.asarray(a, dtype=np.float64))
    out = np.zeros_like(a)
    nz = a > 0
    e = np.floor(np.log2(np.where(nz, a, 1.0)))
    e = np.clip(e, -6, 8)                      # below 2^-6: the subnormal spacing 2^-9
    q = np.exp2(e - 3)                         # spacing of the binade (3 mantissa bits)
    r = _round_half_even(a / q) * q
    out[nz] = np.minimum(r[nz], E4M3_MAX)
    return out


def e4m3_bits(x) -> np.ndarray:
    """Values already within [-448, 448] -> E4M3 bit patterns (uint8), nearest even."""
    x = np.asarray(x, dtype=np.float64)
    m = e4m3_round(x)
    sign = (np.signbit(x) & (m > 0)).astype(np.uint8) << 7
    code = np.zeros(x.shape, dtype=np.uint8)
    nz = m > 0
    e = np.floor(np.log2(np.where(nz, m, 1.0)))
    normal = nz & (e >= -6)
    ef = np.where(normal, e + 7, 0).astype(np.int64)                     # exponent field
    frac = np.where(normal, m / np.exp2(e) - 1.0, m / 2.0 ** -9)          # mantissa units
    mant = np.where(normal, np.round(frac * 8), np.round(frac)).astype(np.int64)
    code[nz] = ((ef[nz] << 3) | mant[nz]).astype(np.uint8)
    return code | sign


def e4m3_decode(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    s = np.where(b & 0x80, -1.0, 1.0)
    ef = (b >> 3) & 0xF
    mant = b & 0x7
    val = np.where(ef == 0, mant * 2.0 ** -9, (1.0 + mant / 8.0) * np.exp2(ef - 7.0))
    return s * val


def fp8_encode(S) -> tuple[np.ndarray, np.ndarray]:
    """Sketch [..., k, d] -> (codes uint8 [..., k, d], scales fp32 [..., k])."""
    S = np.asarray(S, dtype=np.float32)
    amax = np.abs(S).max(axis=-1)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    y = (S / scale[..., None]).astype(np.float32)  # fp32 IEEE division
    return e4m3_bits(np.clip(y.astype(np.float64), -E4M3_MAX, E4M3_MAX)), scale


def fp8_decode(codes, scales) -> np.ndarray:
    return (e4m3_decode(codes) * np.asarray(scales, dtype=np.float64)[..., None]).astype(np.float32)
