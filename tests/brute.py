"""Independent brute-force references used to pin the oracle.

Nothing here calls the oracle or the CUDA path.  Each routine reaches the
method's definitions by a different route than the oracle does:
  - the shared exponent by exact comparison against powers of two (no frexp);
  - codes by searching every grid point for the nearest one (no rounding
    formula), ties to the even code;
  - packed fields by assembling integers bit by bit;
  - sums with exact rational arithmetic (fractions.Fraction).
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np


def exact_exponent(values) -> int:
    """Unique e with 2^e <= max|v| < 2^(e+1), clamped to [-127, 127]; -127 if all zero."""
    amax = max(abs(Fraction(float(v))) for v in values)
    if amax == 0:
        return -127
    e = 0
    while Fraction(2) ** e > amax:
        e -= 1
    while Fraction(2) ** (e + 1) <= amax:
        e += 1
    return max(-127, min(127, e))


def nearest_code(x: float, e: int, m: int) -> int:
    """Nearest of the grid points c * 2^(e-m+2), |c| <= 2^(m-1)-1, ties to even c."""
    L = (1 << (m - 1)) - 1
    step = Fraction(2) ** (e - m + 2)
    fx = Fraction(float(x))
    best, best_d = None, None
    for c in range(-L, L + 1):
        d = abs(fx - c * step)
        if best is None or d < best_d or (d == best_d and c % 2 == 0 and best % 2 != 0):
            best, best_d = c, d
    return best


def brute_block(values, m: int):
    e = exact_exponent(values)
    return [nearest_code(v, e, m) for v in values], e


def code_value(c: int, e: int, m: int) -> Fraction:
    return c * Fraction(2) ** (e - m + 2)


def pack_bits(codes, m: int) -> bytes:
    """Little-endian bit stream: code i occupies bits [m*i, m*i + m)."""
    acc = 0
    for i, c in enumerate(codes):
        acc |= (int(c) & ((1 << m) - 1)) << (m * i)
    nbytes = len(codes) * m // 8
    return acc.to_bytes(nbytes, "little")


def unpack_bits(data: bytes, n: int, m: int):
    acc = int.from_bytes(bytes(data), "little")
    out = []
    for i in range(n):
        v = (acc >> (m * i)) & ((1 << m) - 1)
        if v >= 1 << (m - 1):
            v -= 1 << m
        out.append(v)
    return out


def decode_rows(codes, scales, counts):
    """Decode compact per-segment code/scale arrays with pure-Python bit ops.

    Returns an object array of Fractions, rows x K' (padded positions)."""
    bits = (8, 6, 4)
    rows = max(c.shape[0] for c in codes)
    segs = []
    for g in range(3):
        kp = (int(counts[g]) + 31) // 32 * 32
        seg = np.empty((rows, kp), dtype=object)
        for r in range(rows):
            for b in range(kp // 32):
                raw = bytes(codes[g][r, b * 32 * bits[g] // 8:(b + 1) * 32 * bits[g] // 8])
                q = unpack_bits(raw, 32, bits[g])
                e = int(scales[g][r, b]) - 127
                for t in range(32):
                    seg[r, b * 32 + t] = code_value(q[t], e, bits[g])
        segs.append(seg)
    return np.concatenate(segs, axis=1) if segs else np.empty((rows, 0), dtype=object)


def to_f64(frac_array) -> np.ndarray:
    return np.vectorize(float, otypes=[np.float64])(frac_array)


def ulp(x: float) -> float:
    return math.ulp(x)
