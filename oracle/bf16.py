"""Exact bf16 / fp32 rounding for the any4 oracle (test infrastructure).

The any4 explainer (10100.com, article 149119421, §二 "LUT") stores every row's
16 table values as FP16/BF16; the dequantized weight is the per-group affine
map of the looked-up value. This module provides the rounding steps needed to
state that dequantization exactly:

* ``f32_to_bf16_bits``  - round an fp32 value to bf16, nearest-even.
* ``f64_to_bf16_bits``  - round a float64 value directly to bf16, nearest-even
  (one rounding, no detour through fp32).
* ``fraction_to_f32``   - round an exact rational to fp32, nearest-even.
* ``fma_to_f32``        - the fp32 fused multiply-add of bf16 operands: the
  exact value a*l + b rounded once to fp32.

No NaN or infinity is ever produced or accepted here; fp32 and bf16
subnormals are kept (never flushed).
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

F32_MIN_EXP = -126     # smallest normal fp32 / bf16 exponent
F32_MANT = 23          # fp32 stored fraction bits
BF16_MANT = 7          # bf16 stored fraction bits


def bf16_bits_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact float64 values."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def f32_to_bf16_bits(f32) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even) -> uint16 bits.

    Rounding keeps the top 16 bits of the fp32 pattern after adding half an
    ulp of the kept part (0x7FFF) plus the kept part's lowest bit, which makes
    exact halves go to the even neighbour.
    """
    f = np.asarray(f32, dtype=np.float32)
    if not np.all(np.isfinite(f)):
        raise ValueError("non-finite value in bf16 rounding")
    u = f.view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def f64_to_bf16_bits(x) -> np.ndarray:
    """Round float64 values directly to bf16 (nearest, ties to even).

    With x = m * 2**e, 0.5 <= |m| < 1 (frexp), a normal bf16 keeps 8
    significant bits, i.e. its quantum is 2**(e-8); below the normal range the
    quantum is fixed at 2**-133. Scaling by a power of two is exact, and
    ``np.rint`` rounds half to even.
    """
    x = np.asarray(x, dtype=np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("non-finite value in bf16 rounding")
    _, e = np.frexp(x)
    qexp = np.maximum(e - (BF16_MANT + 1), F32_MIN_EXP - BF16_MANT)
    r = np.ldexp(np.rint(np.ldexp(x, -qexp)), qexp)
    if np.any(np.abs(r) > 3.3895313892515355e38):
        raise ValueError("bf16 overflow")
    # r is bf16-representable, so the float32 cast is exact.
    return (r.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def fraction_to_f32(v: Fraction) -> np.float32:
    """Round an exact rational to fp32, nearest with ties to even."""
    if v == 0:
        return np.float32(0.0)
    neg = v < 0
    a = -v if neg else v
    # exponent e with 2**e <= a < 2**(e+1)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, F32_MIN_EXP)
    quantum = Fraction(2) ** (e - F32_MANT)
    q = a / quantum
    n = q.numerator // q.denominator
    rem = q - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    val = Fraction(n) * quantum
    f = np.float32(float(val))          # val has <= 24 significant bits: exact
    if Fraction(float(f)) != val:
        raise ValueError("fp32 overflow")
    return np.float32(-f) if neg else f


def fma_to_f32(a, l, b) -> np.ndarray:
    """fp32 fused multiply-add a*l + b of bf16-valued operands.

    The exact result is rounded once to fp32. For bf16 operands the product
    a*l has at most 16 significant bits, so it is exact in float64. The sum is
    formed with TwoSum: s = fl(p + b) and err with s + err == p + b exactly.
    When err == 0 the float64 sum is the exact value and numpy's float32 cast
    rounds it correctly (nearest-even); it also gives IEEE signed zeros
    (+0 for an exact cancellation, -0 only for (-0) + (-0)). When err != 0 the
    exact value s + err is rounded by ``fraction_to_f32``.
    """
    a = np.asarray(a, dtype=np.float64)
    l = np.asarray(l, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    a, l, b = np.broadcast_arrays(a, l, b)
    p = a * l
    s = p + b
    bb = s - p
    err = (p - (s - bb)) + (b - bb)
    out = s.astype(np.float32)
    bad = np.nonzero(err != 0.0)
    if bad[0].size:
        sf, ef = s[bad], err[bad]
        out[bad] = np.array([fraction_to_f32(Fraction(float(x)) + Fraction(float(y)))
                             for x, y in zip(sf, ef)], dtype=np.float32)
    return out


def fraction_to_bf16_bits(v: Fraction) -> int:
    """Round an exact rational directly to bf16 (nearest-even) -> bits."""
    if v == 0:
        return 0
    neg = v < 0
    a = -v if neg else v
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, F32_MIN_EXP)
    quantum = Fraction(2) ** (e - BF16_MANT)
    q = a / quantum
    n = q.numerator // q.denominator
    rem = q - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    f = np.float32(float(Fraction(n) * quantum))
    bits = int(f.view(np.uint32) >> np.uint32(16))
    return bits | 0x8000 if neg else bits
