"""Fixed 16-entry tables of the 4-bit baselines (test infrastructure).

The any4 explainer's comparison table (10100.com, article 149119421, §一)
contrasts any4 with int4 (uniform scaling with the fixed integer map -8..7)
and NF4 (16 predefined Gaussian-fitted values read through one global table).
Both are special cases of a per-row table, which the reduction tests use.

The NF4 values are not printed on the pages. They are derived here from the
published construction of the 4-bit NormalFloat type (QLoRA): quantiles of the
standard normal at evenly spaced probabilities, 8 on the positive side and 7
on the negative side, plus an exact zero, scaled so the largest magnitude is
1. The outermost probability is 1 - delta with delta the mean of 1/(2*16) and
1/(2*15). Only the identity of the table on both sides of a reduction test
matters, not its exact digits.
"""
from __future__ import annotations

from statistics import NormalDist

import numpy as np

from .bf16 import f64_to_bf16_bits


def int4_grid() -> np.ndarray:
    """-8, -7, ..., 7 as float64."""
    return np.arange(-8.0, 8.0)


def nf4_levels() -> np.ndarray:
    """The 16 NormalFloat-4 levels in ascending order (float64, in [-1, 1])."""
    nd = NormalDist()
    delta = 0.5 * (1.0 / 32.0 + 1.0 / 30.0)
    top = 1.0 - delta
    pos = [nd.inv_cdf(p) for p in np.linspace(0.5, top, 9)[1:]]       # 8 values > 0
    neg = [-nd.inv_cdf(p) for p in np.linspace(0.5, top, 8)[1:]]      # 7 values < 0
    v = np.array(sorted(neg + [0.0] + pos), dtype=np.float64)
    return v / np.max(np.abs(v))


def nf4_bf16_bits() -> np.ndarray:
    return f64_to_bf16_bits(nf4_levels())


def fp4_e2m1_values() -> np.ndarray:
    """The 16 values of the 4-bit floating-point element type E2M1 by code
    0..15 (float64): bit 3 is the sign, bits 2..1 the exponent (bias 1),
    bit 0 the mantissa; exponent 0 is subnormal (0 or 0.5).

    The explainer's comparison table (§一) names FP4 among the 4-bit
    baselines without defining it; E2M1 is read as the common FP4 element
    format. Code 8 is -0.
    """
    out = np.empty(16, dtype=np.float64)
    for q in range(16):
        s, e, m = q >> 3, (q >> 1) & 3, q & 1
        mag = m * 0.5 if e == 0 else 2.0 ** (e - 1) * (1.0 + 0.5 * m)
        out[q] = -mag if s else mag
    out[8] = -0.0
    return out


FORMATS = ("int4", "nf4", "fp4")


def format_lut_bits(fmt: str) -> np.ndarray:
    """bf16 bits of the fixed 16-entry table of a 4-bit baseline format."""
    if fmt == "int4":
        return f64_to_bf16_bits(int4_grid())
    if fmt == "nf4":
        return nf4_bf16_bits()
    if fmt == "fp4":
        return f64_to_bf16_bits(fp4_e2m1_values())
    raise ValueError(fmt)
