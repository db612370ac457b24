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
