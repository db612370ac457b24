"""Quantizers of the fixed-table 4-bit baselines (test infrastructure).

The any4 explainer's comparison table (10100.com, article 149119421, §一)
sets any4 against int4 (uniform scaling with the fixed integer map -8..7),
NF4 (a fixed table of 16 Gaussian-fitted values) and FP4. Each is a 16-entry
table shared by all rows, so a weight in any of these formats is an any4
weight whose per-row tables are all the same; the CUDA library packs it with
the format's table and runs the same kernels.

Readings (the pages give the tables' roles, not their scaling):

* int4: the any4 group scaling (asymmetric min-max onto [-8, 7]) and
  rounding to the nearest grid value (lowest index on ties);
* NF4: per-group absmax scaling, alpha = bf16(max |w|), beta = 0;
* FP4 (E2M1): per-group absmax scaling onto the largest code, alpha =
  bf16(max |w| / 6), beta = 0;
* for NF4 and FP4 the index is the nearest table value of w / alpha, lowest
  index on ties; a group of zeros gets alpha = 0 and index 0.
"""
from __future__ import annotations

import numpy as np

from .any4 import Any4Tensors, e_step, group_scale, pack_nibbles
from .bf16 import bf16_bits_to_f64, f64_to_bf16_bits
from .tables import format_lut_bits, fp4_e2m1_values, nf4_bf16_bits


def _quantize_format_rows(w_bits: np.ndarray, fmt: str, g: int):
    n, k = w_bits.shape
    table = bf16_bits_to_f64(format_lut_bits(fmt))
    if fmt == "int4":
        alpha_bits, beta_bits, ws = group_scale(w_bits, g)
    else:
        w = bf16_bits_to_f64(w_bits).reshape(n, k // g, g)
        amax = np.max(np.abs(w), axis=2)
        top = 1.0 if fmt == "nf4" else 6.0
        alpha_bits = f64_to_bf16_bits(amax / top)
        beta_bits = np.zeros_like(alpha_bits)
        a = bf16_bits_to_f64(alpha_bits)[:, :, None]
        safe = np.where(a == 0.0, 1.0, a)
        ws = np.where(a == 0.0, 0.0, w / safe).reshape(n, k)
    idx = e_step(ws, np.tile(table, (n, 1)))
    return pack_nibbles(idx), alpha_bits, beta_bits


def quantize_format(w_bits: np.ndarray, fmt: str, g: int = 128) -> Any4Tensors:
    """Quantize a bf16 weight matrix to a fixed-table format (canonical
    tensors), in row chunks to bound memory."""
    w_bits = np.asarray(w_bits, dtype=np.uint16)
    n, k = w_bits.shape
    idx_nib = np.empty((n, k // 2), dtype=np.uint8)
    alpha = np.empty((n, k // g), dtype=np.uint16)
    beta = np.empty((n, k // g), dtype=np.uint16)
    step = max(1, (1 << 19) // k)
    for r0 in range(0, n, step):
        r1 = min(n, r0 + step)
        idx_nib[r0:r1], alpha[r0:r1], beta[r0:r1] = _quantize_format_rows(w_bits[r0:r1], fmt, g)
    return Any4Tensors(idx_nib, np.tile(format_lut_bits(fmt), (n, 1)), alpha, beta, g)


__all__ = ["quantize_format", "format_lut_bits", "fp4_e2m1_values", "nf4_bf16_bits"]
