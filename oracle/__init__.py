"""Oracle for the any4 mixed-precision linear layer.

TEST INFRASTRUCTURE ONLY. This package is a plain, slow, float64 CPU
restatement of any4 (group scaling, single-sample calibration, per-row
weighted k-means, bit-exact dequantization, fp64 linear). It exists to check
the CUDA library. Only the tests, the smoke check of ``__graft_entry__`` and
the CPU-baseline leg of ``bench.py`` may import it; the library itself never
does, and the two share no code.

Every function cites the passage of the source pages it follows (page title
and section). Parity is pinned by the CPU tests (``tests/test_oracle_*.py``)
against values and properties the pages and the mathematics fix.
"""
from .any4 import (Any4Tensors, algorithmic_bytes, calibrate, dequant, dequant_rows,
                   e_step, group_scale, init_lut, int_grid, kmeans_rows, kmeans_weights,
                   linear, linear_rows, m_step, objective, pack_nibbles, quantize,
                   unpack_nibbles)
from .bf16 import (bf16_bits_to_f64, f32_to_bf16_bits, f64_to_bf16_bits, fma_to_f32,
                   fraction_to_bf16_bits, fraction_to_f32)
from .formats import quantize_format
from .tables import FORMATS, format_lut_bits, fp4_e2m1_values, int4_grid, nf4_bf16_bits, nf4_levels

__all__ = [
    "Any4Tensors", "algorithmic_bytes", "calibrate", "dequant", "dequant_rows", "e_step",
    "group_scale", "init_lut", "kmeans_rows", "kmeans_weights", "linear", "linear_rows",
    "m_step", "objective", "pack_nibbles", "quantize", "unpack_nibbles",
    "bf16_bits_to_f64", "f32_to_bf16_bits", "f64_to_bf16_bits", "fma_to_f32",
    "fraction_to_bf16_bits", "fraction_to_f32", "int4_grid", "nf4_bf16_bits", "nf4_levels",
    "int_grid", "FORMATS", "format_lut_bits", "fp4_e2m1_values", "quantize_format",
]
