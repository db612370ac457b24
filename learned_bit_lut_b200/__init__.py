"""any4 mixed-precision linear layer for NVIDIA B200 (sm_100a).

A thin Python binding over the C ABI of ``libany4.so`` (``include/any4.h``):
``any4_pack``, ``any4_dequant``, ``any4_linear`` (and their any3/any2
``*_bits`` forms), the fixed-table formats
(``any4_pack_format``, ``any4_format_lut``) and the size queries. The
CUDA library does all the work; PyTorch only provides device memory and
streams.
"""
from ._lib import (ANY4_EALIGN, ANY4_ECUDA, ANY4_EINVAL, ANY4_ESHAPE, ANY4_EWORKSPACE,
                   ANY4_FORMAT_FP4, ANY4_FORMAT_INT4, ANY4_FORMAT_NF4, ANY4_OK, EXPORTED, FORMATS,
                   LIB_PATH, Any4Error, any4_dequant, any4_format_lut, any4_linear,
                   any4_linear_grid, any4_linear_kernel, KERNELS, any4_linear_noalloc, any4_linear_workspace_bytes, noalloc_status, any4_pack,
                   any4_pack_format,
                   any4_packed_bytes, any4_quantize, any4_strerror, lib, workspace_for,
                   any4_packed_bytes_bits, any4_pack_bits, any4_dequant_bits, any4_linear_bits)

__all__ = ["any4_quantize", "any4_pack", "any4_pack_bits", "any4_dequant_bits", "any4_linear_bits",
           "any4_packed_bytes_bits", "any4_pack_format", "any4_format_lut", "FORMATS", "ANY4_FORMAT_INT4",
           "ANY4_FORMAT_NF4", "ANY4_FORMAT_FP4", "any4_dequant", "any4_linear", "any4_linear_noalloc", "noalloc_status", "any4_packed_bytes",
           "any4_linear_workspace_bytes", "any4_linear_grid", "any4_linear_kernel", "KERNELS", "any4_strerror", "Any4Error", "workspace_for", "lib",
           "LIB_PATH", "EXPORTED", "ANY4_OK", "ANY4_EINVAL", "ANY4_EALIGN", "ANY4_ESHAPE",
           "ANY4_EWORKSPACE", "ANY4_ECUDA"]
