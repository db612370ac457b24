"""C ABI: the library loads, exports what include/any4.h declares, and rejects
invalid calls on the host before any launch (CPU only, no GPU needed)."""
import ctypes
import os
import re

import pytest

import numpy as np

import learned_bit_lut_b200 as a4
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "any4.h")).read()
    return sorted(set(re.findall(r"ANY4_API\s+[\w\s\*]*?\b(any4_\w+)\s*\(", src)))


def test_header_declarations_are_exported():
    names = _declared()
    assert names == sorted(a4.EXPORTED)
    for n in names:
        assert hasattr(a4.lib, n), n
        assert ctypes.cast(getattr(a4.lib, n), ctypes.c_void_p).value


def test_packed_bytes_accounting():
    n, k, g = 4096, 4096, 128
    total = a4.any4_packed_bytes(n, k, g)
    idx, lut, ab = n * k // 2, 32 * n, 4 * n * (k // g)
    assert total == idx + lut + ab            # all sections already 256-byte multiples here
    assert lut * 8 / (n * k) == 0.0625        # explainer section 2.3
    # N is padded to 32 rows; each section is rounded up to 256 bytes
    assert a4.any4_packed_bytes(16, 64, 64) == 32 * 32 + 32 * 32 + 256
    assert a4.any4_packed_bytes(144, 128, 64) == 160 * 64 + 160 * 32 + 160 * 2 * 4


@pytest.mark.parametrize("n,k,g", [(0, 64, 64), (15, 64, 64), (16, 63, 64), (16, 64, 32),
                                   (16, 192, 128), (16, 64, 96), (-16, 64, 64)])
def test_bad_shapes(n, k, g):
    assert a4.any4_packed_bytes(n, k, g) == 0
    assert a4.any4_linear_workspace_bytes(1, n, k, g) == 0
    p = ctypes.c_void_p(256)
    assert a4.lib.any4_pack(p, p, p, p, n, k, g, p, 1 << 30, None) == a4.ANY4_ESHAPE
    assert a4.lib.any4_dequant(p, n, k, g, p, None) == a4.ANY4_ESHAPE
    assert a4.lib.any4_linear(p, p, 1, n, k, g, p, p, 1 << 30, None) == a4.ANY4_ESHAPE


@pytest.mark.parametrize("m", [0, -1, (1 << 20) + 1])
def test_bad_m(m):
    p = ctypes.c_void_p(256)
    assert a4.any4_linear_workspace_bytes(m, 64, 64, 64) == 0
    assert a4.lib.any4_linear(p, p, m, 64, 64, 64, p, p, 1 << 30, None) == a4.ANY4_ESHAPE


def test_null_and_misaligned_pointers():
    p, z = ctypes.c_void_p(256), ctypes.c_void_p(0)
    odd = ctypes.c_void_p(258)
    assert a4.lib.any4_pack(z, p, p, p, 16, 64, 64, p, 4096, None) == a4.ANY4_EINVAL
    assert a4.lib.any4_pack(p, p, p, p, 16, 64, 64, z, 4096, None) == a4.ANY4_EINVAL
    assert a4.lib.any4_pack(p, p, p, p, 16, 64, 64, odd, 4096, None) == a4.ANY4_EALIGN
    assert a4.lib.any4_pack(p, p, p, p, 16, 64, 64, p, 100, None) == a4.ANY4_EWORKSPACE
    assert a4.lib.any4_dequant(z, 16, 64, 64, p, None) == a4.ANY4_EINVAL
    assert a4.lib.any4_dequant(p, 16, 64, 64, ctypes.c_void_p(257), None) == a4.ANY4_EALIGN
    assert a4.lib.any4_linear(z, p, 1, 16, 64, 64, p, p, 1 << 20, None) == a4.ANY4_EINVAL
    assert a4.lib.any4_linear(odd, p, 1, 16, 64, 64, p, p, 1 << 20, None) == a4.ANY4_EALIGN
    assert a4.lib.any4_linear(p, p, 1, 16, 64, 64, p, odd, 1 << 20, None) == a4.ANY4_EALIGN


def test_strerror_covers_all_codes():
    for code in (0, -1, -2, -3, -4, -5):
        assert a4.any4_strerror(code).startswith("ANY4_")
    assert "unknown" in a4.any4_strerror(7)


def test_format_tables_match_oracle():
    # host-side tables of the fixed formats, built independently of the oracle
    for fmt in oracle.FORMATS:
        lib_bits = np.array(a4.any4_format_lut(fmt), dtype=np.uint16)
        np.testing.assert_array_equal(lib_bits, oracle.format_lut_bits(fmt))


def test_format_lut_rejects_unknown_format():
    buf = (ctypes.c_uint16 * 16)()
    assert a4.lib.any4_format_lut(0, ctypes.cast(buf, ctypes.c_void_p)) == a4.ANY4_EINVAL
    assert a4.lib.any4_format_lut(a4.ANY4_FORMAT_NF4, None) == a4.ANY4_EINVAL


def test_pack_format_rejects_bad_arguments():
    dummy = ctypes.c_void_p(256)
    # unknown format, null pointer, bad shape, misaligned buffer: all before any launch
    assert a4.lib.any4_pack_format(9, dummy, dummy, dummy, 32, 64, 64, dummy, 1 << 20, None) == a4.ANY4_EINVAL
    assert a4.lib.any4_pack_format(1, None, dummy, dummy, 32, 64, 64, dummy, 1 << 20, None) == a4.ANY4_EINVAL
    assert a4.lib.any4_pack_format(1, dummy, dummy, dummy, 33, 64, 64, dummy, 1 << 20, None) == a4.ANY4_ESHAPE
    assert a4.lib.any4_pack_format(1, dummy, dummy, dummy, 32, 64, 64, ctypes.c_void_p(258), 1 << 20,
                                   None) == a4.ANY4_EALIGN
    assert a4.lib.any4_pack_format(1, dummy, dummy, dummy, 32, 64, 64, dummy, 16, None) == a4.ANY4_EWORKSPACE


def test_quantize_rejects_bad_arguments():
    d = ctypes.c_void_p(256)
    q = a4.lib.any4_quantize
    assert q(None, d, 32, 64, 64, 4, 10, d, d, d, d, None) == a4.ANY4_EINVAL
    assert q(d, d, 32, 64, 64, 5, 10, d, d, d, d, None) == a4.ANY4_EINVAL      # bits
    assert q(d, d, 32, 64, 64, 1, 10, d, d, d, d, None) == a4.ANY4_EINVAL
    assert q(d, d, 32, 64, 64, 4, -1, d, d, d, d, None) == a4.ANY4_EINVAL      # iters
    assert q(d, d, 31, 64, 64, 4, 10, d, d, d, d, None) == a4.ANY4_ESHAPE
    assert q(d, d, 32, 64, 96, 4, 10, d, d, d, d, None) == a4.ANY4_ESHAPE


def test_bits_sizes_and_rejection():
    # dense any3 / any2 packing: N_pad*K*b/8 bytes of indices, same LUT and scales
    n, k, g = 4096, 4096, 128
    lut, ab = 32 * n, 4 * n * (k // g)
    assert a4.any4_packed_bytes_bits(4, n, k, g) == a4.any4_packed_bytes(n, k, g)
    assert a4.any4_packed_bytes_bits(3, n, k, g) == n * k * 3 // 8 + lut + ab
    assert a4.any4_packed_bytes_bits(2, n, k, g) == n * k // 4 + lut + ab
    for bad in (0, 1, 5, 8, -3):
        assert a4.any4_packed_bytes_bits(bad, n, k, g) == 0
    p = ctypes.c_void_p(256)
    assert a4.lib.any4_pack_bits(5, p, p, p, p, 64, 64, 64, p, 1 << 30, None) == a4.ANY4_ESHAPE
    assert a4.lib.any4_dequant_bits(1, p, 64, 64, 64, p, None) == a4.ANY4_ESHAPE
    assert a4.lib.any4_linear_bits(6, p, p, 1, 64, 64, 64, p, p, 1 << 30, None) == a4.ANY4_ESHAPE
    z = ctypes.c_void_p(0)
    assert a4.lib.any4_pack_bits(3, z, p, p, p, 64, 64, 64, p, 1 << 30, None) == a4.ANY4_EINVAL


def test_linear_grid_rejects_on_host():
    b, c = ctypes.c_int(0), ctypes.c_int(0)
    assert a4.lib.any4_linear_grid(4, 1, 4096, 4096, 128, None, ctypes.byref(c)) == a4.ANY4_EINVAL
    assert a4.lib.any4_linear_grid(4, 1, 4096, 4096, 128, ctypes.byref(b), None) == a4.ANY4_EINVAL
    assert a4.lib.any4_linear_grid(5, 1, 4096, 4096, 128, ctypes.byref(b), ctypes.byref(c)) == a4.ANY4_ESHAPE
    assert a4.lib.any4_linear_grid(4, 0, 4096, 4096, 128, ctypes.byref(b), ctypes.byref(c)) == a4.ANY4_ESHAPE
    assert a4.lib.any4_linear_grid(4, 1, 4096, 4000, 128, ctypes.byref(b), ctypes.byref(c)) == a4.ANY4_ESHAPE


def test_linear_kernel_rejects_on_host():
    assert a4.lib.any4_linear_kernel(5, 1, 4096, 4096, 128) == a4.ANY4_ESHAPE
    assert a4.lib.any4_linear_kernel(4, 0, 4096, 4096, 128) == a4.ANY4_ESHAPE
    assert a4.lib.any4_linear_kernel(4, 1, 4096, 4000, 128) == a4.ANY4_ESHAPE
    assert a4.lib.any4_linear_kernel(4, 1, 4095, 4096, 128) == a4.ANY4_ESHAPE
