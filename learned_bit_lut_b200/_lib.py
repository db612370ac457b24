"""ctypes binding of libany4.so (include/any4.h).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity, and their device pointers plus the current CUDA stream are passed
to the C ABI. Every step of the computation runs in the library's kernels;
there is no fallback path. Importing this module fails loudly when the
library has not been built.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libany4.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python learned_bit_lut_b200/build.py`")

lib = ctypes.CDLL(LIB_PATH)

_c_size = ctypes.c_size_t
_c_int = ctypes.c_int
_p = ctypes.c_void_p

lib.any4_packed_bytes.argtypes = [_c_int, _c_int, _c_int]
lib.any4_packed_bytes.restype = _c_size
lib.any4_pack.argtypes = [_p, _p, _p, _p, _c_int, _c_int, _c_int, _p, _c_size, _p]
lib.any4_pack.restype = _c_int
lib.any4_dequant.argtypes = [_p, _c_int, _c_int, _c_int, _p, _p]
lib.any4_dequant.restype = _c_int
lib.any4_linear_workspace_bytes.argtypes = [_c_int, _c_int, _c_int, _c_int]
lib.any4_linear_workspace_bytes.restype = _c_size
lib.any4_linear_workspace_bytes_bits.argtypes = [_c_int, _c_int, _c_int, _c_int, _c_int]
lib.any4_linear_workspace_bytes_bits.restype = _c_size
lib.any4_linear_grid.argtypes = [_c_int, _c_int, _c_int, _c_int, _c_int, _p, _p]
lib.any4_linear_grid.restype = _c_int
lib.any4_linear_kernel.argtypes = [_c_int, _c_int, _c_int, _c_int, _c_int]
lib.any4_linear_kernel.restype = _c_int
lib.any4_linear.argtypes = [_p, _p, _c_int, _c_int, _c_int, _c_int, _p, _p, _c_size, _p]
lib.any4_linear.restype = _c_int
lib.any4_linear_noalloc.argtypes = [_p, _p, _c_int, _c_int, _c_int, _c_int, _p, _p]
lib.any4_linear_noalloc.restype = _c_int
lib.any4_noalloc_status_word.argtypes = [ctypes.POINTER(_p)]
lib.any4_noalloc_status_word.restype = _c_int
lib.any4_format_lut.argtypes = [_c_int, _p]
lib.any4_format_lut.restype = _c_int
lib.any4_pack_format.argtypes = [_c_int, _p, _p, _p, _c_int, _c_int, _c_int, _p, _c_size, _p]
lib.any4_pack_format.restype = _c_int
lib.any4_quantize.argtypes = [_p, _p, _c_int, _c_int, _c_int, _c_int, _c_int, _p, _p, _p, _p, _p]
lib.any4_quantize.restype = _c_int
lib.any4_packed_bytes_bits.argtypes = [_c_int, _c_int, _c_int, _c_int]
lib.any4_packed_bytes_bits.restype = _c_size
lib.any4_pack_bits.argtypes = [_c_int, _p, _p, _p, _p, _c_int, _c_int, _c_int, _p, _c_size, _p]
lib.any4_pack_bits.restype = _c_int
lib.any4_dequant_bits.argtypes = [_c_int, _p, _c_int, _c_int, _c_int, _p, _p]
lib.any4_dequant_bits.restype = _c_int
lib.any4_linear_bits.argtypes = [_c_int, _p, _p, _c_int, _c_int, _c_int, _c_int, _p, _p, _c_size, _p]
lib.any4_linear_bits.restype = _c_int
lib.any4_strerror.argtypes = [_c_int]
lib.any4_strerror.restype = ctypes.c_char_p
lib.any4_last_cuda_error.argtypes = []
lib.any4_last_cuda_error.restype = _c_int

EXPORTED = ("any4_packed_bytes", "any4_pack", "any4_dequant", "any4_linear_workspace_bytes",
            "any4_linear_workspace_bytes_bits", "any4_linear_grid", "any4_linear_kernel",
            "any4_linear", "any4_linear_noalloc", "any4_noalloc_status_word", "any4_quantize", "any4_format_lut",
            "any4_pack_format", "any4_packed_bytes_bits", "any4_pack_bits", "any4_dequant_bits",
            "any4_linear_bits", "any4_strerror", "any4_last_cuda_error")

ANY4_FORMAT_INT4, ANY4_FORMAT_NF4, ANY4_FORMAT_FP4 = 1, 2, 3
FORMATS = {"int4": ANY4_FORMAT_INT4, "nf4": ANY4_FORMAT_NF4, "fp4": ANY4_FORMAT_FP4}

ANY4_OK, ANY4_EINVAL, ANY4_EALIGN, ANY4_ESHAPE, ANY4_EWORKSPACE, ANY4_ECUDA = 0, -1, -2, -3, -4, -5


class Any4Error(RuntimeError):
    def __init__(self, status: int):
        msg = lib.any4_strerror(status).decode()
        if status == ANY4_ECUDA:
            msg += f" (cudaError {lib.any4_last_cuda_error()})"
        super().__init__(msg)
        self.status = status


def _check(status: int) -> None:
    if status != ANY4_OK:
        raise Any4Error(status)


def _dev(t: torch.Tensor, name: str, itemsize: int, shape=None) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.element_size() != itemsize:
        raise ValueError(f"{name} must have {itemsize}-byte elements, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and t.shape != shape:
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t.data_ptr()


# The current stream's raw handle without building a torch Stream object (the
# binding's per-call cost bounds back-to-back calls of small shapes).
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(device: torch.device) -> int:
    if _raw_stream is not None:
        return _raw_stream(device.index if device.index is not None else torch.cuda.current_device())
    return torch.cuda.current_stream(device).cuda_stream


def _stream_of(t: torch.Tensor) -> int:
    if _raw_stream is not None:
        return _raw_stream(t.get_device())
    return torch.cuda.current_stream(t.device).cuda_stream


def any4_packed_bytes(n: int, k: int, group: int) -> int:
    return lib.any4_packed_bytes(n, k, group)


def any4_linear_workspace_bytes(m: int, n: int, k: int, group: int) -> int:
    return lib.any4_linear_workspace_bytes(m, n, k, group)


KERNELS = {1: "shared_tables", 2: "register_tables", 3: "prefill_fused", 4: "prefill_gemm",
           5: "shared_tables_direct"}


def any4_linear_kernel(m: int, n: int, k: int, group: int, bits: int = 4) -> str:
    """Name of the kernel any4_linear runs for this shape on the current device."""
    code = lib.any4_linear_kernel(bits, m, n, k, group)
    if code < 0:
        raise Any4Error(code)
    return KERNELS[code]


def any4_linear_grid(m: int, n: int, k: int, group: int, bits: int = 4) -> tuple[int, int]:
    """(thread blocks, blocks per cluster) of the any4_linear launch for this shape."""
    blocks, cluster = ctypes.c_int(0), ctypes.c_int(0)
    _check(lib.any4_linear_grid(bits, m, n, k, group, ctypes.byref(blocks), ctypes.byref(cluster)))
    return blocks.value, cluster.value


def any4_pack(idx_nib: torch.Tensor, lut: torch.Tensor, alpha: torch.Tensor, beta: torch.Tensor,
              group: int, packed: torch.Tensor | None = None) -> torch.Tensor:
    """Canonical any4 tensors -> device-layout buffer (uint8 tensor)."""
    n, k2 = idx_nib.shape
    k = 2 * k2
    size = any4_packed_bytes(n, k, group)
    if size == 0:
        raise Any4Error(ANY4_ESHAPE)
    dev = idx_nib.device
    if packed is None:
        packed = torch.empty(size, dtype=torch.uint8, device=dev)
    _check(lib.any4_pack(_dev(idx_nib, "idx_nib", 1, (n, k2)), _dev(lut, "lut", 2, (n, 16)),
                         _dev(alpha, "alpha", 2, (n, k // group)),
                         _dev(beta, "beta", 2, (n, k // group)), n, k, group,
                         _dev(packed, "packed", 1), packed.numel(), _stream(dev)))
    return packed


def any4_packed_bytes_bits(bits: int, n: int, k: int, group: int) -> int:
    return lib.any4_packed_bytes_bits(bits, n, k, group)


def any4_pack_bits(bits: int, idx_nib: torch.Tensor, lut: torch.Tensor, alpha: torch.Tensor,
                   beta: torch.Tensor, group: int, packed: torch.Tensor | None = None) -> torch.Tensor:
    """any3 / any2 (bits = 3 / 2; 4 = any4): canonical tensors with indices
    < 2^bits (as nibbles) -> densely packed device-layout buffer."""
    n, k2 = idx_nib.shape
    k = 2 * k2
    size = any4_packed_bytes_bits(bits, n, k, group)
    if size == 0:
        raise Any4Error(ANY4_ESHAPE)
    dev = idx_nib.device
    if packed is None:
        packed = torch.empty(size, dtype=torch.uint8, device=dev)
    _check(lib.any4_pack_bits(bits, _dev(idx_nib, "idx_nib", 1, (n, k2)), _dev(lut, "lut", 2, (n, 16)),
                              _dev(alpha, "alpha", 2, (n, k // group)),
                              _dev(beta, "beta", 2, (n, k // group)), n, k, group,
                              _dev(packed, "packed", 1), packed.numel(), _stream(dev)))
    return packed


def any4_dequant_bits(bits: int, packed: torch.Tensor, n: int, k: int, group: int,
                      out: torch.Tensor | None = None) -> torch.Tensor:
    if out is None:
        out = torch.empty((n, k), dtype=torch.bfloat16, device=packed.device)
    _check(lib.any4_dequant_bits(bits, _dev(packed, "packed", 1), n, k, group, _dev(out, "out", 2, (n, k)),
                                 _stream(packed.device)))
    return out


def any4_linear_bits(bits: int, x: torch.Tensor, packed: torch.Tensor, n: int, k: int, group: int,
                     out: torch.Tensor | None = None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    m = x.shape[0]
    if out is None:
        out = torch.empty((m, n), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = workspace_for(m, n, k, group, x.device, bits)
    _check(lib.any4_linear_bits(bits, _dev(x, "x", 2, (m, k)), _dev(packed, "packed", 1), m, n, k, group,
                                _dev(out, "out", 2, (m, n)), _dev(workspace, "workspace", 1),
                                workspace.numel(), _stream(x.device)))
    return out


def any4_dequant(packed: torch.Tensor, n: int, k: int, group: int,
                 out: torch.Tensor | None = None) -> torch.Tensor:
    """Device-layout buffer -> dequantized W (N x K, bf16)."""
    if out is None:
        out = torch.empty((n, k), dtype=torch.bfloat16, device=packed.device)
    _check(lib.any4_dequant(_dev(packed, "packed", 1), n, k, group, _dev(out, "out", 2, (n, k)),
                            _stream(packed.device)))
    return out


_WORKSPACES: dict = {}


def workspace_for(m: int, n: int, k: int, group: int, device: torch.device, bits: int = 4) -> torch.Tensor:
    """A zero-initialised workspace for this stream, grown on demand and reused
    by later calls on the same stream (calls on one stream never overlap)."""
    need = lib.any4_linear_workspace_bytes_bits(bits, m, n, k, group)
    if need == 0:
        raise Any4Error(ANY4_ESHAPE)
    key = (device.index if device.index is not None else torch.cuda.current_device(),
           _stream(device))
    ws = _WORKSPACES.get(key)
    if ws is None or ws.numel() < need:
        ws = torch.zeros(max(need, 1 << 20), dtype=torch.uint8, device=device)
        _WORKSPACES[key] = ws
    return ws


def any4_linear(x: torch.Tensor, packed: torch.Tensor, n: int, k: int, group: int,
                out: torch.Tensor | None = None,
                workspace: torch.Tensor | None = None) -> torch.Tensor:
    """y = x . W_hat^T for bf16 x (M x K) -> y (M x N, bf16). M <= 16 runs the
    fused decode kernel, M > 16 the dequantize-then-GEMM prefill path."""
    m = x.shape[0]
    if out is None:
        out = torch.empty((m, n), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = workspace_for(m, n, k, group, x.device)
    st = lib.any4_linear(_dev(x, "x", 2, (m, k)), _dev(packed, "packed", 1), m, n, k, group,
                         _dev(out, "out", 2, (m, n)), _dev(workspace, "workspace", 1),
                         workspace.numel(), _stream_of(x))
    if st != ANY4_OK:
        raise Any4Error(st)
    return out


def any4_linear_noalloc(x: torch.Tensor, packed: torch.Tensor, n: int, k: int, group: int,
                        out: torch.Tensor | None = None) -> torch.Tensor:
    """any4_linear without a workspace, for callers that cannot allocate device
    memory (e.g. an operator inside a runtime that owns all device memory): the
    library's own fixed scratch array is used instead. Calls that may overlap
    on the GPU must be ordered by the caller, since they share that array.
    ``out`` may be passed to avoid the one allocation this Python helper makes."""
    m = x.shape[0]
    if out is None:
        out = torch.empty((m, n), dtype=torch.bfloat16, device=x.device)
    _check(lib.any4_linear_noalloc(_dev(x, "x", 2, (m, k)), _dev(packed, "packed", 1), m, n, k,
                                   group, _dev(out, "out", 2, (m, n)), _stream(x.device)))
    return out


class _DeviceWord:
    """A 32-bit device word exposed through the CUDA array interface."""

    def __init__(self, ptr: int):
        self.__cuda_array_interface__ = {"shape": (1,), "typestr": "<u4", "data": (ptr, False),
                                         "version": 3}


def noalloc_status(device: torch.device | None = None) -> int:
    """The status word of any4_linear_noalloc on ``device`` (0: the last call
    completed normally). Synchronizes that device before reading it."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    with torch.cuda.device(dev):
        ptr = _p()
        _check(lib.any4_noalloc_status_word(ctypes.byref(ptr)))
        torch.cuda.synchronize(dev)
        word = torch.as_tensor(_DeviceWord(ptr.value), device=dev)
        return int(word.view(torch.int32).item()) & 0xFFFFFFFF


def any4_quantize(w: torch.Tensor, ex: torch.Tensor, group: int, bits: int = 4,
                  iters: int = 10):
    """GPU any4 quantizer: bf16 W (N x K) and float64 E|x| (K) -> the canonical
    tensors (idx_nib, lut, alpha, beta) as int16/uint8 device tensors."""
    n, k = w.shape
    dev = w.device
    idx_nib = torch.empty((n, k // 2), dtype=torch.uint8, device=dev)
    lut = torch.empty((n, 16), dtype=torch.int16, device=dev)
    alpha = torch.empty((n, k // group), dtype=torch.int16, device=dev)
    beta = torch.empty((n, k // group), dtype=torch.int16, device=dev)
    if ex.dtype != torch.float64:
        raise ValueError("ex must be float64")
    _check(lib.any4_quantize(_dev(w, "w", 2, (n, k)), _dev(ex, "ex", 8, (k,)), n, k, group, bits,
                             iters, _dev(idx_nib, "idx_nib", 1), _dev(lut, "lut", 2),
                             _dev(alpha, "alpha", 2), _dev(beta, "beta", 2), _stream(dev)))
    return idx_nib, lut, alpha, beta


def _format_code(fmt) -> int:
    return FORMATS[fmt] if isinstance(fmt, str) else int(fmt)


def any4_format_lut(fmt) -> list:
    """The 16 bf16 bit patterns of a fixed-table format ("int4", "nf4", "fp4"),
    by code. Host only."""
    buf = (ctypes.c_uint16 * 16)()
    _check(lib.any4_format_lut(_format_code(fmt), ctypes.cast(buf, _p)))
    return [int(v) for v in buf]


def any4_pack_format(fmt, idx_nib: torch.Tensor, alpha: torch.Tensor, beta: torch.Tensor,
                     group: int, packed: torch.Tensor | None = None) -> torch.Tensor:
    """Fixed-table format codes + alpha/beta -> device-layout buffer; the
    format's table goes to every row, so any4_dequant / any4_linear apply."""
    n, k2 = idx_nib.shape
    k = 2 * k2
    size = any4_packed_bytes(n, k, group)
    if size == 0:
        raise Any4Error(ANY4_ESHAPE)
    dev = idx_nib.device
    if packed is None:
        packed = torch.empty(size, dtype=torch.uint8, device=dev)
    _check(lib.any4_pack_format(_format_code(fmt), _dev(idx_nib, "idx_nib", 1, (n, k2)),
                                _dev(alpha, "alpha", 2, (n, k // group)),
                                _dev(beta, "beta", 2, (n, k // group)), n, k, group,
                                _dev(packed, "packed", 1), packed.numel(), _stream(dev)))
    return packed


def any4_strerror(status: int) -> str:
    return lib.any4_strerror(status).decode()
