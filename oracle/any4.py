"""any4 oracle: quantizer, bit-exact dequantization and fp64 linear (test infrastructure).

Plain, slow CPU code that follows the method step by step, in float64. It is
the parity reference for the CUDA library and shares no code with it.

Sources (page title and section):

* the any4 explainer (10100.com, article 149119421):
  - §一 comparison table: int4 is uniform scaling with a fixed integer map
    -8..7; NF4 is a fixed table of 16 Gaussian-fitted values; any4 adds
    0.0625 bit per entry.
  - §二 intro: each row of W has its own table (LUT) of 16 FP16/BF16 values;
    every weight stores a 4-bit index and inference reads the table value at
    that index.
  - §二.1 "分组缩放" (group scaling): rows are split into contiguous groups
    (usually 128 columns); each group gets a scale alpha and an offset beta
    that map the weights into the quantizable range, exactly as in ordinary
    group quantization.
  - §二.1 "激活校准" (calibration): one calibration sample is run through the
    model; per input channel the mean absolute activation E|x| is recorded.
  - §二.2 E-step: with the 16 table values fixed, every scaled weight is
    assigned to its nearest table value.
  - §二.2 M-step: LUT_q = sum(alpha * w_s * E|x|) / sum(alpha * E|x|) over the
    weights assigned to q, w_s being the group-scaled weight; E and M steps
    alternate until convergence.
  - §二.3: the 16-entry table costs 0.0625 bit per weight at 4096 columns.
* "any4: Learned 4-bit Numeric Representation for LLMs" (arXiv 2507.04610
  summary page, abstract): per-row learned 4-bit numeric representation,
  calibrated with a single curated sample.

Readings where the pages are silent (each also listed in the design notes):

* group scaling is asymmetric min-max onto the int4 range [-8, 7]:
  alpha = (max - min) / 15, beta = min + 8 * alpha, both rounded to bf16
  (nearest-even) and used rounded from then on; w_s = (w - beta) / alpha, and
  w_s = 0 for a constant group (alpha == 0);
* the objective both steps decrease is J = sum_k c_k (w_s,k - LUT[idx_k])^2
  with c_k = alpha_g(k) * E|x|_k;
* initial table: the sorted distinct w_s values of the row when there are at
  most 16 (the last one repeated to fill 16 slots), else the int4 grid
  -8..7, so the first E-step is int4 rounding;
* ties in the E-step go to the lowest index; an empty cluster keeps its
  value; 10 E/M rounds; then the table is rounded to bf16 (nearest-even) and
  one last E-step assigns every weight against the stored bf16 table;
* dequantization is w_hat = fma(alpha, LUT[idx], beta): the exact value
  rounded once to fp32, then rounded to bf16 (both nearest-even);
* the linear layer is y = x . W_hat^T over bf16 x, computed in float64.

Canonical tensors (the layout the CUDA library's pack call consumes):
``idx_nib`` uint8 N x K/2 (byte j of row n holds k = 2j in its low nibble and
k = 2j+1 in its high nibble), ``lut`` uint16 N x 16 (bf16 bits), ``alpha`` and
``beta`` uint16 N x K/G (bf16 bits).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .bf16 import bf16_bits_to_f64, f32_to_bf16_bits, f64_to_bf16_bits, fma_to_f32

INT4_GRID = np.arange(-8.0, 8.0)          # the fixed int4 integer map -8..7


def int_grid(bits: int) -> np.ndarray:
    """The signed integer map of a b-bit code: -2^(b-1) .. 2^(b-1)-1 (float64).

    For b = 4 this is the int4 map -8..7 of the explainer's §一; the any3 and
    any2 variants (named on the arXiv summary page) use the 3- and 2-bit maps
    [reading].
    """
    h = 1 << (bits - 1)
    return np.arange(-h, h, dtype=np.float64)
_CHUNK_ELEMS = 1 << 19                     # rows per chunk = this // K


@dataclass
class Any4Tensors:
    """Quantized weight in the canonical layout (all arrays uint8 / uint16)."""
    idx_nib: np.ndarray
    lut: np.ndarray
    alpha: np.ndarray
    beta: np.ndarray
    group: int
    bits: int = 4          # indices use values < 2**bits; lut columns past that repeat

    @property
    def n(self) -> int:
        return self.lut.shape[0]

    @property
    def k(self) -> int:
        return self.idx_nib.shape[1] * 2


# ----------------------------------------------------------------- nibbles

def pack_nibbles(idx: np.ndarray) -> np.ndarray:
    """N x K indices (0..15) -> N x K/2 bytes, even k in the low nibble."""
    idx = np.asarray(idx, dtype=np.uint8)
    if idx.max(initial=0) > 15:
        raise ValueError("index out of range")
    return (idx[:, 0::2] | (idx[:, 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(idx_nib: np.ndarray) -> np.ndarray:
    """N x K/2 bytes -> N x K indices."""
    b = np.asarray(idx_nib, dtype=np.uint8)
    out = np.empty((b.shape[0], b.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = b & 0x0F
    out[:, 1::2] = b >> 4
    return out


# ----------------------------------------------------------- group scaling

def group_scale(w_bits: np.ndarray, g: int, bits: int = 4):
    """Per-group alpha, beta (bf16 bits) and the scaled weights w_s (float64).

    Follows the group-scaling step (explainer §二.1): contiguous groups of g
    columns in each row; asymmetric min-max onto [-8, 7] (for b bits onto
    [-2^(b-1), 2^(b-1)-1], i.e. alpha = (max-min)/(2^b-1), beta = min +
    2^(b-1) alpha [reading]).
    """
    w = bf16_bits_to_f64(w_bits)
    n, k = w.shape
    if k % g:
        raise ValueError("K must be a multiple of the group size")
    wg = w.reshape(n, k // g, g)
    lo = wg.min(axis=2)
    hi = wg.max(axis=2)
    levels = float((1 << bits) - 1)
    half = float(1 << (bits - 1))
    alpha_bits = f64_to_bf16_bits((hi - lo) / levels)
    alpha = bf16_bits_to_f64(alpha_bits)
    beta_bits = f64_to_bf16_bits(lo + half * alpha)
    beta = bf16_bits_to_f64(beta_bits)
    a = alpha[:, :, None]
    safe = np.where(a == 0.0, 1.0, a)
    ws = np.where(a == 0.0, 0.0, (wg - beta[:, :, None]) / safe)
    return alpha_bits, beta_bits, ws.reshape(n, k)


# -------------------------------------------------------------- calibration

def calibrate(x_cal: np.ndarray) -> np.ndarray:
    """E|x| per input channel: mean over the calibration tokens of |x|
    (explainer §二.1, activation calibration)."""
    return np.mean(np.abs(np.asarray(x_cal, dtype=np.float64)), axis=0)


def kmeans_weights(alpha_bits: np.ndarray, ex: np.ndarray, g: int) -> np.ndarray:
    """c[n, k] = alpha[n, group(k)] * E|x|[k], the M-step weight (explainer §二.2)."""
    a = np.repeat(bf16_bits_to_f64(alpha_bits), g, axis=1)
    return a * np.asarray(ex, dtype=np.float64)[None, :]


# ---------------------------------------------------------------- k-means

def init_lut(ws: np.ndarray, bits: int = 4) -> np.ndarray:
    """Initial 2^b-entry table per row (reading: distinct values or the
    integer grid)."""
    size = 1 << bits
    lut = np.tile(int_grid(bits), (ws.shape[0], 1))
    for r in range(ws.shape[0]):
        u = np.unique(ws[r])
        if u.size <= size:
            lut[r, :u.size] = u
            lut[r, u.size:] = u[-1]
    return lut


def e_step(ws: np.ndarray, lut: np.ndarray) -> np.ndarray:
    """Nearest table entry for every scaled weight; lowest index on ties
    (explainer §二.2, E-step)."""
    d = np.abs(ws[:, :, None] - lut[:, None, :])
    return np.argmin(d, axis=2).astype(np.uint8)


def m_step(ws: np.ndarray, c: np.ndarray, idx: np.ndarray, lut: np.ndarray) -> np.ndarray:
    """LUT_q = sum(c * w_s) / sum(c) over the weights assigned to q
    (explainer §二.2, M-step, c = alpha * E|x|).

    Written as LUT_q + sum(c * (w_s - LUT_q)) / sum(c), which is the same
    quotient; the shift by the current value keeps a cluster of identical
    values at exactly that value in float64. A cluster with sum(c) == 0 keeps
    its value.
    """
    r, size = lut.shape
    slot = (np.arange(r)[:, None] * size + idx).ravel()
    cur = np.take_along_axis(lut, idx.astype(np.int64), axis=1)
    den = np.bincount(slot, weights=c.ravel(), minlength=r * size).reshape(r, size)
    num = np.bincount(slot, weights=(c * (ws - cur)).ravel(), minlength=r * size).reshape(r, size)
    out = lut.copy()
    nz = den > 0.0
    out[nz] = lut[nz] + num[nz] / den[nz]
    return out


def objective(ws: np.ndarray, c: np.ndarray, idx: np.ndarray, lut: np.ndarray) -> np.ndarray:
    """J per row = sum_k c_k (w_s,k - LUT[idx_k])^2."""
    v = np.take_along_axis(lut, idx.astype(np.int64), axis=1)
    return np.sum(c * (ws - v) ** 2, axis=1)


def kmeans_rows(ws: np.ndarray, c: np.ndarray, iters: int = 10, history: bool = False,
                bits: int = 4):
    """Weighted 1-D k-means with 2^bits (16 for any4) centres for each row of ws.

    Returns ``(idx, lut_bits)`` (and the per-row objective after every E and
    M step when ``history``): ``iters`` E/M rounds from ``init_lut``, then the
    table is rounded to bf16 and a last E-step runs against it.
    """
    lut = init_lut(ws, bits)
    hist = []
    for _ in range(iters):
        idx = e_step(ws, lut)
        if history:
            hist.append(objective(ws, c, idx, lut))
        lut = m_step(ws, c, idx, lut)
        if history:
            hist.append(objective(ws, c, idx, lut))
    lut_bits = f64_to_bf16_bits(lut)
    idx = e_step(ws, bf16_bits_to_f64(lut_bits))
    if history:
        return idx, lut_bits, np.stack(hist, axis=1) if hist else np.zeros((ws.shape[0], 0))
    return idx, lut_bits


def quantize(w_bits: np.ndarray, ex: np.ndarray, g: int = 128, iters: int = 10,
             rows=None, bits: int = 4) -> Any4Tensors:
    """any4 quantization of a bf16 weight matrix (all rows, or ``rows`` only).

    Group scaling -> c = alpha * E|x| -> per-row weighted k-means, processed
    in row chunks to bound memory. ``bits`` = 3 or 2 gives the any3 / any2
    variants (8- and 4-entry tables); their tables are returned padded to 16
    columns by repeating the last entry, so the same canonical tensors and
    device layout serve every width.
    """
    w_bits = np.asarray(w_bits, dtype=np.uint16)
    if rows is not None:
        w_bits = w_bits[np.asarray(rows)]
    n, k = w_bits.shape
    idx_nib = np.empty((n, k // 2), dtype=np.uint8)
    lut = np.empty((n, 16), dtype=np.uint16)
    alpha = np.empty((n, k // g), dtype=np.uint16)
    beta = np.empty((n, k // g), dtype=np.uint16)
    step = max(1, _CHUNK_ELEMS // k)
    for r0 in range(0, n, step):
        r1 = min(n, r0 + step)
        a_bits, b_bits, ws = group_scale(w_bits[r0:r1], g, bits)
        c = kmeans_weights(a_bits, ex, g)
        idx, l_bits = kmeans_rows(ws, c, iters, bits=bits)
        idx_nib[r0:r1] = pack_nibbles(idx)
        size = 1 << bits
        lut[r0:r1, :size] = l_bits
        lut[r0:r1, size:] = l_bits[:, size - 1:size]
        alpha[r0:r1] = a_bits
        beta[r0:r1] = b_bits
    return Any4Tensors(idx_nib, lut, alpha, beta, g, bits)


# ------------------------------------------------------------ dequantize

def dequant_rows(q: Any4Tensors, rows=None) -> np.ndarray:
    """Bit-exact dequantized weights (bf16 bits) for all rows or ``rows``.

    w_hat[n, k] = bf16( fp32( alpha[n, g(k)] * LUT[n, idx[n, k]] + beta[n, g(k)] ) )
    (explainer §二 intro and §二.1), one fused multiply-add rounded to fp32,
    then rounded to bf16.
    """
    sel = np.arange(q.n) if rows is None else np.asarray(rows)
    out = np.empty((sel.size, q.k), dtype=np.uint16)
    step = max(1, _CHUNK_ELEMS // q.k)
    for i0 in range(0, sel.size, step):
        r = sel[i0:i0 + step]
        idx = unpack_nibbles(q.idx_nib[r]).astype(np.int64)
        l = np.take_along_axis(bf16_bits_to_f64(q.lut[r]), idx, axis=1)
        a = np.repeat(bf16_bits_to_f64(q.alpha[r]), q.group, axis=1)
        b = np.repeat(bf16_bits_to_f64(q.beta[r]), q.group, axis=1)
        out[i0:i0 + r.size] = f32_to_bf16_bits(fma_to_f32(a, l, b))
    return out


def dequant(q: Any4Tensors) -> np.ndarray:
    return dequant_rows(q)


def linear_rows(x_bits: np.ndarray, q: Any4Tensors, rows=None) -> np.ndarray:
    """y[m, n] = sum_k x[m, k] * w_hat[n, k] in float64 (M x len(rows))."""
    x = bf16_bits_to_f64(np.asarray(x_bits, dtype=np.uint16))
    w = bf16_bits_to_f64(dequant_rows(q, rows))
    return x @ w.T


def linear(x_bits: np.ndarray, q: Any4Tensors) -> np.ndarray:
    return linear_rows(x_bits, q)


def algorithmic_bytes(m: int, n: int, k: int, g: int) -> int:
    """Bytes one call must move: 4-bit indices, alpha/beta and LUT (bf16),
    x and y (bf16)."""
    return n * k // 2 + n * (k // g) * 4 + n * 32 + m * k * 2 + m * n * 2
