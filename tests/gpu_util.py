"""Helpers shared by the GPU parity tests: canonical any4 tensors from the
oracle (or drawn directly for full-size shapes), device copies, and the
comparison rules."""
from __future__ import annotations

import functools

import numpy as np
import torch

import oracle
import synth

# Acceptance bar of the linear layer: per token row m,
#   max_n |y - y_ref| <= REL_TOL * max_n |y_ref|.
REL_TOL = 2e-2


def require_gpu():
    assert torch.cuda.is_available(), "these tests need a CUDA GPU"
    return torch.device("cuda:0")


def to_dev(a: np.ndarray, device="cuda:0") -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(device)
    return torch.from_numpy(a).to(device)


def bf16_dev(bits: np.ndarray, device="cuda:0") -> torch.Tensor:
    return to_dev(bits, device).view(torch.bfloat16)


def bits_host(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def calib(k: int, seed: int, layer: str, sigma: float = 0.5):
    s = synth.channel_scale(k, seed, sigma=sigma, layer=layer)
    ex = oracle.calibrate(synth.calibration_acts(512, s, seed, layer=layer))
    return s, ex


@functools.lru_cache(maxsize=None)
def quantized(n: int, k: int, g: int, seed: int = 0, layer: str = "w", kind: str = "normal",
              sigma: float = 0.5, iters: int = 10):
    """Oracle-quantized weight (all rows) and its activation scale."""
    w = synth.weights_bf16(n, k, seed, kind=kind, layer=layer)
    s, ex = calib(k, seed, layer, sigma)
    return oracle.quantize(w, ex, g=g, iters=iters), s


@functools.lru_cache(maxsize=None)
def mixed(n: int, k: int, g: int, rows: tuple, seed: int = 0, layer: str = "w",
          kind: str = "normal", sigma: float = 0.5):
    """Full-size any4 tensors: directly drawn rows everywhere, oracle-quantized
    rows (k-means on synthetic weights of the workload's distribution) at
    ``rows``. Returns (tensors, activation scale)."""
    idx, lut, a, b = synth.random_any4(n, k, g, seed, layer=layer)
    w = synth.weights_bf16(len(rows), k, seed, kind=kind, layer=layer + "/rows")
    s, ex = calib(k, seed, layer, sigma)
    q = oracle.quantize(w, ex, g=g, iters=10)
    r = np.asarray(rows)
    idx[r], lut[r], a[r], b[r] = q.idx_nib, q.lut, q.alpha, q.beta
    return oracle.Any4Tensors(idx, lut, a, b, g), s


def split_panels(n: int, k: int, g: int, m: int = 1, bits: int = 4) -> list:
    """32-row panels whose K range the any4_linear launch for this shape splits
    between thread blocks (stream-K): a block owns units (panel, 64-column
    chunk) floor(b*U/C) .. floor((b+1)*U/C) - 1 of U = panels * K/64, so a
    block boundary that falls inside a panel splits it (that panel is the
    last of block b - 1 and the first of block b). Empty when the launch
    gives whole panels or clusters to blocks."""
    import learned_bit_lut_b200 as a4
    blocks, cluster = a4.any4_linear_grid(m, n, k, g, bits=bits)
    panels, kc = (n + 31) // 32, k // 64
    units = panels * kc
    if cluster > 1 or blocks * kc == units:
        return []
    cuts = (b * units // blocks for b in range(1, blocks))
    return sorted({u // kc for u in cuts if u % kc})


def sample_rows(n: int, count: int = 48, seed: int = 0, whole_panels: int = 4, split_of=None) -> tuple:
    """Rows of the first and last tiles, spread random rows, and every row of
    ``whole_panels`` 32-row panels (the first, the last and random ones).

    At the benchmark shapes every panel of the any4 decode kernel is split
    along K between several warps and finished by the last one to arrive, so
    whole panels check that reduction element by element. With ``split_of =
    (k, g)`` the random panels are drawn from the panels that the launch
    splits between thread blocks (``split_panels``; the first and the last
    of them always), which checks the stream-K finisher element by element."""
    g = np.random.default_rng(seed)
    pick = set(range(min(16, n))) | set(range(max(0, n - 16), n))
    pick |= set(g.choice(n, size=min(n, count), replace=False).tolist())
    panels = (n + 31) // 32
    chosen = {0, panels - 1}
    pool = split_panels(n, *split_of) if split_of is not None else []
    if pool:
        chosen |= {pool[0], pool[-1]}
        chosen |= set(g.choice(pool, size=min(len(pool), max(0, whole_panels - 2)), replace=False).tolist())
    else:
        chosen |= set(g.choice(panels, size=min(panels, max(0, whole_panels - 2)), replace=False).tolist())
    for p in sorted(chosen):
        pick |= set(range(32 * p, min(n, 32 * p + 32)))
    return tuple(sorted(pick))


def pack_dev(q: oracle.Any4Tensors, device="cuda:0"):
    import learned_bit_lut_b200 as a4
    return a4.any4_pack(to_dev(q.idx_nib, device), to_dev(q.lut, device), to_dev(q.alpha, device),
                        to_dev(q.beta, device), q.group)


def check_linear(y_gpu: torch.Tensor, x_bits: np.ndarray, q: oracle.Any4Tensors, rows=None):
    """Compare y (M x N, bf16 on the GPU) with the oracle on ``rows`` (all if None).

    Two bars: the acceptance bar (REL_TOL of each token row's max |y_ref|) and
    a tight elementwise bar (half a bf16 ulp of the output plus fp32
    accumulation error), since the kernel contracts the same bf16 weights.
    """
    y = y_gpu.float().cpu().numpy().astype(np.float64)
    ref = oracle.linear_rows(x_bits, q, rows)
    if rows is not None:
        y = y[:, np.asarray(rows)]
    scale = np.max(np.abs(ref), axis=1, keepdims=True)
    err = np.abs(y - ref)
    worst = np.max(err / np.maximum(scale, 1e-30), axis=1)
    assert np.all(worst <= REL_TOL), f"relative error per token {worst}"
    tight = np.abs(ref) * 2.0 ** -8 + 1e-4 * scale
    bad = np.argwhere(err > tight)
    assert bad.size == 0, f"{len(bad)} elements off, first {bad[:5].tolist()}"
    return float(worst.max())
