"""Seeded synthetic inputs for the any4 linear layer.

This module is shared by the tests, the benchmark and the oracle checks. It
holds random-number recipes only: none of the any4 arithmetic (group scaling,
calibration statistics, k-means, dequantization, the contraction) lives here.

Recipes (the workloads are the synthetic Llama-shaped layers of the any4
benchmark configurations; no model weights or datasets are used):

* weights: ``N(0, std)`` with ``std = 0.02``; ``round(0.001*N*K)`` distinct,
  uniformly chosen positions are multiplied by 8 ("0.1 % outliers x8"). The
  70B-shape sweep instead draws ``0.015 * StudentT(nu=5)`` with no outliers.
  Values are drawn in float64, rounded to float32 and then to bf16 (both
  round-to-nearest-even, done by torch's casts).
* per-channel activation scale ``s_k ~ LogNormal(0, sigma)`` (sigma 0.5, or
  0.7 for the 70B-shape sweep).
* calibration activations (the single calibration sample): ``T`` tokens of
  ``z * s_k`` with ``z ~ N(0, 1)``, kept in float64.
* test activations ``x = z * s_k`` rounded to bf16.
* ``random_any4``: valid any4 tensors drawn directly (uniform 4-bit indices,
  16 sorted LUT values per row in [-8, 7], positive scales, small offsets).
  They stand in for quantizer output where only the data layout matters
  (timing, full-size sampled checks).

Every draw comes from its own named sub-stream of ``SeedSequence(seed)`` so
adding a draw never shifts another one.
"""
from __future__ import annotations

import zlib
from dataclasses import dataclass

import numpy as np
import torch

__all__ = [
    "rng", "weights_bf16", "channel_scale", "calibration_acts",
    "activations_bf16", "random_any4", "Shape", "LLAMA3_8B_LAYER",
    "LLAMA3_8B_MLP", "WORKLOADS",
]


def rng(seed: int, *names: str) -> np.random.Generator:
    """Independent generator for the sub-stream ``names`` of ``seed``."""
    key = tuple(zlib.crc32(n.encode()) for n in names)
    return np.random.default_rng(np.random.SeedSequence(entropy=seed, spawn_key=key))


def _to_bf16_bits(a64: np.ndarray) -> np.ndarray:
    """float64 -> float32 -> bf16 (RNE at each step, by numpy and torch casts)."""
    t = torch.from_numpy(np.ascontiguousarray(a64, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def weights_bf16(n: int, k: int, seed: int, kind: str = "normal", layer: str = "w",
                 std: float = 0.02, outlier_frac: float = 0.001, outlier_mult: float = 8.0,
                 t_scale: float = 0.015, t_nu: float = 5.0) -> np.ndarray:
    """Weight matrix W (N x K, row = output channel) as bf16 bit patterns."""
    g = rng(seed, layer, "weights")
    if kind == "normal":
        w = g.normal(0.0, std, size=(n, k))
        n_out = int(round(outlier_frac * n * k))
        if n_out:
            pos = rng(seed, layer, "outliers").choice(n * k, size=n_out, replace=False)
            w.reshape(-1)[pos] *= outlier_mult
    elif kind == "student_t":
        w = t_scale * g.standard_t(t_nu, size=(n, k))
    else:
        raise ValueError(f"unknown weight distribution {kind!r}")
    return _to_bf16_bits(w)


def channel_scale(k: int, seed: int, sigma: float = 0.5, layer: str = "w") -> np.ndarray:
    """Per-input-channel activation scale s_k ~ LogNormal(0, sigma), float64."""
    return rng(seed, layer, "channel_scale").lognormal(0.0, sigma, size=k)


def calibration_acts(t: int, s: np.ndarray, seed: int, layer: str = "w") -> np.ndarray:
    """The calibration sample: T tokens x K channels of z * s_k (float64)."""
    z = rng(seed, layer, "calibration").standard_normal((t, s.shape[0]))
    return z * s[None, :]


def activations_bf16(m: int, s: np.ndarray, seed: int, layer: str = "w") -> np.ndarray:
    """Test activations x (M x K) = z * s_k as bf16 bit patterns."""
    z = rng(seed, layer, "activations").standard_normal((m, s.shape[0]))
    return _to_bf16_bits(z * s[None, :])


def random_any4(n: int, k: int, g: int, seed: int, layer: str = "w"):
    """Directly drawn any4 tensors in the canonical layout.

    Returns ``(idx_nib, lut, alpha, beta)``: uint8 N x K/2 nibbles (low nibble
    = even k), uint16 N x 16 bf16 LUT, uint16 N x K/G bf16 scale and offset.
    """
    r = rng(seed, layer, "random_any4")
    idx_nib = r.integers(0, 256, size=(n, k // 2), dtype=np.uint8)
    lut = np.sort(r.uniform(-8.0, 7.0, size=(n, 16)), axis=1)
    alpha = 0.02 * 8.0 / 15.0 * r.lognormal(0.0, 0.3, size=(n, k // g))
    beta = r.normal(0.0, 0.005, size=(n, k // g))
    return idx_nib, _to_bf16_bits(lut), _to_bf16_bits(alpha), _to_bf16_bits(beta)


@dataclass(frozen=True)
class Shape:
    name: str
    n: int
    k: int


# One Llama-3-8B decoder layer's linears (q, k, v, o, gate, up, down).
LLAMA3_8B_LAYER = (
    Shape("q", 4096, 4096), Shape("k", 1024, 4096), Shape("v", 1024, 4096),
    Shape("o", 4096, 4096), Shape("gate", 14336, 4096), Shape("up", 14336, 4096),
    Shape("down", 4096, 14336),
)
LLAMA3_8B_MLP = (Shape("gate", 14336, 4096), Shape("up", 14336, 4096), Shape("down", 4096, 14336))

# The five benchmark workloads: shapes, batch sizes M, group sizes G and the
# weight / activation recipe of each.
WORKLOADS = {
    "single_256x512": dict(shapes=(Shape("w", 256, 512),), ms=(1,), gs=(128,),
                          kind="normal", sigma=0.5, kmeans_iters=10),
    "llama2_7b_attn_4096": dict(shapes=(Shape("proj", 4096, 4096),), ms=(1, 4, 16), gs=(128,),
                               kind="normal", sigma=0.5, kmeans_iters=10),
    "llama3_8b_mlp": dict(shapes=LLAMA3_8B_MLP, ms=(1, 2, 4, 8, 16), gs=(128,),
                         kind="normal", sigma=0.5, kmeans_iters=10),
    "llama3_70b_mlp_gsweep": dict(shapes=(Shape("mlp", 28672, 8192),), ms=(1, 16),
                                 gs=(64, 128, 256, 1024), kind="student_t", sigma=0.7,
                                 kmeans_iters=10),
    "llama3_8b_stack": dict(shapes=LLAMA3_8B_LAYER, layers=32, ms=(1, 16), gs=(128,),
                           kind="normal", sigma=0.5, kmeans_iters=10),
}
