"""GPU parity of any4_quantize (group scaling + per-row weighted k-means)
against the oracle's quantize: the canonical tensors must be bit-identical
(indices, bf16 tables, alpha, beta), for any4, any3 and any2.

Both sides evaluate the same float64 operations in the same order (each
cluster sum over the row's columns in increasing order), so equality is
exact; a mismatch means one side departs from the steps of the explainer's
sections 2.1 and 2.2.
"""
import numpy as np
import pytest
import torch

import learned_bit_lut_b200 as a4
import oracle
import synth
from gpu_util import bits_host, calib, require_gpu, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    torch.cuda.set_device(0)


def _gpu_quantize(w_bits, ex, g, bits, iters=10):
    out = a4.any4_quantize(to_dev(w_bits).view(torch.int16), torch.from_numpy(ex).cuda(), g,
                           bits, iters)
    torch.cuda.synchronize()
    idx, lut, al, be = out
    return (idx.cpu().numpy(), bits_host(lut), bits_host(al), bits_host(be))


def _assert_same(got, q, rows=None):
    idx, lut, al, be = got
    if rows is not None:
        idx, lut, al, be = idx[rows], lut[rows], al[rows], be[rows]
    np.testing.assert_array_equal(al, q.alpha)
    np.testing.assert_array_equal(be, q.beta)
    np.testing.assert_array_equal(lut, q.lut)
    np.testing.assert_array_equal(idx, q.idx_nib)


@pytest.mark.parametrize("bits", [4, 3, 2])
@pytest.mark.parametrize("n,k,g", [(256, 512, 128), (96, 2112, 64), (64, 4096, 1024)])
def test_quantize_bit_identical(bits, n, k, g):
    w = synth.weights_bf16(n, k, 21, layer=f"q{n}x{k}")
    _, ex = calib(k, 21, f"q{n}x{k}")
    got = _gpu_quantize(w, ex, g, bits)
    _assert_same(got, oracle.quantize(w, ex, g, 10, bits=bits))


def test_quantize_student_t_and_degenerate_rows():
    # heavy tails, a constant row (alpha = 0) and rows with few distinct values
    n, k, g = 64, 1024, 128
    w = synth.weights_bf16(n, k, 22, kind="student_t", layer="qdeg")
    w[0] = w[0, 0]                                    # constant row
    w[1] = np.where(np.arange(k) % 3 == 0, w[1, 0], w[1, 1])   # two values
    w[2, :] = oracle.f64_to_bf16_bits(np.tile(np.arange(-8.0, 8.0), k // 16) * 0.01)
    _, ex = calib(k, 22, "qdeg")
    got = _gpu_quantize(w, ex, g, 4)
    _assert_same(got, oracle.quantize(w, ex, g, 10))


def test_quantize_full_size_sampled_rows():
    n, k, g = 14336, 4096, 128
    w = synth.weights_bf16(n, k, 23, layer="qgate")
    _, ex = calib(k, 23, "qgate")
    got = _gpu_quantize(w, ex, g, 4)
    rows = np.array(sorted(set(range(8)) | set(range(n - 8, n)) |
                           set(np.random.default_rng(4).choice(n, 24, replace=False).tolist())))
    _assert_same(got, oracle.quantize(w, ex, g, 10, rows=rows), rows)


def test_quantized_weights_run_through_the_linear():
    # GPU quantizer -> pack -> linear, checked against the oracle on the same tensors
    from gpu_util import check_linear, bf16_dev
    n, k, g = 512, 4096, 128
    w = synth.weights_bf16(n, k, 24, layer="qlin")
    s, ex = calib(k, 24, "qlin")
    idx, lut, al, be = a4.any4_quantize(to_dev(w).view(torch.int16), torch.from_numpy(ex).cuda(), g)
    packed = a4.any4_pack(idx, lut, al, be, g)
    q = oracle.Any4Tensors(idx.cpu().numpy(), bits_host(lut), bits_host(al), bits_host(be), g)
    x = synth.activations_bf16(4, s, 25, layer="qlin")
    check_linear(a4.any4_linear(bf16_dev(x), packed, n, k, g), x, q)
