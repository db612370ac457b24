"""GPU parity of the dense any3 / any2 packing (the *_bits calls) against the
fp64 oracle: weights quantized by the oracle with 3 or 2 bits per index,
packed with 2b-bit row-pair codes; dequant must be bit-exact, the linear
layer (decode kernels for M <= 16, prefill for M > 16) must meet both bars.
bits = 4 through the *_bits calls must be the any4 path itself."""
import numpy as np
import pytest
import torch

import learned_bit_lut_b200 as a4
import oracle
import synth
from gpu_util import bf16_dev, bits_host, calib, check_linear, pack_dev, require_gpu, sample_rows, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    torch.cuda.set_device(0)


def pack_bits(bits: int, q: oracle.Any4Tensors):
    return a4.any4_pack_bits(bits, to_dev(q.idx_nib), to_dev(q.lut), to_dev(q.alpha), to_dev(q.beta), q.group)


def quantized_bits(bits, n, k, g, layer, iters=6):
    w = synth.weights_bf16(n, k, 21, layer=layer)
    s, ex = calib(k, 21, layer)
    return oracle.quantize(w, ex, g, iters=iters, bits=bits), s


@pytest.mark.parametrize("bits", [3, 2])
@pytest.mark.parametrize("n,k,g", [(256, 512, 128), (1024, 4096, 128), (160, 2112, 64), (48, 1024, 1024),
                                   (4096, 1024, 256)])
def test_bits_dequant_bitexact_and_linear(bits, n, k, g):
    q, s = quantized_bits(bits, n, k, g, f"b{bits}_{n}x{k}")
    assert int(q.idx_nib.max() & 0xF) < (1 << bits) and int(q.idx_nib.max() >> 4) < (1 << bits)
    packed = pack_bits(bits, q)
    assert packed.numel() == a4.any4_packed_bytes_bits(bits, n, k, g)
    wd = a4.any4_dequant_bits(bits, packed, n, k, g)
    np.testing.assert_array_equal(bits_host(wd), oracle.dequant(q))
    for m in (1, 5, 16, 33):
        x = synth.activations_bf16(m, s, 22 + m, layer=f"b{bits}_{n}x{k}")
        y = a4.any4_linear_bits(bits, bf16_dev(x), packed, n, k, g)
        check_linear(y, x, q)


@pytest.mark.parametrize("bits", [3, 2])
@pytest.mark.parametrize("m", [1, 16])
def test_bits_llama3_8b_gate_sampled(bits, m):
    n, k, g = 14336, 4096, 128
    rows = sample_rows(n, 32, seed=bits, split_of=(k, g, 1, bits))
    idx, lut, al, be = synth.random_any4(n, k, g, 0, layer=f"bgate{bits}")
    mask = np.uint8((1 << bits) - 1)
    idx = (idx & mask) | (idx & np.uint8(mask << 4))   # both nibbles below 2^bits
    w = synth.weights_bf16(len(rows), k, 23, layer=f"bgate{bits}/rows")
    s, ex = calib(k, 23, f"bgate{bits}")
    qr = oracle.quantize(w, ex, g, iters=6, bits=bits)
    r = np.asarray(rows)
    idx[r], lut[r], al[r], be[r] = qr.idx_nib, qr.lut, qr.alpha, qr.beta
    q = oracle.Any4Tensors(idx, lut, al, be, g)
    packed = pack_bits(bits, q)
    wd = a4.any4_dequant_bits(bits, packed, n, k, g)
    np.testing.assert_array_equal(bits_host(wd)[r], oracle.dequant_rows(q, rows))
    x = synth.activations_bf16(m, s, 24, layer=f"bgate{bits}")
    y = a4.any4_linear_bits(bits, bf16_dev(x), packed, n, k, g)
    check_linear(y, x, q, rows)


def test_bits4_is_the_any4_path():
    n, k, g = 512, 1024, 128
    q, s = quantized_bits(4, n, k, g, "b4same", iters=4)
    p4 = pack_bits(4, q)
    assert torch.equal(p4, pack_dev(q))
    x = bf16_dev(synth.activations_bf16(3, s, 25, layer="b4same"))
    y1 = a4.any4_linear_bits(4, x, p4, n, k, g)
    y2 = a4.any4_linear(x, p4, n, k, g)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_bits_rejects_bad_width():
    d = ctypes_ptr = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda:0")
    p = d.data_ptr()
    assert a4.any4_packed_bytes_bits(5, 64, 64, 64) == 0
    assert a4.lib.any4_pack_bits(1, p, p, p, p, 32, 64, 64, p, 1 << 16, None) == a4.ANY4_ESHAPE
    assert a4.lib.any4_linear_bits(0, p, p, 1, 32, 64, 64, p, p, 1 << 16, None) == a4.ANY4_ESHAPE
    del ctypes_ptr
