"""GPU parity of the fixed-table formats (int4, NF4, FP4) and of the b-bit
any3 / any2 variants through the any4 kernels, against the fp64 oracle.

A fixed-format weight is packed with any4_pack_format (the format's table in
every row); an any3 / any2 weight is packed with any4_pack (its 8- or
4-entry table padded to 16). Both then use the same dequant (bit-exact) and
linear (2e-2 of max |y| per token row, plus the tight elementwise bar) as any4.
"""
import numpy as np
import pytest
import torch

import learned_bit_lut_b200 as a4
import oracle
import synth
from gpu_util import bf16_dev, bits_host, calib, check_linear, pack_dev, require_gpu, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    torch.cuda.set_device(0)


def _pack_format(q: oracle.Any4Tensors, fmt: str):
    return a4.any4_pack_format(fmt, to_dev(q.idx_nib), to_dev(q.alpha), to_dev(q.beta), q.group)


@pytest.mark.parametrize("fmt", ["int4", "nf4", "fp4"])
@pytest.mark.parametrize("n,k,g", [(256, 512, 128), (1024, 4096, 64), (160, 2112, 64)])
def test_format_dequant_bitexact_and_linear(fmt, n, k, g):
    w = synth.weights_bf16(n, k, 11, layer=f"fmt{n}x{k}")
    q = oracle.quantize_format(w, fmt, g)
    packed = _pack_format(q, fmt)
    # the fixed-table pack equals an any4 pack of the same table in every row
    assert torch.equal(packed, pack_dev(q))
    wd = a4.any4_dequant(packed, n, k, g)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bits_host(wd), oracle.dequant(q))
    s = synth.channel_scale(k, 11, layer=f"fmt{n}x{k}")
    for m in (1, 5, 16):
        x = synth.activations_bf16(m, s, 12 + m, layer=f"fmt{n}x{k}")
        check_linear(a4.any4_linear(bf16_dev(x), packed, n, k, g), x, q)


@pytest.mark.parametrize("fmt", ["nf4"])
def test_format_full_size_sampled(fmt):
    n, k, g = 14336, 4096, 128
    w = synth.weights_bf16(n, k, 13, layer="fmt_gate")
    q = oracle.quantize_format(w, fmt, g)
    packed = _pack_format(q, fmt)
    rows = np.array(sorted(set(range(32)) | set(range(n - 32, n)) |
                           set(np.random.default_rng(3).choice(n, 64, replace=False).tolist())))
    wd = a4.any4_dequant(packed, n, k, g)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bits_host(wd)[rows], oracle.dequant_rows(q, rows))
    s = synth.channel_scale(k, 13, layer="fmt_gate")
    x = synth.activations_bf16(4, s, 14, layer="fmt_gate")
    check_linear(a4.any4_linear(bf16_dev(x), packed, n, k, g), x, q, rows)


@pytest.mark.parametrize("bits", [3, 2])
@pytest.mark.parametrize("n,k,g", [(256, 512, 128), (512, 4096, 128)])
def test_any3_any2_through_the_any4_kernels(bits, n, k, g):
    w = synth.weights_bf16(n, k, 17, layer=f"any{bits}_{n}")
    s, ex = calib(k, 17, f"any{bits}_{n}")
    q = oracle.quantize(w, ex, g, iters=10, bits=bits)
    packed = pack_dev(q)
    wd = a4.any4_dequant(packed, n, k, g)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bits_host(wd), oracle.dequant(q))
    for m in (1, 8, 16):
        x = synth.activations_bf16(m, s, 18 + m, layer=f"any{bits}_{n}")
        check_linear(a4.any4_linear(bf16_dev(x), packed, n, k, g), x, q)
