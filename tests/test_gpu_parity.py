"""GPU parity: the CUDA library (through the C ABI) against the fp64 oracle.

Dequantization must be bit-exact; the linear layer must meet the acceptance
bar (2e-2 of max |y| per token row) and, because it contracts the same bf16
weights, a tight elementwise bar as well. Shapes cover the benchmark
workloads (full sizes use sampled rows), several tiles with split tiles, and
the degenerate cases (one atom, one tile, every M from 1 to 16).
"""
import numpy as np
import pytest
import torch

import learned_bit_lut_b200 as a4
import oracle
import synth
from gpu_util import (bf16_dev, bits_host, check_linear, mixed, pack_dev, quantized,
                      require_gpu, sample_rows, split_panels, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    torch.cuda.set_device(0)


# ------------------------------------------------------------------ dequant

def test_dequant_bitexact_single_layer():
    q, _ = quantized(256, 512, 128, layer="single")
    packed = pack_dev(q)
    w = a4.any4_dequant(packed, 256, 512, 128)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bits_host(w), oracle.dequant(q))


def test_dequant_bitexact_4096():
    q, _ = quantized(4096, 4096, 128, layer="proj")
    w = a4.any4_dequant(pack_dev(q), 4096, 4096, 128)
    np.testing.assert_array_equal(bits_host(w), oracle.dequant(q))


@pytest.mark.parametrize("n,k,g,kind", [(14336, 4096, 128, "normal"), (4096, 14336, 128, "normal"),
                                        (28672, 8192, 64, "student_t"),
                                        (28672, 8192, 1024, "student_t")])
def test_dequant_bitexact_full_size_sampled(n, k, g, kind):
    rows = sample_rows(n, 32, seed=n + g)
    q, _ = mixed(n, k, g, rows, layer=f"dq{n}x{k}", kind=kind)
    w = a4.any4_dequant(pack_dev(q), n, k, g)
    got = bits_host(w[torch.as_tensor(rows, device=w.device)])
    np.testing.assert_array_equal(got, oracle.dequant_rows(q, rows))


def test_dequant_int4_and_nf4_tables():
    g = np.random.default_rng(20)
    n, k, gs = 64, 256, 64
    grid = np.tile(oracle.f64_to_bf16_bits(oracle.int4_grid()), (n, 1))
    nf4 = np.tile(oracle.nf4_bf16_bits(), (n, 1))
    idx = g.integers(0, 16, (n, k))
    scale = oracle.f64_to_bf16_bits(g.uniform(0.001, 0.2, (n, k // gs)))
    beta = oracle.f64_to_bf16_bits(g.normal(0, 0.01, (n, k // gs)))
    for lut, b in ((grid, beta), (nf4, np.zeros_like(beta))):
        q = oracle.Any4Tensors(oracle.pack_nibbles(idx), lut, scale, b, gs)
        w = a4.any4_dequant(pack_dev(q), n, k, gs)
        np.testing.assert_array_equal(bits_host(w), oracle.dequant(q))


def test_dequant_special_values():
    # subnormal products, signed zeros, exact cancellations, large exponents
    n, k, gs = 16, 64, 64
    lut_vals = np.array([0.0, -0.0, 1.0, -1.0, 2.0 ** -126, -(2.0 ** -130), 3.0, -2.5, 0.5, 7.0,
                         -8.0, 1.0078125, 2.0 ** 100, -(2.0 ** -100), 0.25, 6.0])
    lut = np.tile(oracle.f64_to_bf16_bits(lut_vals), (n, 1))
    idx = np.tile(np.arange(16), (n, k // 16))
    avals = np.array([0.0, 1.0, 0.5, 2.0 ** -20, 2.0 ** 20, -1.0, 1.0078125, 3.0,
                      0.0, 1.0, 0.5, 2.0 ** -20, 2.0 ** 20, -1.0, 1.0078125, 3.0])[:, None]
    bvals = np.array([-0.0, 0.0, -1.0, 2.0 ** -126, -3.0, 1.0, -1.0078125, 0.25,
                      0.0, -0.0, 1.0, -(2.0 ** -126), 3.0, -1.0, 1.0078125, -0.25])[:, None]
    q = oracle.Any4Tensors(oracle.pack_nibbles(idx), lut, oracle.f64_to_bf16_bits(avals),
                           oracle.f64_to_bf16_bits(bvals), gs)
    w = a4.any4_dequant(pack_dev(q), n, k, gs)
    np.testing.assert_array_equal(bits_host(w), oracle.dequant(q))


# ------------------------------------------------------------------- linear

@pytest.mark.parametrize("m", list(range(1, 17)))
def test_linear_single_layer_every_m(m):
    q, s = quantized(256, 512, 128, layer="single")
    x = synth.activations_bf16(m, s, 1, layer="single")
    y = a4.any4_linear(bf16_dev(x), pack_dev(q), 256, 512, 128)
    check_linear(y, x, q)


@pytest.mark.parametrize("m", [1, 4, 16])
def test_linear_4096(m):
    q, s = quantized(4096, 4096, 128, layer="proj")
    x = synth.activations_bf16(m, s, 2, layer="proj")
    y = a4.any4_linear(bf16_dev(x), pack_dev(q), 4096, 4096, 128)
    check_linear(y, x, q)


@pytest.mark.parametrize("shape", [(14336, 4096), (4096, 14336)])
@pytest.mark.parametrize("m", [1, 2, 4, 8, 16])
def test_linear_llama3_8b_mlp(shape, m):
    n, k = shape
    rows = sample_rows(n, 48, seed=n, split_of=(k, 128))
    if n == 14336:   # 448 panels over the SMs: stream-K splits panels between blocks
        assert set(split_panels(n, k, 128)) & {r // 32 for r in rows}
    q, s = mixed(n, k, 128, rows, layer=f"mlp{n}x{k}")
    x = synth.activations_bf16(m, s, 3, layer=f"mlp{n}x{k}")
    y = a4.any4_linear(bf16_dev(x), pack_dev(q), n, k, 128)
    check_linear(y, x, q, rows)


@pytest.mark.parametrize("g", [64, 128, 256, 1024])
@pytest.mark.parametrize("m", [1, 16])
def test_linear_llama3_70b_group_sweep(g, m):
    n, k = 28672, 8192
    rows = sample_rows(n, 32, seed=g, split_of=(k, g))
    q, s = mixed(n, k, g, rows, layer=f"g{g}", kind="student_t", sigma=0.7)
    x = synth.activations_bf16(m, s, 4, layer=f"g{g}")
    y = a4.any4_linear(bf16_dev(x), pack_dev(q), n, k, g)
    check_linear(y, x, q, rows)


@pytest.mark.parametrize("n,k,g,m", [(16, 64, 64, 1), (16, 64, 64, 16), (16, 4096, 128, 5),
                                     (4096, 64, 64, 3), (48, 1024, 1024, 9), (32, 192, 64, 13),
                                     (1024, 4096, 128, 16), (160, 2112, 64, 7)])
def test_linear_edge_shapes(n, k, g, m):
    q, s = quantized(n, k, g, layer=f"edge{n}x{k}", iters=4)
    x = synth.activations_bf16(m, s, 5, layer=f"edge{n}x{k}")
    y = a4.any4_linear(bf16_dev(x), pack_dev(q), n, k, g)
    check_linear(y, x, q)


@pytest.mark.parametrize("n,k,m", [(4096, 4096, 16), (4096, 4096, 7), (4096, 4096, 2), (1024, 4096, 12), (1024, 4096, 3)])
def test_linear_x_on_16_byte_boundary(n, k, m):
    # x that starts 16 bytes past a 32-byte boundary takes the 128-bit
    # activation loads instead of the 256-bit ones: same result bit for bit
    q, s = quantized(n, k, 128, layer=f"xal{n}x{k}", iters=4)
    xb = synth.activations_bf16(m, s, 70 + m, layer=f"xal{n}x{k}")
    packed = pack_dev(q)
    buf = torch.zeros(m * k + 16, dtype=torch.int16, device="cuda:0")
    assert buf.data_ptr() % 32 == 0
    x_off = buf[8:8 + m * k].view(m, k)
    x_off.copy_(to_dev(xb).view(m, k))
    assert x_off.data_ptr() % 32 == 16
    y_off = a4.any4_linear(x_off.view(torch.bfloat16), packed, n, k, 128)
    y_al = a4.any4_linear(bf16_dev(xb), packed, n, k, 128)
    torch.cuda.synchronize()
    assert torch.equal(y_off.view(torch.int16), y_al.view(torch.int16))
    check_linear(y_off, xb, q)


def test_linear_repeatable_and_workspace_restored():
    q, s = quantized(1024, 4096, 128, layer="rep", iters=4)
    x = bf16_dev(synth.activations_bf16(16, s, 6, layer="rep"))
    packed = pack_dev(q)
    need = a4.any4_linear_workspace_bytes(16, 1024, 4096, 128)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    y1 = a4.any4_linear(x, packed, 1024, 4096, 128, workspace=ws)
    y2 = a4.any4_linear(x, packed, 1024, 4096, 128, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    header = 65536 * 4 + 256         # arrival counters, then a reserved area
    assert int(ws[:header].view(torch.int32).abs().sum()) == 0   # counters back to zero


def test_linear_guard_bands_untouched():
    q, s = quantized(64, 1024, 128, layer="guard", iters=4)
    x = bf16_dev(synth.activations_bf16(3, s, 7, layer="guard"))
    pad = 128
    buf = torch.full((3 * 64 + 2 * pad,), -23131, dtype=torch.int16, device="cuda")   # 0xA5A5
    out = buf[pad:pad + 3 * 64].view(torch.bfloat16).view(3, 64)
    a4.any4_linear(x, pack_dev(q), 64, 1024, 128, out=out)
    torch.cuda.synchronize()
    assert torch.all(buf[:pad] == -23131) and torch.all(buf[pad + 3 * 64:] == -23131)


def test_linear_on_side_stream():
    q, s = quantized(256, 512, 128, layer="single")
    xb = synth.activations_bf16(2, s, 8, layer="single")
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        y = a4.any4_linear(bf16_dev(xb), pack_dev(q), 256, 512, 128)
    st.synchronize()
    check_linear(y, xb, q)


def test_linear_workspace_too_small_is_rejected():
    q, s = quantized(256, 512, 128, layer="single")
    x = bf16_dev(synth.activations_bf16(1, s, 9, layer="single"))
    with pytest.raises(a4.Any4Error) as e:
        a4.any4_linear(x, pack_dev(q), 256, 512, 128,
                       workspace=torch.zeros(16, dtype=torch.uint8, device="cuda"))
    assert e.value.status == a4.ANY4_EWORKSPACE
