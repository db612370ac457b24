"""GPU parity of the prefill path (M > 16).

any4 up to 512 tokens decodes each 128-row weight tile straight into the
tensor-core GEMM's shared-memory stages (row tables in registers, no bf16
copy of W); any4 beyond 512 tokens and any3 / any2 dequantize into a
workspace scratch first, which must equal any4_dequant_bits bit for bit. y must meet the linear layer's acceptance bar
and the tight elementwise bar (both paths contract bf16 weights with fp32
accumulation). Shapes cover every token-tile width of the fused path (64,
128, 256 and several 256-token tiles), ragged token and row tails (a last
128-row tile with panels past N), K not a multiple of a tile's stage count,
every group size, split-K, and the Llama-3-8B MLP shapes at full size
(sampled rows, whole panels among them)."""
import numpy as np
import pytest
import torch

import learned_bit_lut_b200 as a4
import synth
from gpu_util import bf16_dev, bits_host, check_linear, mixed, pack_dev, quantized, require_gpu, sample_rows

pytestmark = pytest.mark.gpu

STATUS_OFFSET = 65536 * 4


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    torch.cuda.set_device(0)


@pytest.mark.parametrize("n,k,g,m", [(256, 512, 128, 17), (256, 512, 128, 64), (16, 64, 64, 17),
                                     (256, 512, 128, 65), (256, 512, 128, 128), (256, 512, 128, 129),
                                     (1024, 4096, 128, 256), (160, 2112, 64, 300),
                                     (4096, 1024, 256, 33), (48, 1024, 1024, 513), (272, 1536, 512, 257),
                                     (2080, 1024, 128, 96), (256, 1024, 128, 512)])
def test_prefill_shapes(n, k, g, m):
    q, s = quantized(n, k, g, layer=f"pre{n}x{k}", iters=4)
    x = synth.activations_bf16(m, s, 7, layer=f"pre{n}x{k}")
    ws = a4.workspace_for(m, n, k, g, torch.device("cuda:0"))
    y = a4.any4_linear(bf16_dev(x), pack_dev(q), n, k, g, workspace=ws)
    torch.cuda.synchronize()
    check_linear(y, x, q)
    assert int(ws[STATUS_OFFSET:STATUS_OFFSET + 4].view(torch.int32)[0]) == 0


@pytest.mark.parametrize("shape,m", [((14336, 4096), 512), ((4096, 14336), 384)])
def test_prefill_llama3_8b_mlp_sampled(shape, m):
    n, k = shape
    rows = sample_rows(n, 48, seed=n + 1)
    q, s = mixed(n, k, 128, rows, layer=f"pmlp{n}x{k}")
    x = synth.activations_bf16(m, s, 8, layer=f"pmlp{n}x{k}")
    y = a4.any4_linear(bf16_dev(x), pack_dev(q), n, k, 128)
    check_linear(y, x, q, rows)


def test_prefill_scratch_is_the_dequantized_weight_any3():
    from gpu_util import calib, to_dev
    import oracle
    n, k, g, m = 1024, 2048, 128, 40
    w = synth.weights_bf16(n, k, 0, layer="pscratch3")
    s, ex = calib(k, 0, "pscratch3")
    q = oracle.quantize(w, ex, g, iters=4, bits=3)
    x = synth.activations_bf16(m, s, 9, layer="pscratch3")
    packed = a4.any4_pack_bits(3, to_dev(q.idx_nib), to_dev(q.lut), to_dev(q.alpha), to_dev(q.beta), g)
    ws = a4.workspace_for(m, n, k, g, torch.device("cuda:0"), bits=3)
    assert a4.lib.any4_linear_workspace_bytes_bits(3, m, n, k, g) >= STATUS_OFFSET + 256 + n * k * 2
    y = a4.any4_linear_bits(3, bf16_dev(x), packed, n, k, g, workspace=ws)
    wd = a4.any4_dequant_bits(3, packed, n, k, g)
    torch.cuda.synchronize()
    off = STATUS_OFFSET + 256
    scratch = ws[off:off + n * k * 2].view(torch.int16).view(n, k)
    assert torch.equal(scratch, wd.view(torch.int16))
    check_linear(y, x, q)


def test_prefill_repeatable_and_guard_rows_untouched():
    n, k, g, m = 512, 1024, 128, 100
    q, s = quantized(n, k, g, layer="pguard", iters=4)
    x = bf16_dev(synth.activations_bf16(m, s, 10, layer="pguard"))
    packed = pack_dev(q)
    buf = torch.full((m + 2, n), 7, dtype=torch.int16, device="cuda:0")
    out = buf.view(torch.bfloat16)[1:m + 1]
    a4.any4_linear(x, packed, n, k, g, out=out)
    first = bits_host(out).copy()
    a4.any4_linear(x, packed, n, k, g, out=out)
    torch.cuda.synchronize()
    assert np.array_equal(first, bits_host(out))
    assert torch.all(buf[0] == 7) and torch.all(buf[m + 1] == 7)


def test_prefill_kernel_choice():
    # any4 up to 512 tokens decodes into the GEMM's shared memory; beyond that,
    # and for any3 / any2, the weight is dequantized into the workspace first
    assert a4.any4_linear_kernel(17, 4096, 4096, 128) == "prefill_fused"
    assert a4.any4_linear_kernel(512, 4096, 4096, 128) == "prefill_fused"
    assert a4.any4_linear_kernel(513, 4096, 4096, 128) == "prefill_gemm"
    assert a4.any4_linear_kernel(40, 4096, 4096, 128, bits=3) == "prefill_gemm"
    assert a4.any4_linear_kernel(16, 4096, 4096, 128) == "shared_tables"


def test_prefill_workspace_size():
    n, k, g = 4096, 4096, 128
    header = STATUS_OFFSET + 256
    need = a4.any4_linear_workspace_bytes(17, n, k, g)
    assert header <= need < header + n * k * 2          # any4: no dequantized copy of W
    assert a4.lib.any4_linear_workspace_bytes(17, n, k, g) == need
    x = torch.zeros((17, k), dtype=torch.bfloat16, device="cuda:0")
    y = torch.empty((17, n), dtype=torch.bfloat16, device="cuda:0")
    packed = torch.zeros(a4.any4_packed_bytes(n, k, g), dtype=torch.uint8, device="cuda:0")
    ws = torch.zeros(need - 256, dtype=torch.uint8, device="cuda:0")
    rc = a4.lib.any4_linear(x.data_ptr(), packed.data_ptr(), 17, n, k, g, y.data_ptr(), ws.data_ptr(),
                            ws.numel(), None)
    assert rc == a4.ANY4_EWORKSPACE


@pytest.mark.parametrize("n,k,g,m", [(1024, 4096, 128, 64), (4096, 4096, 128, 17), (256, 512, 128, 300),
                                     (1024, 1024, 64, 40)])
def test_prefill_split_k(n, k, g, m):
    # few output tiles: the K range of each tile is split between blocks and
    # the partials are added in split order; two calls must agree bit for bit
    q, s = quantized(n, k, g, layer=f"psplit{n}x{k}", iters=4)
    x = bf16_dev(synth.activations_bf16(m, s, 11, layer=f"psplit{n}x{k}"))
    packed = pack_dev(q)
    ws = a4.workspace_for(m, n, k, g, torch.device("cuda:0"))
    y1 = a4.any4_linear(x, packed, n, k, g, workspace=ws)
    y2 = a4.any4_linear(x, packed, n, k, g, workspace=ws)
    torch.cuda.synchronize()
    check_linear(y1, bits_host(x), q)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    assert int(ws[STATUS_OFFSET:STATUS_OFFSET + 4].view(torch.int32)[0]) == 0
    assert int(ws[:4 * 65536].view(torch.int32).abs().sum()) == 0   # tile counters back to zero
