"""GPU parity of the cluster-split decode path: shapes with fewer 32-row
panels than SMs run every panel on a cluster of 2, 4 or 8 thread blocks, each
on a K slice, and the cluster's first block adds the others' fp32 partials
(received through distributed shared memory) in rank order. Checks that the
launch really is clustered, the linear layer's acceptance bar against the
oracle for every decode mode (M = 1, 3, 8, 16), ragged K slices and a ragged
last panel, any3 / any2, and that repeated calls are bit-identical. For any4
the shapes with at most 16 chunks per block (1024 x 4096, 1008 x 4096 and
2048 x 2048) take the short-split kernels, which split the same way
(tests/test_gpu_regt.py); the others and any3 / any2 run the streaming
shared-table kernel."""
import numpy as np
import pytest
import torch

import learned_bit_lut_b200 as a4
import oracle
import synth
from gpu_util import bf16_dev, bits_host, calib, check_linear, pack_dev, quantized, require_gpu, to_dev

pytestmark = pytest.mark.gpu

STATUS_OFFSET = 65536 * 4


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    torch.cuda.set_device(0)


# (n, k, g, blocks per cluster on a 148-SM B200)
SHAPES = [
    (1024, 4096, 128, 4),    # Llama-3-8B k/v: 32 panels x 4
    (256, 8192, 128, 8),     # 8 panels x 8
    (2048, 2048, 128, 2),    # 64 panels x 2
    (512, 4160, 64, 4),      # 65 chunks per panel: K slices of 16 and 17 chunks
    (1008, 4096, 128, 4),    # ragged last panel (N = 1008)
]


@pytest.mark.parametrize("n,k,g,cl", SHAPES)
def test_cluster_grid(n, k, g, cl):
    panels = (n + 31) // 32
    for m in (1, 8, 16):
        blocks, cluster = a4.any4_linear_grid(m, n, k, g)
        assert cluster == cl and blocks == panels * cl
    blocks, cluster = a4.any4_linear_grid(17, n, k, g)   # prefill: no clusters
    assert cluster == 1
    # which decode kernel splits the panels (any4 with at most 16 chunks per
    # block: the short-split kernels)
    short = cl <= 4 and k // 64 <= 16 * cl
    assert a4.any4_linear_kernel(1, n, k, g) == ("shared_tables_direct" if short else "shared_tables")
    assert a4.any4_linear_kernel(16, n, k, g) == ("register_tables" if short else "shared_tables")


@pytest.mark.parametrize("n,k,g,cl", SHAPES)
def test_cluster_linear_matches_oracle(n, k, g, cl):
    q, s = quantized(n, k, g, layer=f"cl{n}x{k}", iters=4)
    packed = pack_dev(q)
    for m in (1, 3, 8, 16):
        x = synth.activations_bf16(m, s, 30 + m, layer=f"cl{n}x{k}")
        ws = a4.workspace_for(m, n, k, g, torch.device("cuda:0"))
        y = a4.any4_linear(bf16_dev(x), packed, n, k, g, workspace=ws)
        torch.cuda.synchronize()
        check_linear(y, x, q)
        assert int(ws[STATUS_OFFSET:STATUS_OFFSET + 4].view(torch.int32)[0]) == 0


@pytest.mark.parametrize("m", [1, 16])
def test_cluster_repeatable(m):
    n, k, g = 1024, 4096, 128
    q, s = quantized(n, k, g, layer="clrep", iters=4)
    packed = pack_dev(q)
    x = bf16_dev(synth.activations_bf16(m, s, 40, layer="clrep"))
    first = bits_host(a4.any4_linear(x, packed, n, k, g))
    for _ in range(3):
        again = bits_host(a4.any4_linear(x, packed, n, k, g))
        assert np.array_equal(first, again)


@pytest.mark.parametrize("bits", [3, 2])
def test_cluster_bits(bits):
    n, k, g = 1024, 4096, 128
    assert a4.any4_linear_grid(1, n, k, g, bits=bits)[1] == 4
    w = synth.weights_bf16(n, k, 41, layer=f"clb{bits}")
    s, ex = calib(k, 41, f"clb{bits}")
    q = oracle.quantize(w, ex, g, iters=4, bits=bits)
    packed = a4.any4_pack_bits(bits, to_dev(q.idx_nib), to_dev(q.lut), to_dev(q.alpha), to_dev(q.beta), g)
    for m in (1, 16):
        x = synth.activations_bf16(m, s, 42 + m, layer=f"clb{bits}")
        y = a4.any4_linear_bits(bits, bf16_dev(x), packed, n, k, g)
        check_linear(y, x, q)


def test_cluster_noalloc_entry_point():
    n, k, g, m = 1024, 4096, 128, 4
    q, s = quantized(n, k, g, layer="clna", iters=4)
    packed = pack_dev(q)
    x = synth.activations_bf16(m, s, 44, layer="clna")
    y = a4.any4_linear_noalloc(bf16_dev(x), packed, n, k, g)
    check_linear(y, x, q)
