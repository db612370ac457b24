"""GPU parity of the short-K-split decode kernels (any4, M <= 16).

Shapes whose 32-row panels fit the SMs two or four times over, with at most
16 chunks of 64 columns per thread block and at least one per warp, run on a
cluster of 2 or 4 blocks per panel that adds its K slices in rank order
through distributed shared memory: for M = 5..16 the register-table kernel
(every lane holds the 16-entry tables of its four rows as byte planes and
decodes with byte permutes), for M <= 4 the shared row-pair tables with each
warp loading its own operands (which also takes whole panels of at most 128
chunks at M <= 4 where the streaming kernel would run whole panels too).
Checks the plan (grid and cluster size on a 148-SM B200), the linear layer's
acceptance bar and the tight elementwise bar against the oracle for token
counts of both operand tiles (1-8 and 9-16 tokens), ragged last panels
(N = 16, 1008, 1040), K slices that split unevenly between warps, every group
size, bit-identical repeated calls, output rows outside y untouched, and the
status word."""
import numpy as np
import pytest
import torch

import learned_bit_lut_b200 as a4
import synth
from gpu_util import bf16_dev, bits_host, check_linear, pack_dev, quantized, require_gpu

pytestmark = pytest.mark.gpu

STATUS_OFFSET = 65536 * 4


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    torch.cuda.set_device(0)


def sm_count():
    return torch.cuda.get_device_properties(0).multi_processor_count


# (n, k, g, cluster for M <= 8 or None (shared-table kernel), cluster for M = 9..16)
SHAPES = [
    (1024, 4096, 128, 4, 4),    # Llama-3-8B k/v: 64 chunks, 16 per block
    (2048, 2048, 64, 2, 2),     # 64 panels x 2
    (768, 2048, 128, 2, 4),     # M = 16: 8 chunks per block, one per warp
    (1040, 2048, 256, 2, 4),    # 33 panels, ragged last panel
    (16, 4096, 1024, 4, 4),     # one half-filled panel
    (1008, 3136, 64, None, 4),  # M = 16: 49 chunks -> slices of 12 and 13, ragged warps
    (1024, 2560, 512, None, 4), # M = 16: slices of 10 chunks, 1-2 per warp
]


@pytest.mark.parametrize("n,k,g,c8,c16", SHAPES)
def test_regt_plan(n, k, g, c8, c16):
    if sm_count() != 148:
        pytest.skip("cluster sizes are stated for a 148-SM B200")
    panels = (n + 31) // 32
    for m, cl in ((1, c8), (4, c8), (5, c8), (8, c8), (9, c16), (16, c16)):
        blocks, cluster = a4.any4_linear_grid(m, n, k, g)
        kernel = a4.any4_linear_kernel(m, n, k, g)
        if cl is not None:
            assert (blocks, cluster) == (panels * cl, cl)
            assert kernel == ("shared_tables_direct" if m <= 4 else "register_tables")
        else:   # these shapes split panels over a cluster of the streaming kernel
            assert kernel == "shared_tables" and cluster > 1
    # the shared-table kernel keeps 3- and 2-bit weights
    assert a4.any4_linear_grid(1, 1024, 4096, 128, bits=3)[1] == 4
    assert a4.any4_linear_kernel(1, 1024, 4096, 128, bits=3) == "shared_tables"


@pytest.mark.parametrize("n,k,g,c8,c16", SHAPES)
def test_regt_matches_oracle(n, k, g, c8, c16):
    q, s = quantized(n, k, g, layer=f"rt{n}x{k}", iters=4)
    packed = pack_dev(q)
    for m in (1, 2, 5, 8, 9, 13, 16):
        x = synth.activations_bf16(m, s, 50 + m, layer=f"rt{n}x{k}")
        ws = a4.workspace_for(m, n, k, g, torch.device("cuda:0"))
        y = a4.any4_linear(bf16_dev(x), packed, n, k, g, workspace=ws)
        torch.cuda.synchronize()
        check_linear(y, x, q)
        assert int(ws[STATUS_OFFSET:STATUS_OFFSET + 4].view(torch.int32)[0]) == 0


@pytest.mark.parametrize("m", [1, 7, 16])
def test_regt_repeatable_and_guard_rows_untouched(m):
    n, k, g = 1024, 4096, 128
    q, s = quantized(n, k, g, layer="rtrep", iters=4)
    packed = pack_dev(q)
    x = bf16_dev(synth.activations_bf16(m, s, 60, layer="rtrep"))
    buf = torch.full((m + 2, n), 7, dtype=torch.int16, device="cuda:0")
    out = buf.view(torch.bfloat16)[1:m + 1]
    a4.any4_linear(x, packed, n, k, g, out=out)
    first = bits_host(out).copy()
    for _ in range(3):
        a4.any4_linear(x, packed, n, k, g, out=out)
        torch.cuda.synchronize()
        assert np.array_equal(first, bits_host(out))
    assert torch.all(buf[0] == 7) and torch.all(buf[m + 1] == 7)


def test_regt_zero_and_constant_weights():
    # degenerate tables: every entry the same value; alpha = 1, beta = 0 gives
    # y = LUT value x sum of x for every row
    n, k, g, m = 1024, 4096, 128, 3
    idx = np.random.default_rng(1).integers(0, 256, size=(n, k // 2), dtype=np.uint8)   # two nibbles a byte
    lut = np.full((n, 16), 0x3F80, dtype=np.uint16)            # 1.0
    alpha = np.full((n, k // g), 0x3F80, dtype=np.uint16)
    beta = np.zeros((n, k // g), dtype=np.uint16)
    from gpu_util import to_dev
    packed = a4.any4_pack(to_dev(idx), to_dev(lut), to_dev(alpha), to_dev(beta), g)
    xs = np.zeros((m, k), dtype=np.uint16)
    xs[0, :] = 0x3F80                                            # token 0: all ones
    xs[2, ::2] = 0xBF80                                          # token 2: -1 at even columns
    y = a4.any4_linear(bf16_dev(xs), packed, n, k, g).float().cpu().numpy()
    assert np.all(y[0] == float(k)) and np.all(y[1] == 0.0) and np.all(y[2] == -float(k // 2))


@pytest.mark.parametrize("m", [8, 16])
def test_regt_one_hot_columns_read_back_indices(m):
    # LUT_n[q] = q - 8, alpha = 1, beta = 0, token j one-hot at column c_j:
    # y[j, n] = idx[n, c_j] - 8 exactly, which pins where every index lands
    n, k, g = 1024, 4096, 128
    rng = np.random.default_rng(2)
    idx_nib = rng.integers(0, 256, size=(n, k // 2), dtype=np.uint8)
    vals = np.arange(16, dtype=np.float32) - 8.0
    lut1 = (vals.view(np.uint32) >> 16).astype(np.uint16)          # exact in bf16
    lut = np.tile(lut1, (n, 1))
    alpha = np.full((n, k // g), 0x3F80, dtype=np.uint16)
    beta = np.zeros((n, k // g), dtype=np.uint16)
    from gpu_util import to_dev
    packed = a4.any4_pack(to_dev(idx_nib), to_dev(lut), to_dev(alpha), to_dev(beta), g)
    cols = (np.arange(m) * 263 + 5) % k
    xs = np.zeros((m, k), dtype=np.uint16)
    xs[np.arange(m), cols] = 0x3F80
    y = a4.any4_linear(bf16_dev(xs), packed, n, k, g).float().cpu().numpy()
    idx = np.empty((n, k), dtype=np.int64)
    idx[:, 0::2] = idx_nib & 15
    idx[:, 1::2] = idx_nib >> 4
    expect = (idx[:, cols] - 8).T.astype(np.float32)
    assert np.array_equal(y, expect)


@pytest.mark.parametrize("m", [1, 4])
def test_direct_kernel_whole_panels_up_to_128_chunks(m):
    # 128 panels of 128 chunks: at M <= 4 one block per panel of the shared
    # tables with per-warp loads (each warp takes 8 chunks in turn)
    from gpu_util import mixed, sample_rows
    n, k, g = 4096, 8192, 128
    if sm_count() >= 128:
        assert a4.any4_linear_kernel(m, n, k, g) == "shared_tables_direct"
        assert a4.any4_linear_grid(m, n, k, g) == (128, 1)
    rows = sample_rows(n, 32, seed=m, whole_panels=4)
    q, s = mixed(n, k, g, rows, layer="direct_long")
    x = synth.activations_bf16(m, s, 80 + m, layer="direct_long")
    y = a4.any4_linear(bf16_dev(x), pack_dev(q), n, k, g)
    check_linear(y, x, q, rows)
