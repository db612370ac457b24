"""any4_linear_noalloc: the linear layer for callers that cannot allocate
device memory (for example an operator inside a serving runtime that owns all
device memory and only hands it inputs and outputs). It uses the library's own
fixed scratch array instead of a caller workspace.

Checked through the C ABI on two calls in a row: bit-identical to any4_linear
with a caller workspace (the same kernel and plan, so the same fixed summation
order), within the acceptance bar of the oracle, and with the scratch's status
word zero afterwards. M > 16 (the prefill path) is rejected. This file is
collected last, so a run that stops at the first failure has run everything
else first.
"""
import pytest
import torch

import learned_bit_lut_b200 as a4
import synth
from gpu_util import bf16_dev, check_linear, pack_dev, quantized, require_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n,k,g,m", [(1024, 4096, 128, 1), (1024, 4096, 128, 16),
                                     (4096, 14336, 128, 5), (256, 512, 64, 12)])
def test_noalloc_matches_workspace_call_twice(n, k, g, m):
    require_gpu()
    q, s = quantized(n, k, g, layer=f"noalloc{n}x{k}", iters=4)
    xb = synth.activations_bf16(m, s, 11, layer=f"noalloc{n}x{k}")
    x = bf16_dev(xb)
    packed = pack_dev(q)
    ref = a4.any4_linear(x, packed, n, k, g)
    for _ in range(2):
        out = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device="cuda")
        a4.any4_linear_noalloc(x, packed, n, k, g, out=out)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
        assert a4.noalloc_status() == 0
    check_linear(out, xb, q)


def test_noalloc_rejects_prefill_token_counts():
    require_gpu()
    n, k, g = 256, 512, 128
    q, s = quantized(n, k, g, layer="noalloc_m17", iters=4)
    x = bf16_dev(synth.activations_bf16(17, s, 12, layer="noalloc_m17"))
    with pytest.raises(a4.Any4Error) as e:
        a4.any4_linear_noalloc(x, pack_dev(q), n, k, g)
    assert e.value.status == a4.ANY4_ESHAPE
