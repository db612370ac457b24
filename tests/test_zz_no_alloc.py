"""any4_linear_noalloc: the linear layer for callers that cannot allocate
device memory (for example an operator inside a serving runtime that owns all
device memory and only hands it inputs and outputs). It uses the library's own
fixed scratch array instead of a caller workspace.

Checked through the C ABI against any4_linear (caller workspace) on two calls
in a row, with the acceptance bar the other tests use. This file is collected
last, so a run that stops at the first failure has run everything else first.
"""
import numpy as np
import pytest
import torch

import learned_bit_lut_b200 as a4
import synth
from gpu_util import REL_TOL, bf16_dev, pack_dev, quantized, require_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n,k,g,m", [(1024, 4096, 128, 1), (1024, 4096, 128, 16),
                                     (4096, 14336, 128, 5)])
def test_noalloc_matches_workspace_call_twice(n, k, g, m):
    require_gpu()
    q, s = quantized(n, k, g, layer=f"noalloc{n}x{k}", iters=4)
    x = bf16_dev(synth.activations_bf16(m, s, 11, layer=f"noalloc{n}x{k}"))
    packed = pack_dev(q)
    ref = a4.any4_linear(x, packed, n, k, g).float()
    for _ in range(2):
        out = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device="cuda")
        a4.any4_linear_noalloc(x, packed, n, k, g, out=out)
        torch.cuda.synchronize()
        got = out.float()
        scale = ref.abs().amax(dim=1, keepdim=True).clamp_min(1e-30)
        worst = ((got - ref).abs() / scale).amax(dim=1)
        assert torch.isfinite(got).all()
        assert torch.all(worst <= REL_TOL), worst
