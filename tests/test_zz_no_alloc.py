"""qmoe_forward_noalloc: the forward whose scratch is the library's fixed
device array, for callers that cannot allocate device memory where they run
the operator (a plugin whose host framework owns all device memory, a serving
loop that must not allocate mid-request).

Its output must match qmoe_forward's (same kernels, caller workspace) within
the parity tolerance, on two calls in a row; the array keeps the previous
call's contents, so the second call checks that nothing stale leaks into it.
This file sorts last so a stop-at-first-failure run has run everything else.
"""
from __future__ import annotations

import numpy as np
import pytest

from weight_only_quantized_warp_b200 import inputs as gen

from gpu_helpers import TOL_BF16, max_rel, to_numpy

pytestmark = pytest.mark.gpu


def _forward_both(cfg, seed, path=None):
    import torch
    from weight_only_quantized_warp_b200 import qmoe
    inp = gen.make_inputs(cfg, seed, bias_std=0.1)
    m = qmoe.QMoE(cfg, "cuda:0", path=path)
    m.set_weights_from(inp)
    x = qmoe.to_device(inp.x, "cuda:0")
    lg = qmoe.to_device(inp.logits, "cuda:0")
    sh = qmoe.to_device(inp.shared, "cuda:0")
    ref = to_numpy(m.forward(x, lg, sh))
    outs = []
    for _ in range(2):
        y = torch.full_like(x, float("nan"))
        qmoe.qmoe_forward_noalloc(m.handle, cfg.T, x, lg, sh, y)
        torch.cuda.synchronize()
        outs.append(to_numpy(y))
    return ref, outs, m


@pytest.mark.parametrize("path", [1, 2], ids=["decode", "tc"])
def test_noalloc_matches_workspace_forward_twice(cuda_device, path):
    cfg = gen.MoEConfig(T=12, H=256, I=192, E=8, k=2, bits=4, block_size=64, fusion=2,
                        has_fc1_bias=True, has_fc2_bias=True, has_shared=True)
    ref, outs, m = _forward_both(cfg, 41, path)
    for y in outs:
        assert np.isfinite(y).all()
        assert max_rel(y, ref) <= TOL_BF16
    # the device status word of the no-alloc forward lives in the fixed array
    from weight_only_quantized_warp_b200 import qmoe
    assert qmoe.qmoe_noalloc_read_device_status(m.handle) == qmoe.QMOE_OK


def test_noalloc_rejects_calls_above_the_fixed_scratch(cuda_device):
    from weight_only_quantized_warp_b200 import qmoe
    cfg = gen.MoEConfig(T=4, H=256, I=192, E=8, k=2, bits=4, block_size=64, fusion=2)
    m = qmoe.QMoE(cfg, "cuda:0")
    limit = qmoe.qmoe_noalloc_scratch_bytes()
    T = 4
    while qmoe.qmoe_workspace_size(m.handle, T) <= limit:
        T *= 2
    st = qmoe.lib.qmoe_forward_noalloc(m.handle, T, 16, 16, None, 16, None)
    assert st == qmoe.QMOE_INVALID_ARGUMENT
    assert b"scratch" in qmoe.lib.qmoe_last_error(m.handle)
