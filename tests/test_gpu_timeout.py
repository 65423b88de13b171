"""Failure detection on the GPU without a fault: a bounded device wait is made
to run out and the library reports it.

With QMOE_OPT_TEST_WITHHOLD the tcgen05 kernels' MMA warp never announces its
first work item's accumulator, so the epilogue's wait on that signal (limited
here to 1 ms by QMOE_OPT_WAIT_LIMIT_NS) expires: the kernel writes
QMOE_TIMEOUT to the workspace status word, every role leaves its loop and the
CTA frees its tensor memory. The same handle then runs a normal forward that
matches the oracle, so the context stays usable.
"""
from __future__ import annotations

import pytest

from weight_only_quantized_warp_b200 import inputs as gen

from gpu_helpers import TOL_BF16, max_rel, to_numpy

pytestmark = pytest.mark.gpu

CASES = {
    # token tile 64 (decoded weights in tensor memory)
    "tile64": dict(T=96, E=4, k=2, H=256, I=384, bits=4, block_size=64, fusion=2),
    # token tile 256 (decoded weights in shared memory)
    "tile256": dict(T=300, E=2, k=1, H=256, I=384, bits=8, block_size=128, fusion=1),
}


@pytest.mark.parametrize("name", list(CASES))
def test_expired_wait_reports_timeout_then_recovers(cuda_device, name):
    import torch
    from weight_only_quantized_warp_b200 import qmoe
    cfg = gen.MoEConfig(act_dtype=gen.DT_BF16, scale_dtype=gen.DT_BF16, **CASES[name])
    inp = gen.make_inputs(cfg, seed=61)
    m = qmoe.QMoE(cfg, "cuda:0", path=qmoe.PATH_TC)
    m.set_weights_from(inp)
    x = qmoe.to_device(inp.x, "cuda:0")
    lg = qmoe.to_device(inp.logits, "cuda:0")
    assert qmoe.qmoe_path_for(m.handle, cfg.T) == qmoe.PATH_TC

    qmoe.qmoe_set_option(m.handle, qmoe.QMOE_OPT_WAIT_LIMIT_NS, 10**6)
    qmoe.qmoe_set_option(m.handle, qmoe.QMOE_OPT_TEST_WITHHOLD, 1)
    m.forward(x, lg)                                   # the call itself returns
    torch.cuda.synchronize()
    ws = m.workspace(cfg.T)
    assert qmoe.qmoe_read_device_status(m.handle, ws) == qmoe.QMOE_TIMEOUT

    qmoe.qmoe_set_option(m.handle, qmoe.QMOE_OPT_TEST_WITHHOLD, 0)
    qmoe.qmoe_set_option(m.handle, qmoe.QMOE_OPT_WAIT_LIMIT_NS, 2 * 10**9)
    y = m.forward(x, lg)
    torch.cuda.synchronize()
    assert qmoe.qmoe_read_device_status(m.handle, ws) == qmoe.QMOE_OK
    # the same handle's normal forward against the oracle
    import oracle
    err = max_rel(to_numpy(y), oracle.forward(inp)["y"])
    assert err <= TOL_BF16, f"y max rel err {err:.3e} after the timed-out call"
