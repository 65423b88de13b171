"""The forward enqueues only stream-ordered device work (no host
synchronisation, allocation or blocking copy), so a caller can capture it
into a CUDA graph once and replay it with new inputs in the same buffers.
A replay must give bitwise the same output as a direct forward on those
inputs (the kernels are deterministic)."""
from __future__ import annotations

import numpy as np
import pytest

from weight_only_quantized_warp_b200 import inputs as gen

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("path,T", [(1, 12), (2, 96), (2, 700)], ids=["decode", "tc", "tc_wide"])
def test_forward_replays_from_a_cuda_graph(cuda_device, path, T):
    import torch
    from weight_only_quantized_warp_b200 import qmoe
    cfg = gen.MoEConfig(T=T, H=256, I=384, E=4, k=2, bits=4, block_size=64, fusion=1,
                        has_fc1_bias=True, has_fc2_bias=True, has_shared=True)
    first = gen.make_inputs(cfg, 61)
    m = qmoe.QMoE(cfg, "cuda:0", path=path)
    m.set_weights_from(first)
    x = qmoe.to_device(first.x, "cuda:0")
    lg = qmoe.to_device(first.logits, "cuda:0")
    sh = qmoe.to_device(first.shared, "cuda:0")
    y = torch.empty_like(x)
    m.workspace(T)  # allocate before capture

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        m.forward(x, lg, sh, out=y)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        m.forward(x, lg, sh, out=y)

    second_x, second_lg, second_sh = gen.make_token_batch(cfg, 62)
    x.copy_(qmoe.to_device(second_x, "cuda:0"))
    lg.copy_(qmoe.to_device(second_lg, "cuda:0"))
    sh.copy_(qmoe.to_device(second_sh, "cuda:0"))
    graph.replay()
    torch.cuda.synchronize()
    replayed = y.float().cpu().numpy()

    direct = m.forward(qmoe.to_device(second_x, "cuda:0"), qmoe.to_device(second_lg, "cuda:0"),
                       qmoe.to_device(second_sh, "cuda:0"))
    torch.cuda.synchronize()
    assert qmoe.qmoe_path_for(m.handle, T) == path
    np.testing.assert_array_equal(replayed, direct.float().cpu().numpy())
    del graph
