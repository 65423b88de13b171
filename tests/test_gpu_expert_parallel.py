"""Expert parallel through the library's kernels on one GPU.

The three device steps of ``expert_parallel`` (``qmoe_ep_dispatch``,
``qmoe_ep_expert_rows``, ``qmoe_ep_combine``) run for G simulated ranks in
one process: each rank's handles hold its own experts, and the all-to-alls
between the steps are done by slicing and concatenating the device tensors
exactly as ``all_to_all_single`` would order them. No kernel waits on
another rank, so this needs one GPU only. Every rank's output is compared
with the oracle's single-device forward of its tokens, and the dispatch
outputs with the oracle's routing and permutation bit for bit.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import pytest

import oracle
from weight_only_quantized_warp_b200 import inputs as gen

from gpu_helpers import TOL_BF16, TOL_F32, max_rel, to_numpy

pytestmark = pytest.mark.gpu


def _cfg(**kw):
    base = dict(T=40, H=256, I=384, E=8, k=2, bits=4, block_size=64, act=gen.ACT_SWIGLU, fusion=2)
    base.update(kw)
    return gen.MoEConfig(**base)


CASES = {
    "int4_bs64": dict(),
    "int8_percol_bias": dict(bits=8, block_size=0, has_fc1_bias=True, has_fc2_bias=True),
    "tensor_core_rows": dict(T=300, E=4, k=2),          # 150+ rows per expert: the tcgen05 GEMM
    "weights_on_input_shared_scaled": dict(k=1, apply_router_weight_on_input=True, has_shared=True,
                                           routed_scaling_factor=1.5, expert_output_scale=0.75),
    "grouped_topk": dict(E=8, k=2, n_group=4, topk_group=2, normalize=False),
    "int8_tier": dict(compute_mode=gen.COMPUTE_INT8_BLOCK, block_size=128, T=48),
    "f32_acts": dict(act_dtype=gen.DT_F32, scale_dtype=gen.DT_F32, block_size=32),
    "score_bias_fc3_bias": dict(has_score_bias=True, fusion=0, has_fc3=True, has_fc1_bias=True,
                                has_fc3_bias=True),
}


def _rank_inputs(cfg, seed, world):
    """Shared weights (one draw) and each rank's own tokens."""
    w = gen.make_inputs(cfg, seed, bias_std=0.1)
    out = []
    for r in range(world):
        t = gen.make_inputs(dataclasses.replace(cfg, T=cfg.T + 5 * r), seed + 1000 + r, bias_std=0.1)
        out.append(dataclasses.replace(w, cfg=t.cfg, x=t.x, logits=t.logits, shared=t.shared))
    return out


def _simulate(inps, world, dev):
    """One expert-parallel forward of `world` ranks, exchanges done in process."""
    import torch
    from weight_only_quantized_warp_b200 import expert_parallel as ep
    from weight_only_quantized_warp_b200 import qmoe
    ops = [ep.LibraryOps(inps[r].cfg, inps[r], world, r, dev) for r in range(world)]
    xs = [qmoe.to_device(i.x, dev) for i in inps]
    lgs = [qmoe.to_device(i.logits, dev) for i in inps]
    shs = [qmoe.to_device(i.shared, dev) for i in inps]
    ds = [ops[r].dispatch(xs[r], lgs[r]) for r in range(world)]
    starts = [np.concatenate([[0], np.cumsum(d.send_counts)]).astype(int) for d in ds]
    recv_rows, recv_ids = [], []
    for q in range(world):
        recv_rows.append(torch.cat([ds[r].rows[starts[r][q]:starts[r][q + 1]] for r in range(world)]))
        recv_ids.append(torch.cat([ds[r].row_expert[starts[r][q]:starts[r][q + 1]] for r in range(world)]))
    outs = [ops[q].expert_rows(recv_rows[q], recv_ids[q]) for q in range(world)]
    ys = []
    for r in range(world):
        parts = []
        for q in range(world):
            o = sum(ds[s].send_counts[q] for s in range(r))
            parts.append(outs[q][o:o + ds[r].send_counts[q]])
        ys.append(ops[r].combine(ds[r], torch.cat(parts), shs[r], like=xs[r]))
    torch.cuda.synchronize()
    return ys, ds, ops


@pytest.mark.parametrize("world", [1, 2, 4])
@pytest.mark.parametrize("name", list(CASES))
def test_expert_parallel_ranks_match_the_oracle(cuda_device, name, world):
    cfg = _cfg(**CASES[name])
    if cfg.E % world:
        pytest.skip("experts do not divide over the ranks")
    inps = _rank_inputs(cfg, 500 + list(CASES).index(name), world)
    ys, _, _ = _simulate(inps, world, cuda_device)
    tol = TOL_BF16 if cfg.act_dtype == gen.DT_BF16 else TOL_F32
    for r in range(world):
        ref = oracle.forward(inps[r])["y"]
        err = max_rel(to_numpy(ys[r]), ref)
        assert err <= tol, f"rank {r}: y max rel err {err:.3e} > {tol}"


def test_dispatch_is_the_oracle_routing_in_expert_order(cuda_device):
    cfg = _cfg(T=70, E=8, k=3)
    inp = _rank_inputs(cfg, 77, 1)[0]
    ys, ds, ops = _simulate([inp], 1, cuda_device)
    d = ds[0]
    idx, _ = oracle.route(inp.logits, cfg.k, cfg.normalize)
    offsets, perm, inv = oracle.permute(idx, cfg.E)
    assert np.array_equal(d.row_expert.cpu().numpy(), np.repeat(np.arange(cfg.E), np.diff(offsets)))
    # the rows are x's rows in the permuted order, bit for bit (bf16 bits)
    xb = np.asarray(inp.x).view(np.uint16)
    got = d.rows.cpu().view(dtype=__import__("torch").int16).numpy().view(np.uint16)
    assert np.array_equal(got, xb[perm])
    assert d.send_counts == [int(offsets[-1])]


def test_out_of_range_expert_ids_set_the_status_word(cuda_device):
    import torch
    from weight_only_quantized_warp_b200 import expert_parallel as ep
    from weight_only_quantized_warp_b200 import qmoe
    cfg = _cfg(T=16, E=4, k=1)
    inp = _rank_inputs(cfg, 12, 1)[0]
    ops = ep.LibraryOps(cfg, inp, 2, 1, cuda_device)    # experts 2 and 3
    rows = qmoe.to_device(inp.x, cuda_device)
    ok_ids = torch.tensor([2, 3] * 8, dtype=torch.int32, device=cuda_device)
    bad_ids = ok_ids.clone()
    bad_ids[5] = 0                                       # held by the other rank
    bad_ids[9] = 7                                       # no such expert
    ops.expert_rows(rows, bad_ids)
    h = ops.local.handle
    assert qmoe.qmoe_read_device_status(h, ops._rows_ws) == qmoe.QMOE_INVALID_ARGUMENT
    good = ops.expert_rows(rows, ok_ids)
    assert qmoe.qmoe_read_device_status(h, ops._rows_ws) == qmoe.QMOE_OK
    # each row's output is its expert's layers: the oracle with routing forced onto it
    c1 = dataclasses.replace(cfg, k=1)
    lg = np.full((16, cfg.E), -1e30, dtype=np.float32)
    lg[np.arange(16), ok_ids.cpu().numpy()] = 0.0
    ref = oracle.forward(dataclasses.replace(inp, cfg=c1, logits=gen._store(lg, cfg.act_dtype), shared=None))["y"]
    assert max_rel(good.cpu().numpy(), ref) <= TOL_BF16


def _nccl_rank_main(rank, port, out_path):
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from datetime import timedelta

    import torch
    import torch.distributed as dist

    from weight_only_quantized_warp_b200 import expert_parallel as ep
    from weight_only_quantized_warp_b200 import qmoe

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=timedelta(seconds=60), device_id=dev)
    try:
        cfg = _cfg(T=40, E=4, k=2)
        inp = _rank_inputs(cfg, 91, 1)[0]
        ops = ep.LibraryOps(cfg, inp, 1, 0, dev)
        # the collectives forced on: NCCL all-to-alls of the counts, the bf16
        # rows, the int32 expert ids and the fp32 outputs (one rank)
        model = ep.ExpertParallelQMoE(ops, 1, 0, exchange=ep.torch_all_to_all(),
                                      counts=lambda c: ep.exchange_counts(c, dev))
        y = model(qmoe.to_device(inp.x, dev), qmoe.to_device(inp.logits, dev))
        torch.cuda.synchronize()
        np.save(out_path, to_numpy(y))
    finally:
        dist.destroy_process_group()


def test_nccl_all_to_all_path_on_one_rank(cuda_device, tmp_path):
    import socket

    import torch.multiprocessing as mp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    out = str(tmp_path / "y.npy")
    mp.start_processes(_nccl_rank_main, args=(port, out), nprocs=1, join=True, start_method="spawn")
    cfg = _cfg(T=40, E=4, k=2)
    inp = _rank_inputs(cfg, 91, 1)[0]
    err = max_rel(np.load(out), oracle.forward(inp)["y"])
    assert err <= TOL_BF16, f"y max rel err {err:.3e}"


@pytest.mark.parametrize("name", ["int4_bs64", "tensor_core_rows", "weights_on_input_shared_scaled", "int8_tier",
                                  "f32_acts"])
def test_one_rank_split_path_equals_the_fused_forward_bitwise(cuda_device, name):
    """With one rank nothing is exchanged: the split calls run the same plan
    and kernels as qmoe_forward, the expert outputs cross in fp32 and the
    combine rounds once, so y matches the fused forward bit for bit."""
    import torch
    from weight_only_quantized_warp_b200 import expert_parallel as ep
    from weight_only_quantized_warp_b200 import qmoe
    cfg = _cfg(**CASES[name])
    inp = _rank_inputs(cfg, 700 + list(CASES).index(name), 1)[0]
    m = qmoe.QMoE(cfg, cuda_device)
    m.set_weights_from(inp)
    x, lg = qmoe.to_device(inp.x, cuda_device), qmoe.to_device(inp.logits, cuda_device)
    sh = qmoe.to_device(inp.shared, cuda_device)
    y_fused = m.forward(x, lg, sh)
    y_split = ep.ExpertParallelQMoE(ep.LibraryOps(cfg, inp, 1, 0, cuda_device), 1, 0)(x, lg, sh)
    torch.cuda.synchronize()
    assert torch.equal(y_fused.view(torch.int16) if y_fused.dtype == torch.bfloat16 else y_fused,
                       y_split.view(torch.int16) if y_split.dtype == torch.bfloat16 else y_split)
