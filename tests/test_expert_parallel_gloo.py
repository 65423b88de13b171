"""Expert-parallel host logic on CPU process groups (gloo, world size 2).

``weight_only_quantized_warp_b200.expert_parallel`` cuts the forward at its
two exchange points and moves the routed rows between ranks with all-to-all
collectives. These tests run that exchange logic on two real gloo ranks with
the three device steps (dispatch, expert rows, combine) carried out by the
oracle, and check that every rank's output equals the oracle's single-device
forward of its own tokens: the split sizes, the row order across the two
all-to-alls and the expert-id rebasing must all be right for that to hold.
The GPU side of the same three steps is tested through the library in
``test_gpu_expert_parallel.py``.
"""
from __future__ import annotations

import dataclasses
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


CASES = {
    "plain": dict(),
    "weights_on_input_scaled": dict(apply_router_weight_on_input=True, k=1, routed_scaling_factor=2.5,
                                    expert_output_scale=0.5),
    "int8_tier_bias_shared": dict(compute_mode=1, bits=8, block_size=32, has_fc1_bias=True, has_fc2_bias=True,
                                  has_shared=True, normalize=False),
}


def _cfg(name, rank):
    from weight_only_quantized_warp_b200 import inputs as gen
    kw = dict(T=13 + 6 * rank, H=64, I=96, E=4, k=2, bits=4, block_size=32, act=gen.ACT_SWIGLU, fusion=1,
              act_dtype=gen.DT_F32, scale_dtype=gen.DT_F32)
    kw.update(CASES[name])
    return gen.MoEConfig(**kw)


class OracleOps:
    """The three device steps of one rank, done by the oracle on CPU tensors."""

    def __init__(self, inp, world, rank):
        import torch
        from weight_only_quantized_warp_b200 import expert_parallel as ep
        self.inp, self.cfg = inp, inp.cfg
        self.world, self.rank = world, rank
        self.device = torch.device("cpu")
        self.experts = ep.experts_of_rank(self.cfg.E, world, rank)

    def dispatch(self, x, logits, stream=None):
        import torch

        import oracle
        from weight_only_quantized_warp_b200 import expert_parallel as ep
        c = self.cfg
        idx, w = oracle.route(logits.numpy(), c.k, c.normalize, c.n_group, c.topk_group)
        offsets, perm, inv = oracle.permute(idx, c.E)
        T = x.shape[0]
        xs = x.numpy().astype(np.float64)
        rows = np.empty((T * c.k, c.H), dtype=np.float32)
        row_expert = np.empty(T * c.k, dtype=np.int32)
        for t in range(T):
            for j in range(c.k):
                r = inv[t, j]
                v = xs[t] * w[t, j] if c.apply_router_weight_on_input else xs[t]
                rows[r] = v.astype(np.float32)
                row_expert[r] = idx[t, j]
        counts = ep.split_counts(offsets.tolist(), self.world)
        return ep.Dispatched(T, torch.from_numpy(rows), torch.from_numpy(row_expert), counts,
                             dict(idx=idx, w=w, inv=inv))

    def expert_rows(self, rows, row_expert, stream=None):
        """Each row's expert output (o + fc2 bias) of global expert row_expert
        (which must be one of this rank's): the oracle forward of the row alone
        with routing forced onto that expert at weight 1."""
        import torch

        import oracle
        ids = row_expert.numpy()
        assert all(e in self.experts for e in ids.tolist()), "a row reached a rank that does not hold its expert"
        R = rows.shape[0]
        c1 = dataclasses.replace(self.cfg, T=R, k=1, apply_router_weight_on_input=False, routed_scaling_factor=1.0,
                                 expert_output_scale=1.0, n_group=0, topk_group=0, has_shared=False)
        lg = np.full((R, self.cfg.E), -1e30, dtype=np.float32)
        lg[np.arange(R), ids] = 0.0
        one = dataclasses.replace(self.inp, cfg=c1, x=rows.numpy(), logits=lg, shared=None, score_bias=None)
        return torch.from_numpy(oracle.forward(one)["y"].astype(np.float32))

    def combine(self, d, expert_out, shared=None, like=None, stream=None):
        import torch
        c = self.cfg
        s = (c.routed_scaling_factor or 1.0) * (c.expert_output_scale or 1.0)
        o = expert_out.numpy().astype(np.float64)
        y = np.zeros((d.T, c.H))
        for t in range(d.T):
            for j in range(c.k):
                wt = 1.0 if c.apply_router_weight_on_input else d.state["w"][t, j]
                y[t] += wt * o[d.state["inv"][t, j]]
        y *= s
        if shared is not None:
            y += shared.numpy().astype(np.float64)
        return torch.from_numpy(y.astype(np.float32))


def _rank_main(rank, world, port, name, seed, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    from datetime import timedelta

    import torch
    import torch.distributed as dist

    import oracle
    from weight_only_quantized_warp_b200 import expert_parallel as ep
    from weight_only_quantized_warp_b200 import inputs as gen

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=60))
    try:
        # the same weights on every rank (one seed), each rank its own tokens
        w_inp = gen.make_inputs(_cfg(name, 0), seed, bias_std=0.1)
        tok = gen.make_inputs(_cfg(name, rank), seed + 100 + rank, bias_std=0.1)
        inp = dataclasses.replace(w_inp, cfg=tok.cfg, x=tok.x, logits=tok.logits, shared=tok.shared)
        model = ep.ExpertParallelQMoE(OracleOps(inp, world, rank), world, rank)
        sh = None if inp.shared is None else torch.from_numpy(np.asarray(inp.shared, dtype=np.float32))
        y = model(torch.from_numpy(np.asarray(inp.x, dtype=np.float32)),
                  torch.from_numpy(np.asarray(inp.logits, dtype=np.float32)), sh)
        ref = oracle.forward(inp)["y"]
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), y=y.numpy(), ref=ref)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name", list(CASES))
def test_two_gloo_ranks_expert_parallel_equals_one_device(tmp_path, name):
    import oracle
    oracle.build.build()  # once here, not concurrently in both ranks
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), name, 41 + len(name), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    for r in range(world):
        d = np.load(tmp_path / f"rank{r}.npz")
        # fp32 rounding of the expert outputs between the two collectives and of y
        np.testing.assert_allclose(d["y"], d["ref"], rtol=2e-5, atol=2e-6)


def test_rank_expert_ranges_and_split_counts():
    from weight_only_quantized_warp_b200 import expert_parallel as ep
    assert [list(ep.experts_of_rank(8, 4, r)) for r in range(4)] == [[0, 1], [2, 3], [4, 5], [6, 7]]
    with pytest.raises(ValueError):
        ep.experts_of_rank(6, 4, 0)
    # offsets of 8 experts over 2 ranks: rows 0..9 to rank 0, 10..16 to rank 1
    assert ep.split_counts([0, 3, 3, 7, 10, 12, 12, 16, 17], 2) == [10, 7]
    assert ep.split_counts([0, 0, 0, 0, 0], 4) == [0, 0, 0, 0]


def test_local_config_keeps_the_expert_layers_and_drops_routing():
    from weight_only_quantized_warp_b200 import expert_parallel as ep
    from weight_only_quantized_warp_b200 import inputs as gen
    c = gen.MoEConfig(T=4, H=64, I=96, E=8, k=3, n_group=4, topk_group=2, routed_scaling_factor=2.0,
                      apply_router_weight_on_input=True, expert_output_scale=3.0, has_fc2_bias=True,
                      compute_mode=1, block_size=32)
    lc = ep.local_config(c, 4, 1)
    assert (lc.E, lc.k, lc.n_group, lc.topk_group) == (2, 1, 0, 0)
    assert (lc.routed_scaling_factor, lc.expert_output_scale, lc.apply_router_weight_on_input) == (1.0, 1.0, False)
    assert (lc.H, lc.I, lc.bits, lc.block_size, lc.has_fc2_bias, lc.compute_mode) == (64, 96, 4, 32, True, 1)
