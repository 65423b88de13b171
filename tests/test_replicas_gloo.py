"""Multi-rank host logic on CPU process groups (gloo, world size 2).

The forward shards by tokens: each rank runs the whole operator on its own
batch with the same weights and no exchange on the data path. These tests
check, with two real ranks, that (a) every rank builds the same expert
weights and its own token batch, (b) the union of the ranks' outputs equals
one forward over the concatenated batch (so the replicas compute exactly what
one big batch would), and (c) the timing reduction takes the slowest rank and
the job throughput counts every rank's tokens.
"""
from __future__ import annotations

import hashlib
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


def _digest(*arrays) -> str:
    h = hashlib.sha256()
    for a in arrays:
        if a is not None:
            h.update(np.ascontiguousarray(a).tobytes())
    return h.hexdigest()


def _rank_main(rank, world, port, workload, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    from datetime import timedelta

    import torch.distributed as dist

    import oracle
    from weight_only_quantized_warp_b200 import replicas

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=60))
    try:
        inp = replicas.replica_inputs(workload, rank)
        ref = oracle.forward(inp)
        digests = [None] * world
        dist.all_gather_object(digests, {
            "weights": _digest(inp.fc1_w, inp.fc1_s, inp.fc2_w, inp.fc2_s, inp.fc3_w, inp.fc3_s,
                               inp.fc1_b, inp.fc2_b, inp.fc3_b),
            "tokens": _digest(inp.x, inp.logits, inp.shared)})
        # rank r took 10 + r ms; the job's time is the slowest rank's
        slowest = replicas.max_over_ranks([10.0 + rank, 5.0 - rank])
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), y=ref["y"], x=inp.x, logits=inp.logits,
                 shared=inp.shared if inp.shared is not None else np.zeros(0),
                 slowest=np.array(slowest), same_weights=np.array(
                     all(d["weights"] == digests[0]["weights"] for d in digests)),
                 distinct_tokens=np.array(len({d["tokens"] for d in digests}) == world))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("workload", ["tiny", "tiny_i8"])
def test_two_gloo_replicas_equal_one_batch(tmp_path, workload):
    import oracle
    from weight_only_quantized_warp_b200 import inputs as gen
    from weight_only_quantized_warp_b200 import replicas

    oracle.build.build()  # build once here, not concurrently in both ranks
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), workload, str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    r = [np.load(tmp_path / f"rank{i}.npz") for i in range(world)]
    for d in r:
        assert bool(d["same_weights"])
        assert bool(d["distinct_tokens"])
        np.testing.assert_array_equal(d["slowest"], [11.0, 5.0])

    # one forward over the concatenated batch gives the ranks' rows
    whole = replicas.replica_inputs(workload, 0)
    whole.x = np.concatenate([d["x"] for d in r])
    whole.logits = np.concatenate([d["logits"] for d in r])
    if whole.cfg.has_shared:
        whole.shared = np.concatenate([d["shared"] for d in r])
    whole.cfg = gen.MoEConfig(**{**whole.cfg.__dict__, "T": whole.x.shape[0]})
    y = oracle.forward(whole)["y"]
    np.testing.assert_array_equal(y, np.concatenate([d["y"] for d in r]))


def test_job_throughput_counts_every_rank():
    from weight_only_quantized_warp_b200 import replicas
    # 8 tokens per rank per step, 4 ranks, 10 steps, slowest rank 2 ms
    assert replicas.job_tokens_per_s(8, 4, 10, 2.0) == pytest.approx(8 * 4 * 10 / 2e-3)
    with pytest.raises(ValueError):
        replicas.job_tokens_per_s(8, 1, 1, 0.0)


def test_max_over_ranks_without_a_group_is_identity():
    from weight_only_quantized_warp_b200 import replicas
    assert replicas.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]


def test_rank_batches_are_seeded_and_reproducible():
    from weight_only_quantized_warp_b200 import replicas
    a = replicas.replica_inputs("tiny", 1)
    b = replicas.replica_inputs("tiny", 1)
    c = replicas.replica_inputs("tiny", 0)
    np.testing.assert_array_equal(a.x, b.x)
    np.testing.assert_array_equal(a.fc1_w, c.fc1_w)
    assert not np.array_equal(a.x, c.x)
