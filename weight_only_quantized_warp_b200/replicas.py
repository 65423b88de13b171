"""Data-parallel replicas of the QMoE forward: one process per GPU.

Every token of the operator is routed, passed through its experts and
combined independently of every other token (QMoE operator page, the
operator's inputs are per-token rows and its output row t depends only on
input row t and the shared weights). A job over many GPUs therefore needs no
exchange on the data path: each rank holds the same packed expert weights and
runs the whole forward on its own token batch. The only cross-rank traffic is
the timing reduction (the job's time is the slowest rank's) and the barriers
that line up the timed regions.

This module holds the host-side pieces of that scheme, so that they can be
exercised on CPU process groups as well as on NCCL ones.
"""
from __future__ import annotations

from . import inputs as gen

# Seed offset between the token batches of consecutive ranks.
RANK_SEED_STRIDE = 1000


def replica_inputs(name: str, rank: int) -> gen.MoEInputs:
    """The named workload's inputs as rank ``rank`` sees them: the workload's
    own expert weights on every rank; rank 0 keeps the workload's token batch,
    rank r > 0 draws its own (same shapes and distributions) from the seed
    ``workload seed + RANK_SEED_STRIDE * r``."""
    cfg, seed, kw = gen.workload(name)
    inp = gen.make_inputs(cfg, seed, **kw)
    if rank > 0:
        inp.x, inp.logits, shared = gen.make_token_batch(cfg, seed + RANK_SEED_STRIDE * rank, **kw)
        if cfg.has_shared:
            inp.shared = shared
    return inp


def max_over_ranks(values, device=None):
    """Element-wise maximum of a list of floats over all ranks of the default
    process group (the identity without one, or with a single rank)."""
    import torch
    import torch.distributed as dist
    vals = [float(v) for v in values]
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu().tolist()]


def job_tokens_per_s(tokens_per_rank_step: int, world: int, steps: int, slowest_ms: float) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    if slowest_ms <= 0.0:
        raise ValueError("timed region must be positive")
    return tokens_per_rank_step * world * steps / (slowest_ms / 1e3)
