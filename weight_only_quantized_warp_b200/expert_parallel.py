"""Expert-parallel execution of the QMoE forward: experts spread over ranks.

Each of G ranks holds E / G consecutive experts (rank r: experts
r*E/G .. (r+1)*E/G - 1) in its own library handle, and routes its own tokens
with a routing handle of the full expert set. One forward is the single-GPU
forward ("ClikaRT::nn::QMoEWoQ", forward(); the "MoE" page's routed combine)
cut at its two exchange points:

1. dispatch (token owner): route, sort the T*k routes by expert and gather
   x's rows in that order (``qmoe_ep_dispatch``). Expert order is rank order,
   so the rows for rank r are one contiguous range, found from the expert
   offsets at the rank boundaries.
2. all-to-all of the rows and their global expert ids (NCCL over NVLink on
   GPUs, gloo in the CPU tests), after one all-to-all of the row counts.
3. expert rows (expert owner): FC1, activation, FC2 and the fc2 bias of each
   received row, fp32 out (``qmoe_ep_expert_rows``).
4. all-to-all back, with the counts of step 2 reversed: the outputs arrive in
   the order the rows left.
5. combine (token owner): router weights, scaling factors and the shared
   output, one rounding (``qmoe_ep_combine``).

Every step on the data runs in the library's kernels; this module only sizes
buffers, reads the per-rank row counts (one small device-to-host copy per
forward: the all-to-all needs its split sizes on the host) and calls the
collectives. The device operations are an object with ``dispatch``,
``expert_rows`` and ``combine`` (``LibraryOps`` here), so the exchange logic
can be tested on CPU ranks with another implementation of the same three
steps.
"""
from __future__ import annotations

import dataclasses
from typing import Callable, List, Optional, Sequence


def experts_of_rank(E: int, world: int, rank: int) -> range:
    """The experts rank ``rank`` holds: a contiguous E / world range."""
    if world < 1 or E % world:
        raise ValueError(f"num_experts ({E}) must be a multiple of the number of ranks ({world})")
    n = E // world
    return range(rank * n, (rank + 1) * n)


def local_config(cfg, world: int, rank: int):
    """The expert owner's config: its experts only; routing attributes are
    not used by the rows entry (k = 1 keeps the config valid for any E / G)."""
    n = len(experts_of_rank(cfg.E, world, rank))
    return dataclasses.replace(cfg, E=n, k=1, n_group=0, topk_group=0, routed_scaling_factor=1.0,
                               apply_router_weight_on_input=False, expert_output_scale=1.0,
                               has_score_bias=False, has_shared=False)


def split_counts(offsets: Sequence[int], world: int) -> List[int]:
    """Rows for each rank from the dispatch's expert offsets [E + 1]."""
    E = len(offsets) - 1
    n = E // world
    return [int(offsets[(r + 1) * n]) - int(offsets[r * n]) for r in range(world)]


@dataclasses.dataclass
class Dispatched:
    """What the token owner keeps between dispatch and combine."""
    T: int
    rows: object            # [T*k, H] in expert order
    row_expert: object      # [T*k] global expert ids
    send_counts: List[int]  # rows to each rank
    state: object           # routing state for the combine


class LibraryOps:
    """The three device steps through the library's C ABI (one GPU)."""

    def __init__(self, cfg, inputs, world: int, rank: int, device=None):
        import torch
        from . import qmoe
        self.q = qmoe
        self.cfg = cfg
        self.world, self.rank = world, rank
        self.device = torch.device(device or "cuda")
        self.experts = experts_of_rank(cfg.E, world, rank)
        # routing handle: the full expert set, no weights
        self.router = qmoe.qmoe_create(qmoe.make_config(cfg))
        sb = getattr(inputs, "score_bias", None)
        if sb is not None:
            qmoe.qmoe_set_score_correction_bias(self.router, qmoe.to_device(sb, self.device))
        # expert handle: this rank's experts
        lo, hi = self.experts.start, self.experts.stop
        self.local = qmoe.QMoE(local_config(cfg, world, rank), self.device)
        sl = lambda a: None if a is None else a[lo:hi]  # noqa: E731
        d = self.device
        self.local.set_weights(*(qmoe.to_device(sl(getattr(inputs, n)), d) for n in ("fc1_w", "fc1_s", "fc2_w", "fc2_s")),
                               fc1_b=qmoe.to_device(sl(inputs.fc1_b), d), fc2_b=qmoe.to_device(sl(inputs.fc2_b), d),
                               fc3_w=qmoe.to_device(sl(inputs.fc3_w), d), fc3_s=qmoe.to_device(sl(inputs.fc3_s), d),
                               fc3_b=qmoe.to_device(sl(inputs.fc3_b), d))
        self._rows_ws = None

    def close(self):
        if self.router:
            self.q.qmoe_destroy(self.router)
            self.router = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # interpreter shutdown
            pass

    def dispatch(self, x, logits, stream=None) -> Dispatched:
        import torch
        T, k, E = x.shape[0], self.cfg.k, self.cfg.E
        rows = torch.empty((T * k, x.shape[1]), dtype=x.dtype, device=self.device)
        row_expert = torch.empty(T * k, dtype=torch.int32, device=self.device)
        offsets = torch.empty(E + 1, dtype=torch.int32, device=self.device)
        nstate = max(self.q.qmoe_ep_state_bytes(self.router, T), 256)
        state = torch.empty(nstate, dtype=torch.uint8, device=self.device)
        if T:
            self.q.qmoe_ep_dispatch(self.router, T, x, logits, rows, row_expert, offsets, state, nstate, stream)
            counts = split_counts(offsets.cpu().tolist(), self.world)
        else:
            counts = [0] * self.world
        return Dispatched(T, rows, row_expert, counts, state)

    def expert_rows(self, rows, row_expert, stream=None):
        import torch
        R = rows.shape[0]
        out = torch.empty((R, rows.shape[1]), dtype=torch.float32, device=self.device)
        if R:
            n = self.q.qmoe_ep_rows_workspace_size(self.local.handle, R)
            if self._rows_ws is None or self._rows_ws.numel() < n:
                self._rows_ws = torch.empty(max(n, 256), dtype=torch.uint8, device=self.device)
            self.q.qmoe_ep_expert_rows(self.local.handle, R, rows, row_expert, self.experts.start, out,
                                       self._rows_ws, self._rows_ws.numel(), stream)
        return out

    def combine(self, d: Dispatched, expert_out, shared=None, y=None, like=None, stream=None):
        import torch
        if y is None:
            y = torch.empty((d.T, self.cfg.H), dtype=like.dtype if like is not None else torch.bfloat16,
                            device=self.device)
        if d.T:
            self.q.qmoe_ep_combine(self.router, d.T, expert_out, d.state, shared, y, stream)
        return y


def torch_all_to_all(group=None) -> Callable:
    """all_to_all of a row tensor with host-known split sizes over a
    torch.distributed group (NCCL on GPUs, gloo on CPU)."""
    import torch
    import torch.distributed as dist

    def exchange(send, send_counts: List[int], recv_counts: List[int]):
        recv = torch.empty((sum(recv_counts),) + tuple(send.shape[1:]), dtype=send.dtype, device=send.device)
        dist.all_to_all_single(recv, send.contiguous(), output_split_sizes=recv_counts,
                               input_split_sizes=send_counts, group=group)
        return recv

    return exchange


def exchange_counts(send_counts: List[int], device, group=None) -> List[int]:
    """Each rank's row counts for every other rank (one all-to-all)."""
    import torch
    import torch.distributed as dist
    s = torch.tensor(send_counts, dtype=torch.int64, device=device)
    r = torch.empty_like(s)
    dist.all_to_all_single(r, s, group=group)
    return [int(v) for v in r.cpu().tolist()]


class ExpertParallelQMoE:
    """One rank of an expert-parallel QMoE operator.

    ``ops`` performs the three device steps (``LibraryOps`` for the GPU);
    ``exchange(send, send_counts, recv_counts)`` moves rows between ranks and
    ``counts(send_counts)`` returns the counts every rank sends here. Both
    default to torch.distributed collectives on ``group``; with one rank no
    collective runs.
    """

    def __init__(self, ops, world: int, rank: int, group=None, exchange: Optional[Callable] = None,
                 counts: Optional[Callable] = None):
        self.ops, self.world, self.rank = ops, world, rank
        if world > 1:
            self.exchange = exchange or torch_all_to_all(group)
            self.counts = counts or (lambda c: exchange_counts(c, ops.device, group))
        else:
            self.exchange = exchange or (lambda send, sc, rc: send)
            self.counts = counts or (lambda c: list(c))

    def forward(self, x, logits, shared=None, stream=None):
        d = self.ops.dispatch(x, logits, stream)
        recv_counts = self.counts(d.send_counts)
        rows = self.exchange(d.rows, d.send_counts, recv_counts)
        ids = self.exchange(d.row_expert, d.send_counts, recv_counts)
        out = self.ops.expert_rows(rows, ids, stream)
        back = self.exchange(out, recv_counts, d.send_counts)
        return self.ops.combine(d, back, shared, like=x, stream=stream)

    __call__ = forward
