"""Shared plumbing for the GPU parity tests: run one forward through the C ABI
and the oracle on the same seeded inputs, and compare stage by stage."""
from __future__ import annotations

import dataclasses

import numpy as np

import oracle
from weight_only_quantized_warp_b200 import inputs as gen

# Tolerances (max |gpu - ref| / max |ref| over a tensor): bf16 activations with
# fp32 accumulation, and fp32 activations.
TOL_BF16 = 1e-2
TOL_F32 = 1e-4
# Router weights: fp32 expf/division against fp64.
TOL_ROUTE_W = 2e-6


def max_rel(got: np.ndarray, ref: np.ndarray) -> float:
    den = float(np.abs(ref).max())
    if den == 0.0:
        return float(np.abs(got).max())
    return float(np.abs(got - ref).max()) / den


def to_numpy(t) -> np.ndarray:
    import torch
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy()


@dataclasses.dataclass
class GpuRun:
    y: np.ndarray
    topk_idx: np.ndarray
    topk_w: np.ndarray
    offsets: np.ndarray
    perm: np.ndarray
    inv: np.ndarray
    hidden: np.ndarray  # [T*k, I] in permuted row order
    path: int


def run_gpu(inp: gen.MoEInputs, device="cuda:0", repeat: int = 1, path=None) -> GpuRun:
    """path: None (chosen by shape), 1 (weight-streaming kernels) or 2
    (tcgen05 grouped GEMM); ignored for fp32 activations."""
    import torch
    from weight_only_quantized_warp_b200 import qmoe
    c = inp.cfg
    m = qmoe.QMoE(c, device, path=path if c.act_dtype == gen.DT_BF16 else None)
    m.set_weights_from(inp)
    x = qmoe.to_device(inp.x, device)
    lg = qmoe.to_device(inp.logits, device)
    sh = qmoe.to_device(inp.shared, device)
    y = None
    for _ in range(repeat):
        y = m.forward(x, lg, sh)
    T, k, E = c.T, c.k, c.E
    R = T * k
    i32 = dict(dtype=torch.int32, device=device)
    idx = torch.empty((T, k), **i32)
    w = torch.empty((T, k), dtype=torch.float32, device=device)
    off = torch.empty(E + 1, **i32)
    perm = torch.empty(max(R, 1), **i32)
    inv = torch.empty((T, k), **i32)
    ws = m.workspace(T)
    qmoe.qmoe_debug_routing(m.handle, T, ws, idx, w, off, perm, inv)
    hid = torch.empty((max(R, 1), c.I), dtype=x.dtype, device=device)
    qmoe.qmoe_debug_hidden(m.handle, T, ws, hid)
    torch.cuda.synchronize()
    status = qmoe.qmoe_read_device_status(m.handle, ws)
    assert status == qmoe.QMOE_OK, f"device status {status}"
    path = qmoe.qmoe_path_for(m.handle, T)
    return GpuRun(to_numpy(y), idx.cpu().numpy(), w.cpu().numpy(), off.cpu().numpy(),
                  perm.cpu().numpy()[:R], inv.cpu().numpy(), to_numpy(hid)[:R], path)


def check_routing(inp: gen.MoEInputs, g: GpuRun):
    c = inp.cfg
    idx, w = oracle.route(inp.logits, c.k, c.normalize, c.n_group, c.topk_group)
    np.testing.assert_array_equal(g.topk_idx, idx)
    np.testing.assert_allclose(g.topk_w, w, rtol=TOL_ROUTE_W, atol=1e-30)
    off, perm, inv = oracle.permute(idx, c.E)
    np.testing.assert_array_equal(g.offsets, off)
    np.testing.assert_array_equal(g.perm, perm)
    np.testing.assert_array_equal(g.inv, inv)


def check_full(inp: gen.MoEInputs, g: GpuRun, check_hidden: bool = True):
    c = inp.cfg
    tol = TOL_BF16 if c.act_dtype == gen.DT_BF16 else TOL_F32
    check_routing(inp, g)
    ref = oracle.forward(inp, want_h=check_hidden)
    err = max_rel(g.y, ref["y"])
    assert err <= tol, f"y max rel err {err:.3e} > {tol}"
    if check_hidden and c.T > 0:
        # oracle h row t*k+j sits at permuted row inv[t, j]
        h_gpu = g.hidden[g.inv.reshape(-1)]
        herr = max_rel(h_gpu, ref["h"])
        assert herr <= tol, f"h max rel err {herr:.3e} > {tol}"
    return err


def check_sampled(inp: gen.MoEInputs, g: GpuRun, tokens):
    """Full-size runs: routing and permutation in full, outputs on sampled
    token rows that the oracle computes one by one."""
    c = inp.cfg
    tol = TOL_BF16 if c.act_dtype == gen.DT_BF16 else TOL_F32
    check_routing(inp, g)
    ref = oracle.forward(inp, tokens=tokens)
    err = max_rel(g.y[tokens], ref["y"])
    assert err <= tol, f"sampled y max rel err {err:.3e} > {tol}"
    return err
