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
    hidden: np.ndarray  # [T*k, I] in permuted row order, or the sampled tokens' rows
    path: int
    tile: int = 0       # token tile of the tensor-core paths (0 otherwise)


def run_gpu(inp: gen.MoEInputs, device="cuda:0", repeat: int = 1, path=None, hidden_tokens=None) -> GpuRun:
    """path: None (chosen by shape), 1 (weight-streaming kernels) or 2
    (tcgen05 grouped GEMM); ignored for fp32 activations. hidden_tokens:
    copy back only the h rows of these tokens ([len * k, I], token-major),
    for full-size runs whose whole h would not fit the host comfortably."""
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
    if hidden_tokens is not None:
        rows = inv[torch.as_tensor(np.asarray(hidden_tokens), device=device, dtype=torch.long)].reshape(-1)
        hid = hid[rows.long()]
    else:
        hid = hid[:R]
    torch.cuda.synchronize()
    status = qmoe.qmoe_read_device_status(m.handle, ws)
    assert status == qmoe.QMOE_OK, f"device status {status}"
    path = qmoe.qmoe_path_for(m.handle, T)
    tile = qmoe.qmoe_token_tile_for(m.handle, T)
    return GpuRun(to_numpy(y), idx.cpu().numpy(), w.cpu().numpy(), off.cpu().numpy(),
                  perm.cpu().numpy()[:R], inv.cpu().numpy(), to_numpy(hid), path, tile)


def check_routing(inp: gen.MoEInputs, g: GpuRun):
    c = inp.cfg
    idx, w = oracle.route(inp.logits, c.k, c.normalize, c.n_group, c.topk_group,
                          score_bias=getattr(inp, "score_bias", None))
    np.testing.assert_array_equal(g.topk_idx, idx)
    np.testing.assert_allclose(g.topk_w, w, rtol=TOL_ROUTE_W, atol=1e-30)
    off, perm, inv = oracle.permute(idx, c.E)
    np.testing.assert_array_equal(g.offsets, off)
    np.testing.assert_array_equal(g.perm, perm)
    np.testing.assert_array_equal(g.inv, inv)


def elementwise_rel(got: np.ndarray, ref: np.ndarray) -> float:
    """Largest |got - ref| / |ref| over the elements with |ref| >= 0.1 rms(ref)
    (the element-wise error reported beside the per-tensor tolerance)."""
    rms = float(np.sqrt(np.mean(np.square(ref)))) if ref.size else 0.0
    sel = np.abs(ref) >= 0.1 * rms
    if rms == 0.0 or not sel.any():
        return 0.0
    return float((np.abs(got[sel] - ref[sel]) / np.abs(ref[sel])).max())


# per-test parity figures, written out by conftest when QMOE_PARITY_REPORT names a file
REPORT: list = []


def _record(name, **kw):
    REPORT.append(dict(case=name, **kw))


def check_full(inp: gen.MoEInputs, g: GpuRun, check_hidden: bool = True, name: str = ""):
    c = inp.cfg
    tol = TOL_BF16 if c.act_dtype == gen.DT_BF16 else TOL_F32
    check_routing(inp, g)
    ref = oracle.forward(inp, want_h=check_hidden)
    err = max_rel(g.y, ref["y"])
    _record(name or f"T{c.T}_H{c.H}_I{c.I}_E{c.E}_k{c.k}", path=g.path, tile=g.tile, y_max_rel=err,
            y_elementwise=elementwise_rel(g.y, ref["y"]))
    assert err <= tol, f"y max rel err {err:.3e} > {tol}"
    if check_hidden and c.T > 0:
        # oracle h row t*k+j sits at permuted row inv[t, j]
        h_gpu = g.hidden[g.inv.reshape(-1)]
        herr = max_rel(h_gpu, ref["h"])
        assert herr <= tol, f"h max rel err {herr:.3e} > {tol}"
    return err


def check_sampled(inp: gen.MoEInputs, g: GpuRun, tokens, name: str = "", hidden: bool = False):
    """Full-size runs: routing and permutation in full, outputs on sampled
    token rows that the oracle computes one by one. hidden: g.hidden holds
    the h rows of exactly these tokens (run_gpu's hidden_tokens), compared
    with the oracle's h of the same (token, slot) pairs."""
    c = inp.cfg
    tol = TOL_BF16 if c.act_dtype == gen.DT_BF16 else TOL_F32
    check_routing(inp, g)
    ref = oracle.forward(inp, tokens=tokens, want_h=hidden)
    err = max_rel(g.y[tokens], ref["y"])
    rec = dict(path=g.path, tile=g.tile, tokens=len(tokens), y_max_rel=err,
               y_elementwise=elementwise_rel(g.y[tokens], ref["y"]))
    herr = None
    if hidden:
        herr = max_rel(g.hidden, ref["h"])
        rec.update(h_max_rel=herr, h_elementwise=elementwise_rel(g.hidden, ref["h"]))
    _record(name or f"T{c.T}_H{c.H}_I{c.I}_E{c.E}_k{c.k}", **rec)
    assert err <= tol, f"sampled y max rel err {err:.3e} > {tol}"
    if hidden:
        assert herr <= tol, f"sampled h max rel err {herr:.3e} > {tol}"
    return err


def boundary_tokens(g: GpuRun, k: int, per_tile: int = 2, extra: int = 0, seed: int = 0):
    """Tokens whose routed rows sit at the ends of every expert segment and
    on both sides of token-tile boundaries inside each segment (the first
    and last tile boundaries when a segment has many), plus ``extra`` random
    tokens: every expert, both ends of its tiles, and (through the FC2 K
    split) every split's partial are then compared."""
    rows = set()
    off = g.offsets
    tile = g.tile if g.tile > 0 else 8
    for e in range(len(off) - 1):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi <= lo:
            continue
        rows.update({lo, hi - 1})
        inner = list(range(lo + tile, hi, tile))
        for b in inner[:per_tile] + inner[-per_tile:]:
            rows.update({b - 1, b})
    toks = {int(g.perm[r]) for r in rows}
    if extra:
        rng = np.random.default_rng(seed)
        T = g.inv.shape[0]
        toks.update(rng.choice(T, size=min(extra, T), replace=False).tolist())
    return np.array(sorted(toks), dtype=np.int64)
