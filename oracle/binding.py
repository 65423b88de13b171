"""ctypes binding of the C oracle (test infrastructure only).

Float inputs may be fp32 arrays or bf16 bit patterns (``np.uint16``); both
are widened to fp64 exactly before the C code sees them ("read inputs at
their stored precision").
"""
from __future__ import annotations

import ctypes
import math
from typing import Optional, Sequence

import numpy as np

from . import build as _build

_lib = None

_f64p = ctypes.POINTER(ctypes.c_double)
_i32p = ctypes.POINTER(ctypes.c_int32)
_u8p = ctypes.POINTER(ctypes.c_uint8)


class _Cfg(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("H", ctypes.c_int64), ("I", ctypes.c_int64),
                ("E", ctypes.c_int64), ("k", ctypes.c_int64), ("bits", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("act", ctypes.c_int32),
                ("fusion", ctypes.c_int32), ("normalize", ctypes.c_int32),
                ("has_fc3", ctypes.c_int32), ("alpha", ctypes.c_double),
                ("beta", ctypes.c_double), ("limit", ctypes.c_double),
                ("n_group", ctypes.c_int32), ("topk_group", ctypes.c_int32),
                ("apply_router_weight_on_input", ctypes.c_int32),
                ("routed_scaling_factor", ctypes.c_double),
                ("mxfp4", ctypes.c_int32), ("act_bf16", ctypes.c_int32),
                ("int8_block", ctypes.c_int32), ("pad_", ctypes.c_int32),
                ("expert_output_scale", ctypes.c_double),
                ("score_bias", ctypes.c_void_p)]


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        lib.oracle_forward.restype = ctypes.c_int
        lib.oracle_gated_act.restype = ctypes.c_double
        lib.oracle_gated_act.argtypes = [ctypes.c_int32] + [ctypes.c_double] * 5
        lib.oracle_plain_act.restype = ctypes.c_double
        lib.oracle_plain_act.argtypes = [ctypes.c_int32, ctypes.c_double]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_e2m1.restype = ctypes.c_double
        lib.oracle_e2m1.argtypes = [ctypes.c_int32]
        lib.oracle_round_act.restype = ctypes.c_double
        lib.oracle_round_act.argtypes = [ctypes.c_double, ctypes.c_int32]
        _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def to_f64(a: Optional[np.ndarray]) -> Optional[np.ndarray]:
    """Widen stored values to fp64: uint16 arrays are bf16 bit patterns,
    uint8 arrays E8M0 scales (2^(x - 127); x = 255 is NaN)."""
    if a is None:
        return None
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return np.ascontiguousarray((a.astype(np.uint32) << 16).view(np.float32).astype(np.float64))
    if a.dtype == np.uint8:
        v = np.ldexp(1.0, a.astype(np.int64) - 127)
        return np.ascontiguousarray(np.where(a == 255, np.nan, v))
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a, typ):
    return None if a is None else a.ctypes.data_as(typ)


def unpack(packed: np.ndarray, N: int, K: int, bits: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    assert packed.size == N * K * bits // 8
    q = np.empty((N, K), dtype=np.int32)
    _load().oracle_unpack(_p(packed, _u8p), ctypes.c_int64(N), ctypes.c_int64(K),
                          ctypes.c_int32(bits), _p(q, _i32p))
    return q


def dequant(packed: np.ndarray, scales: np.ndarray, N: int, K: int, bits: int,
            block_size: int, mxfp4: bool = False) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    s = to_f64(scales)
    assert s.size == (N * (K // block_size) if block_size > 0 else N)
    w = np.empty((N, K), dtype=np.float64)
    _load().oracle_dequant(_p(packed, _u8p), _p(s, _f64p), ctypes.c_int64(N), ctypes.c_int64(K),
                           ctypes.c_int32(bits), ctypes.c_int64(block_size), ctypes.c_int32(int(mxfp4)),
                           _p(w, _f64p))
    return w


def route(logits: np.ndarray, k: int, normalize: bool, n_group: int = 0, topk_group: int = 0,
          score_bias: Optional[np.ndarray] = None):
    """Top-k routing of ``logits`` [T, E]; ``score_bias`` [E] (fp32 values,
    the e_score_correction_bias) shifts the selection keys only."""
    lg = to_f64(logits)
    T, E = lg.shape
    sb = None if score_bias is None else to_f64(np.asarray(score_bias, dtype=np.float32))
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    _load().oracle_route(_p(lg, _f64p), ctypes.c_int64(T), ctypes.c_int64(E), ctypes.c_int64(k),
                         ctypes.c_int32(int(normalize)), ctypes.c_int32(n_group), ctypes.c_int32(topk_group),
                         _p(sb, _f64p), _p(idx, _i32p), _p(w, _f64p))
    return idx, w


def permute(idx: np.ndarray, E: int):
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    offsets = np.empty(E + 1, dtype=np.int32)
    perm = np.empty(T * k, dtype=np.int32)
    inv = np.empty((T, k), dtype=np.int32)
    _load().oracle_permute(_p(idx, _i32p), ctypes.c_int64(T), ctypes.c_int64(E), ctypes.c_int64(k),
                           _p(offsets, _i32p), _p(perm, _i32p), _p(inv, _i32p))
    return offsets, perm, inv


def e2m1(code: int) -> float:
    """Value of one MXFP4 (e2m1) code."""
    return float(_load().oracle_e2m1(code))


def round_act(v: float, bf16: bool) -> float:
    """Round one value to the activation dtype (nearest, ties to even)."""
    return float(_load().oracle_round_act(float(v), int(bf16)))


def quantize_i8(x: np.ndarray, block_size: int):
    """Per-block int8 rounding of activation rows (int8 block compute tier).

    ``x`` [rows, K] (fp32 values or bf16 bit patterns). Returns the codes
    [rows, K] int8 and the scales [rows, K / block_size] float32."""
    v = to_f64(x)
    rows, K = v.shape
    q = np.empty((rows, K), dtype=np.int8)
    s = np.empty((rows, K // block_size), dtype=np.float32)
    lib = _load()
    for r in range(rows):
        lib.oracle_quantize_i8(_p(np.ascontiguousarray(v[r]), _f64p), ctypes.c_int64(K),
                               ctypes.c_int64(block_size),
                               q[r].ctypes.data_as(ctypes.POINTER(ctypes.c_int8)),
                               s[r].ctypes.data_as(ctypes.POINTER(ctypes.c_float)))
    return q, s


def linear_i8(x: np.ndarray, packed: np.ndarray, scales: np.ndarray, N: int, K: int, bits: int,
              block_size: int) -> np.ndarray:
    """The int8-tier dot of activation rows ``x`` [rows, K] (values as stored;
    they are widened, not rounded) with the packed weight [N, K]: [rows, N] fp64."""
    v = to_f64(x)
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    s = to_f64(scales)
    rows = v.shape[0]
    y = np.empty((rows, N), dtype=np.float64)
    _load().oracle_linear_i8(_p(v, _f64p), ctypes.c_int64(rows), _p(packed, _u8p), _p(s, _f64p),
                             ctypes.c_int64(N), ctypes.c_int64(K), ctypes.c_int32(bits),
                             ctypes.c_int64(block_size), _p(y, _f64p))
    return y


def gated_act(act: int, g: float, u: float, alpha: float, beta: float, limit: float) -> float:
    return float(_load().oracle_gated_act(act, g, u, alpha, beta, limit))


def plain_act(act: int, a: float) -> float:
    return float(_load().oracle_plain_act(act, a))


def forward(inp, tokens: Optional[Sequence[int]] = None, want_h: bool = False) -> dict:
    """Run the whole forward on ``inp`` (an object with the fields of a
    generated input set: ``cfg``, ``x``, ``logits``, ``fc1_w`` ... ``shared``).

    ``tokens`` restricts the run to a subset of token rows (tokens are
    independent, so the result equals those rows of the full output).
    Returns ``y`` [T', H] fp64 (unrounded), ``topk_idx``, ``topk_w`` and,
    with ``want_h``, ``h`` [T'*k, I].
    """
    c = inp.cfg
    x = to_f64(inp.x)
    lg = to_f64(inp.logits)
    sh = to_f64(inp.shared)
    if tokens is not None:
        tokens = np.asarray(tokens, dtype=np.int64)
        x, lg = np.ascontiguousarray(x[tokens]), np.ascontiguousarray(lg[tokens])
        sh = None if sh is None else np.ascontiguousarray(sh[tokens])
    T = x.shape[0]
    sb = getattr(inp, "score_bias", None)
    sb = None if sb is None else to_f64(np.asarray(sb, dtype=np.float32))
    eos = float(getattr(c, "expert_output_scale", 1.0) or 1.0)
    act = 5 if (c.act == 1 and int(getattr(c, "gelu_mode", 0)) == 1) else c.act  # GELU, tanh form
    cfg = _Cfg(T=T, H=c.H, I=c.I, E=c.E, k=c.k, bits=c.bits, block_size=c.block_size,
               act=act, fusion=c.fusion, normalize=int(c.normalize), has_fc3=int(c.has_fc3),
               alpha=float(c.alpha), beta=float(c.beta),
               limit=float(c.limit) if c.limit is not None else math.inf,
               n_group=int(c.n_group), topk_group=int(c.topk_group),
               apply_router_weight_on_input=int(c.apply_router_weight_on_input),
               routed_scaling_factor=float(c.routed_scaling_factor) if c.routed_scaling_factor else 1.0,
               mxfp4=int(c.weight_format == 1),
               act_bf16=int(np.asarray(inp.x).dtype == np.uint16),
               int8_block=int(getattr(c, "compute_mode", 0) == 1),
               expert_output_scale=eos, score_bias=None if sb is None else sb.ctypes.data)
    y = np.empty((T, c.H), dtype=np.float64)
    idx = np.empty((T, c.k), dtype=np.int32)
    w = np.empty((T, c.k), dtype=np.float64)
    h = np.empty((T * c.k, c.I), dtype=np.float64) if want_h else None
    u8 = lambda a: None if a is None else np.ascontiguousarray(a, dtype=np.uint8)  # noqa: E731
    f1w, f2w, f3w = u8(inp.fc1_w), u8(inp.fc2_w), u8(inp.fc3_w)
    f1s, f2s, f3s = to_f64(inp.fc1_s), to_f64(inp.fc2_s), to_f64(inp.fc3_s)
    f1b, f2b, f3b = to_f64(inp.fc1_b), to_f64(inp.fc2_b), to_f64(inp.fc3_b)
    rc = _load().oracle_forward(
        ctypes.byref(cfg), _p(x, _f64p), _p(lg, _f64p),
        _p(f1w, _u8p), _p(f1s, _f64p), _p(f1b, _f64p),
        _p(f2w, _u8p), _p(f2s, _f64p), _p(f2b, _f64p),
        _p(f3w, _u8p), _p(f3s, _f64p), _p(f3b, _f64p),
        _p(sh, _f64p), _p(y, _f64p), _p(idx, _i32p), _p(w, _f64p), _p(h, _f64p))
    if rc != 0:
        raise MemoryError("oracle_forward: allocation failed")
    out = dict(y=y, topk_idx=idx, topk_w=w)
    if want_h:
        out["h"] = h
    return out
