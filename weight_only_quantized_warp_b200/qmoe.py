"""ctypes binding of ``libqmoe.so`` (declared in ``include/qmoe.h``).

Argument marshalling only: every step of the forward runs in the library's
CUDA kernels. The names mirror the C ABI (``qmoe_create``,
``qmoe_set_weights``, ``qmoe_workspace_size``, ``qmoe_forward``, ...); the
``QMoE`` class strings them together for PyTorch tensors, which serve as
device memory and streams. Importing this module raises ``ImportError`` when
the library has not been built: there is no fallback.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
# QMOE_LIB may point at another build of the same library (same ABI).
LIB_PATH = os.environ.get("QMOE_LIB") or os.path.join(HERE, "libqmoe.so")

if not os.path.exists(LIB_PATH):
    raise ImportError("libqmoe.so is not built (run weight_only_quantized_warp_b200/build.py or "
                      "__graft_entry__.build()); the QMoE forward has no other implementation")

lib = ctypes.CDLL(LIB_PATH)

QMOE_OK, QMOE_INVALID_ARGUMENT, QMOE_NOT_BOUND, QMOE_UNSUPPORTED = 0, 1, 2, 3
QMOE_CUDA_ERROR, QMOE_TIMEOUT, QMOE_OUT_OF_MEMORY = 4, 5, 6
ACT_RELU, ACT_GELU, ACT_SILU, ACT_SWIGLU, ACT_IDENTITY = 0, 1, 2, 3, 4
DTYPE_F32, DTYPE_BF16, DTYPE_E8M0 = 0, 1, 2
WEIGHTS_INT, WEIGHTS_MXFP4 = 0, 1
COMPUTE_FLOAT, COMPUTE_INT8_BLOCK = 0, 1
GELU_ERF, GELU_TANH = 0, 1
PATH_SIMT, PATH_DECODE, PATH_TC, PATH_TC_DECODE, PATH_INT8, PATH_INT8_TC = 0, 1, 2, 3, 4, 5

# Every function the header declares (checked against include/qmoe.h by the tests).
EXPORTS = ("qmoe_create", "qmoe_set_weights", "qmoe_workspace_size", "qmoe_forward",
           "qmoe_forward_profiled",
           "qmoe_debug_routing", "qmoe_debug_hidden", "qmoe_read_device_status", "qmoe_destroy",
           "qmoe_status_string", "qmoe_last_error", "qmoe_path_for", "qmoe_launches_for",
           "qmoe_token_tile_for",
           "qmoe_set_option", "qmoe_forward_noalloc", "qmoe_noalloc_scratch_bytes",
           "qmoe_noalloc_read_device_status", "qmoe_set_score_correction_bias",
           "qmoe_quantize_act_i8", "qmoe_ep_state_bytes", "qmoe_ep_dispatch",
           "qmoe_ep_rows_workspace_size", "qmoe_ep_expert_rows", "qmoe_ep_combine")
QMOE_OPT_PATH, QMOE_OPT_WAIT_LIMIT_NS, QMOE_OPT_TEST_WITHHOLD, QMOE_OPT_PDL, QMOE_OPT_DECODE_TILES = 1, 2, 3, 4, 5


class qmoe_config(ctypes.Structure):
    _fields_ = [("num_experts", ctypes.c_int64), ("hidden_size", ctypes.c_int64),
                ("inter_size", ctypes.c_int64), ("k", ctypes.c_int64),
                ("expert_weight_bits", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("activation_type", ctypes.c_int32), ("swiglu_fusion", ctypes.c_int32),
                ("activation_alpha", ctypes.c_float), ("activation_beta", ctypes.c_float),
                ("swiglu_limit", ctypes.c_float), ("normalize_routing_weights", ctypes.c_int32),
                ("act_dtype", ctypes.c_int32), ("scale_dtype", ctypes.c_int32),
                ("has_fc1_bias", ctypes.c_int32), ("has_fc2_bias", ctypes.c_int32),
                ("has_fc3", ctypes.c_int32), ("has_fc3_bias", ctypes.c_int32),
                ("use_sparse_mixer", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("n_group", ctypes.c_int32), ("topk_group", ctypes.c_int32),
                ("routed_scaling_factor", ctypes.c_float), ("apply_router_weight_on_input", ctypes.c_int32),
                ("weight_format", ctypes.c_int32), ("compute_mode", ctypes.c_int32),
                ("expert_output_scale", ctypes.c_float), ("gelu_mode", ctypes.c_int32)]


_vp, _i64, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
lib.qmoe_create.restype = ctypes.c_int
lib.qmoe_create.argtypes = [ctypes.POINTER(qmoe_config), ctypes.POINTER(_vp)]
lib.qmoe_set_weights.restype = ctypes.c_int
lib.qmoe_set_weights.argtypes = [_vp] * 11
lib.qmoe_workspace_size.restype = _sz
lib.qmoe_workspace_size.argtypes = [_vp, _i64]
lib.qmoe_forward.restype = ctypes.c_int
lib.qmoe_forward.argtypes = [_vp, _i64, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
lib.qmoe_forward_profiled.restype = ctypes.c_int
lib.qmoe_forward_profiled.argtypes = [_vp, _i64, _vp, _vp, _vp, _vp, _vp, _sz, _vp,
                                      ctypes.POINTER(_vp), ctypes.c_int32]
lib.qmoe_debug_routing.restype = ctypes.c_int
lib.qmoe_debug_routing.argtypes = [_vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
lib.qmoe_debug_hidden.restype = ctypes.c_int
lib.qmoe_debug_hidden.argtypes = [_vp, _i64, _vp, _vp, _vp]
lib.qmoe_read_device_status.restype = ctypes.c_int
lib.qmoe_read_device_status.argtypes = [_vp, _vp, _vp]
lib.qmoe_destroy.restype = None
lib.qmoe_destroy.argtypes = [_vp]
lib.qmoe_status_string.restype = ctypes.c_char_p
lib.qmoe_status_string.argtypes = [ctypes.c_int]
lib.qmoe_last_error.restype = ctypes.c_char_p
lib.qmoe_last_error.argtypes = [_vp]
lib.qmoe_path_for.restype = ctypes.c_int32
lib.qmoe_path_for.argtypes = [_vp, _i64]
lib.qmoe_forward_noalloc.restype = ctypes.c_int
lib.qmoe_forward_noalloc.argtypes = [_vp, _i64, _vp, _vp, _vp, _vp, _vp]
lib.qmoe_noalloc_scratch_bytes.restype = _sz
lib.qmoe_noalloc_scratch_bytes.argtypes = []
lib.qmoe_noalloc_read_device_status.restype = ctypes.c_int
lib.qmoe_noalloc_read_device_status.argtypes = [_vp, _vp]
lib.qmoe_set_score_correction_bias.restype = ctypes.c_int
lib.qmoe_set_score_correction_bias.argtypes = [_vp, _vp, _vp]
lib.qmoe_set_option.restype = ctypes.c_int
lib.qmoe_set_option.argtypes = [_vp, ctypes.c_int32, _i64]
lib.qmoe_launches_for.restype = ctypes.c_int32
lib.qmoe_launches_for.argtypes = [_vp, _i64]
lib.qmoe_token_tile_for.restype = ctypes.c_int32
lib.qmoe_token_tile_for.argtypes = [_vp, _i64]
lib.qmoe_quantize_act_i8.restype = ctypes.c_int
lib.qmoe_quantize_act_i8.argtypes = [_vp, ctypes.c_int32, _i64, _i64, ctypes.c_int32, _vp, _vp, _vp]
lib.qmoe_ep_state_bytes.restype = _sz
lib.qmoe_ep_state_bytes.argtypes = [_vp, _i64]
lib.qmoe_ep_dispatch.restype = ctypes.c_int
lib.qmoe_ep_dispatch.argtypes = [_vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
lib.qmoe_ep_rows_workspace_size.restype = _sz
lib.qmoe_ep_rows_workspace_size.argtypes = [_vp, _i64]
lib.qmoe_ep_expert_rows.restype = ctypes.c_int
lib.qmoe_ep_expert_rows.argtypes = [_vp, _i64, _vp, _vp, ctypes.c_int32, _vp, _vp, _sz, _vp]
lib.qmoe_ep_combine.restype = ctypes.c_int
lib.qmoe_ep_combine.argtypes = [_vp, _i64, _vp, _vp, _vp, _vp, _vp]


class QMoEError(RuntimeError):
    def __init__(self, status: int, message: str = ""):
        self.status = status
        name = lib.qmoe_status_string(status).decode()
        super().__init__(f"{name}: {message}" if message else name)


def _ptr(t) -> Optional[int]:
    """Device address of a tensor (or an int address); None passes NULL."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("tensors passed to the QMoE ABI must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, handle=None):
    if status != QMOE_OK:
        msg = lib.qmoe_last_error(handle).decode() if handle else ""
        raise QMoEError(status, msg)


# ------------------------------------------------------------- the C ABI names

def make_config(cfg) -> qmoe_config:
    """A ``qmoe_config`` from an object with the fields of ``inputs.MoEConfig``."""
    lim = cfg.limit if cfg.limit is not None else math.inf
    return qmoe_config(
        num_experts=cfg.E, hidden_size=cfg.H, inter_size=cfg.I, k=cfg.k,
        expert_weight_bits=cfg.bits, block_size=cfg.block_size, activation_type=cfg.act,
        swiglu_fusion=cfg.fusion, activation_alpha=cfg.alpha, activation_beta=cfg.beta,
        swiglu_limit=lim, normalize_routing_weights=int(cfg.normalize), act_dtype=cfg.act_dtype,
        scale_dtype=cfg.scale_dtype, has_fc1_bias=int(cfg.has_fc1_bias),
        has_fc2_bias=int(cfg.has_fc2_bias), has_fc3=int(cfg.has_fc3),
        has_fc3_bias=int(cfg.has_fc3_bias), use_sparse_mixer=0, reserved=0,
        n_group=int(getattr(cfg, "n_group", 0)), topk_group=int(getattr(cfg, "topk_group", 0)),
        routed_scaling_factor=float(getattr(cfg, "routed_scaling_factor", 1.0)),
        apply_router_weight_on_input=int(getattr(cfg, "apply_router_weight_on_input", False)),
        weight_format=int(getattr(cfg, "weight_format", 0)),
        compute_mode=int(getattr(cfg, "compute_mode", 0)),
        expert_output_scale=float(getattr(cfg, "expert_output_scale", 1.0)),
        gelu_mode=int(getattr(cfg, "gelu_mode", 0)))


def qmoe_create(cfg: qmoe_config) -> int:
    h = _vp()
    _check(lib.qmoe_create(ctypes.byref(cfg), ctypes.byref(h)))
    return h.value


def qmoe_set_weights(h, fc1_w, fc1_s, fc1_b, fc2_w, fc2_s, fc2_b, fc3_w=None, fc3_s=None,
                     fc3_b=None, stream=None):
    _check(lib.qmoe_set_weights(h, _ptr(fc1_w), _ptr(fc1_s), _ptr(fc1_b), _ptr(fc2_w), _ptr(fc2_s),
                                _ptr(fc2_b), _ptr(fc3_w), _ptr(fc3_s), _ptr(fc3_b), _stream(stream)), h)


def qmoe_set_score_correction_bias(h, bias, stream=None):
    """Bind the e_score_correction_bias ([E] fp32 device tensor, or None to
    clear); it moves the expert selection only."""
    _check(lib.qmoe_set_score_correction_bias(h, _ptr(bias), _stream(stream)), h)


def qmoe_workspace_size(h, T: int) -> int:
    return int(lib.qmoe_workspace_size(h, T))


def qmoe_forward(h, T, x, router_logits, shared_output, y, workspace, workspace_bytes, stream=None):
    _check(lib.qmoe_forward(h, T, _ptr(x), _ptr(router_logits), _ptr(shared_output), _ptr(y),
                            _ptr(workspace), workspace_bytes, _stream(stream)), h)


def qmoe_forward_noalloc(h, T, x, router_logits, shared_output, y, stream=None):
    """The forward with its scratch in the library's fixed device array (no
    workspace argument, nothing allocated); see include/qmoe.h."""
    _check(lib.qmoe_forward_noalloc(h, T, _ptr(x), _ptr(router_logits), _ptr(shared_output), _ptr(y),
                                    _stream(stream)), h)


def qmoe_noalloc_scratch_bytes() -> int:
    return int(lib.qmoe_noalloc_scratch_bytes())


def qmoe_noalloc_read_device_status(h, stream=None) -> int:
    """Device status word of the last no-alloc forward on the current device."""
    return int(lib.qmoe_noalloc_read_device_status(h, _stream(stream)))


def qmoe_forward_profiled(h, T, x, router_logits, shared_output, y, workspace, workspace_bytes,
                          events, stream=None):
    """``events``: torch.cuda.Event objects (timing enabled, already created by
    one record), ``qmoe_launches_for(h, T) + 1`` of them."""
    arr = (_vp * len(events))(*[e.cuda_event for e in events])
    _check(lib.qmoe_forward_profiled(h, T, _ptr(x), _ptr(router_logits), _ptr(shared_output), _ptr(y),
                                     _ptr(workspace), workspace_bytes, _stream(stream), arr,
                                     len(events)), h)


def qmoe_debug_routing(h, T, workspace, topk_idx=None, topk_w=None, offsets=None, perm_tok=None,
                       inv=None, stream=None):
    _check(lib.qmoe_debug_routing(h, T, _ptr(workspace), _ptr(topk_idx), _ptr(topk_w), _ptr(offsets),
                                  _ptr(perm_tok), _ptr(inv), _stream(stream)), h)


def qmoe_debug_hidden(h, T, workspace, hidden, stream=None):
    _check(lib.qmoe_debug_hidden(h, T, _ptr(workspace), _ptr(hidden), _stream(stream)), h)


def qmoe_read_device_status(h, workspace, stream=None) -> int:
    return int(lib.qmoe_read_device_status(h, _ptr(workspace), _stream(stream)))


def qmoe_destroy(h):
    lib.qmoe_destroy(h)


def qmoe_path_for(h, T: int) -> int:
    return int(lib.qmoe_path_for(h, T))


def qmoe_set_option(h, option: int, value: int):
    _check(lib.qmoe_set_option(h, option, value), h)


def qmoe_launches_for(h, T: int) -> int:
    return int(lib.qmoe_launches_for(h, T))


def qmoe_token_tile_for(h, T: int) -> int:
    return int(lib.qmoe_token_tile_for(h, T))


def qmoe_quantize_act_i8(x, dtype: int, rows: int, K: int, block_size: int, q, scales, stream=None):
    """Int8 block tier rounding of activation rows x [rows, K] into codes q
    [rows, K] int8 and scales [rows, K / block_size] fp32 (device buffers)."""
    _check(lib.qmoe_quantize_act_i8(_ptr(x), dtype, rows, K, block_size, _ptr(q), _ptr(scales),
                                    _stream(stream)))


def qmoe_ep_state_bytes(h, T: int) -> int:
    return int(lib.qmoe_ep_state_bytes(h, T))


def qmoe_ep_dispatch(h, T, x, router_logits, rows, row_expert, offsets, state, state_bytes, stream=None):
    """Expert parallel, token owner: route, sort the routes by expert, gather
    x's rows in that order (see include/qmoe.h)."""
    _check(lib.qmoe_ep_dispatch(h, T, _ptr(x), _ptr(router_logits), _ptr(rows), _ptr(row_expert),
                                _ptr(offsets), _ptr(state), state_bytes, _stream(stream)), h)


def qmoe_ep_rows_workspace_size(h, R: int) -> int:
    return int(lib.qmoe_ep_rows_workspace_size(h, R))


def qmoe_ep_expert_rows(h, R, rows, row_expert, expert_base, out, workspace, workspace_bytes, stream=None):
    """Expert parallel, expert owner: each row's expert output (o + fc2 bias,
    fp32) for global expert ids expert_base .. expert_base + E_h - 1."""
    _check(lib.qmoe_ep_expert_rows(h, R, _ptr(rows), _ptr(row_expert), int(expert_base), _ptr(out),
                                   _ptr(workspace), workspace_bytes, _stream(stream)), h)


def qmoe_ep_combine(h, T, expert_out, state, shared_output, y, stream=None):
    """Expert parallel, token owner: the router-weighted combine of the expert
    outputs that came back in dispatch order."""
    _check(lib.qmoe_ep_combine(h, T, _ptr(expert_out), _ptr(state), _ptr(shared_output), _ptr(y),
                               _stream(stream)), h)


# ------------------------------------------------------------- torch plumbing

def to_device(a, device):
    """Upload a numpy array (bf16 carried as uint16 bits) to a torch tensor."""
    import numpy as np
    import torch
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(a).to(device)


class QMoE:
    """One QMoE operator instance on one GPU (marshalling around the C ABI)."""

    def __init__(self, cfg, device=None, path=None):
        import torch
        self.cfg = cfg
        self.device = torch.device(device or "cuda")
        self.handle = qmoe_create(make_config(cfg))
        self._ws = None
        if path is not None:
            qmoe_set_option(self.handle, QMOE_OPT_PATH, path)

    def __del__(self):
        h = getattr(self, "handle", None)
        if h and lib is not None:
            lib.qmoe_destroy(h)
            self.handle = None

    def set_weights(self, fc1_w, fc1_s, fc2_w, fc2_s, fc1_b=None, fc2_b=None, fc3_w=None, fc3_s=None,
                    fc3_b=None, stream=None):
        qmoe_set_weights(self.handle, fc1_w, fc1_s, fc1_b, fc2_w, fc2_s, fc2_b, fc3_w, fc3_s, fc3_b,
                         stream)

    def set_weights_from(self, inp, stream=None):
        """Upload a generated input set's weights and bind them."""
        d = self.device
        t = {n: to_device(getattr(inp, n), d) for n in
             ("fc1_w", "fc1_s", "fc1_b", "fc2_w", "fc2_s", "fc2_b", "fc3_w", "fc3_s", "fc3_b")}
        self.set_weights(t["fc1_w"], t["fc1_s"], t["fc2_w"], t["fc2_s"], t["fc1_b"], t["fc2_b"],
                         t["fc3_w"], t["fc3_s"], t["fc3_b"], stream)
        sb = getattr(inp, "score_bias", None)
        qmoe_set_score_correction_bias(self.handle, to_device(sb, d) if sb is not None else None, stream)

    def workspace(self, T: int):
        import torch
        n = qmoe_workspace_size(self.handle, T)
        if self._ws is None or self._ws.numel() < n:
            self._ws = torch.empty(max(n, 256), dtype=torch.uint8, device=self.device)
        return self._ws

    def forward(self, x, router_logits, shared_output=None, out=None, stream=None):
        import torch
        T = x.shape[0]
        if out is None:
            out = torch.empty_like(x)
        ws = self.workspace(T)
        qmoe_forward(self.handle, T, x, router_logits, shared_output, out, ws, ws.numel(), stream)
        return out

    __call__ = forward
