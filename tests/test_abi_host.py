"""Host-side checks of the C ABI: the library loads without a GPU, exports
every symbol that include/qmoe.h declares, and rejects bad configurations
and calls before touching the device."""
from __future__ import annotations

import ctypes
import math
import os
import re

import pytest

from weight_only_quantized_warp_b200 import build as libbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def q():
    libbuild.build()
    from weight_only_quantized_warp_b200 import qmoe
    return qmoe


def _declared():
    with open(os.path.join(ROOT, "include", "qmoe.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"QMOE_API\s+[\w\s\*]+?\b(qmoe_\w+)\s*\(", text)))


def test_header_declares_every_binding_name(q):
    assert _declared() == sorted(q.EXPORTS)


def test_library_exports_every_declared_symbol(q):
    lib = ctypes.CDLL(q.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name


def test_config_struct_layout(q):
    assert ctypes.sizeof(q.qmoe_config) == 128
    assert q.qmoe_config.expert_output_scale.offset == 120
    assert q.qmoe_config.gelu_mode.offset == 124
    assert q.qmoe_config.expert_weight_bits.offset == 32
    assert q.qmoe_config.activation_alpha.offset == 48
    assert q.qmoe_config.reserved.offset == 92
    assert q.qmoe_config.n_group.offset == 96
    assert q.qmoe_config.apply_router_weight_on_input.offset == 108
    assert q.qmoe_config.compute_mode.offset == 116


def _cfg(q, **kw):
    base = dict(num_experts=8, hidden_size=256, inter_size=512, k=2, expert_weight_bits=4,
                block_size=64, activation_type=q.ACT_SWIGLU, swiglu_fusion=2,
                activation_alpha=0.0, activation_beta=0.0, swiglu_limit=math.inf,
                normalize_routing_weights=1, act_dtype=q.DTYPE_BF16, scale_dtype=q.DTYPE_BF16)
    base.update(kw)
    return q.qmoe_config(**base)


BAD = [
    (dict(k=0), 1), (dict(k=9), 1), (dict(expert_weight_bits=3), 1), (dict(expert_weight_bits=0), 1),
    (dict(block_size=8), 1), (dict(block_size=48), 1), (dict(block_size=512), 1),
    (dict(activation_type=7), 1), (dict(swiglu_fusion=3), 1),
    (dict(swiglu_fusion=0, activation_type=3), 1),              # swiglu without a gate/up pair
    (dict(swiglu_fusion=1, has_fc3=1), 1),                      # fc3 only when unfused
    (dict(has_fc3_bias=1), 1),                                  # bias without its slot
    (dict(act_dtype=5), 1), (dict(scale_dtype=2), 1), (dict(reserved=1), 1),
    (dict(num_experts=0), 1), (dict(hidden_size=0), 1),
    (dict(use_sparse_mixer=1), 3),                              # valid per the page, not built
    (dict(num_experts=512, k=2), 3),
    (dict(hidden_size=96, block_size=32), 3),                   # not a multiple of 64
    (dict(n_group=3), 1),                                       # E = 8 not divisible by 3
    (dict(n_group=4, topk_group=0), 1), (dict(n_group=4, topk_group=5), 1),
    (dict(n_group=4, topk_group=1, k=3), 1),                    # k > topk_group * E / n_group
    (dict(num_experts=128, n_group=64, topk_group=1, k=1), 3),  # more than 32 groups: not built
    (dict(apply_router_weight_on_input=2), 1), (dict(routed_scaling_factor=-1.0), 1),
    (dict(weight_format=2), 1), (dict(compute_mode=2), 1), (dict(compute_mode=-1), 1),
    (dict(compute_mode=1, block_size=0), 1),                    # the int8 tier needs block scales
    (dict(compute_mode=1, weight_format=1, block_size=32, scale_dtype=2), 1),  # ... and integer codes
    (dict(compute_mode=1, block_size=32), 3),                   # 4-bit codes: blocks below 64 not built
    (dict(compute_mode=1, expert_weight_bits=8, block_size=16), 3),
    (dict(weight_format=1, block_size=32), 1),                  # MXFP4 needs E8M0 scales
    (dict(weight_format=1, block_size=64, scale_dtype=2), 1),   # ... and block_size 32
    (dict(weight_format=1, expert_weight_bits=8, block_size=32, scale_dtype=2), 1),
    (dict(scale_dtype=2), 1),                                   # E8M0 only with MXFP4
    (dict(expert_output_scale=-0.5), 1), (dict(expert_output_scale=math.inf), 1),
    (dict(gelu_mode=2), 1), (dict(gelu_mode=-1), 1),
]


@pytest.mark.parametrize("kw,status", BAD, ids=[str(i) for i in range(len(BAD))])
def test_create_rejects(q, kw, status):
    h = ctypes.c_void_p()
    assert q.lib.qmoe_create(ctypes.byref(_cfg(q, **kw)), ctypes.byref(h)) == status
    assert not h.value


def test_create_accepts_and_plans_without_gpu(q):
    h = q.qmoe_create(_cfg(q))
    try:
        assert q.qmoe_workspace_size(h, 0) > 0
        ws8 = q.qmoe_workspace_size(h, 8)
        assert ws8 > q.qmoe_workspace_size(h, 1) and ws8 % 256 == 0
        assert q.qmoe_workspace_size(h, -1) == 0
        assert q.qmoe_path_for(h, 8) == q.PATH_DECODE
        assert q.qmoe_launches_for(h, 8) == 4     # route+permute, FC1, FC2, combine
        assert q.qmoe_launches_for(h, 32) == 4
        assert q.qmoe_launches_for(h, 33) == 5    # tensor-core path: route+permute, gather, FC1, FC2, combine
        assert q.qmoe_launches_for(h, 64) == 5
        assert q.qmoe_launches_for(h, 65) == 6    # route, permute, gather, ...
        assert q.qmoe_launches_for(h, 0) == 0
        assert q.qmoe_token_tile_for(h, 8) == 0  # decode path: no token tile
        assert q.qmoe_token_tile_for(h, -1) == -1
    finally:
        q.qmoe_destroy(h)
    hf = q.qmoe_create(_cfg(q, act_dtype=q.DTYPE_F32, scale_dtype=q.DTYPE_F32))
    assert q.qmoe_path_for(hf, 8) == q.PATH_SIMT
    q.qmoe_destroy(hf)
    q.qmoe_destroy(None)  # no-op


@pytest.mark.parametrize("T,path,tile", [(8, 1, 0), (32, 1, 0), (33, 2, 16), (96, 2, 32), (128, 2, 64),
                                         (384, 2, 128), (2048, 2, 256)])
def test_plan_token_tile_covers_the_average_segment(q, T, path, tile):
    # 8 experts, k = 2: T*2/8 rows per expert on average; up to 8 the weights
    # stream (no token tile), above it the tile is the power of two covering
    # 4/3 of that, at most 256
    h = q.qmoe_create(_cfg(q))
    try:
        assert q.qmoe_path_for(h, T) == path
        assert q.qmoe_token_tile_for(h, T) == tile
    finally:
        q.qmoe_destroy(h)


def test_forward_before_set_weights_is_not_bound(q):
    h = q.qmoe_create(_cfg(q))
    try:
        st = q.lib.qmoe_forward(h, 4, 16, 16, None, 16, 256, 1 << 20, None)
        assert st == q.QMOE_NOT_BOUND
        assert b"set_weights" in q.lib.qmoe_last_error(h)
    finally:
        q.qmoe_destroy(h)


def test_set_weights_argument_errors_precede_device_work(q):
    h = q.qmoe_create(_cfg(q, has_fc1_bias=1))
    try:
        a = 256  # any non-null address; validation fails before it is used
        # missing required slot
        assert q.lib.qmoe_set_weights(h, None, a, a, a, a, None, None, None, None, None) == 1
        # declared fc1 bias missing
        assert q.lib.qmoe_set_weights(h, a, a, None, a, a, None, None, None, None, None) == 1
        # fc2 bias given without its declared slot
        assert q.lib.qmoe_set_weights(h, a, a, a, a, a, a, None, None, None, None) == 1
        # fc3 given without has_fc3
        assert q.lib.qmoe_set_weights(h, a, a, a, a, a, None, a, a, None, None) == 1
        # bf16 scales or bias on an odd address; codes may sit anywhere
        assert q.lib.qmoe_set_weights(h, a, a + 1, a, a, a, None, None, None, None, None) == 1
        assert b"scales" in q.lib.qmoe_last_error(h)
        assert q.lib.qmoe_set_weights(h, a, a, a + 1, a, a, None, None, None, None, None) == 1
        assert b"biases" in q.lib.qmoe_last_error(h)
        assert b"bias" in q.lib.qmoe_last_error(h) or b"fc3" in q.lib.qmoe_last_error(h)
    finally:
        q.qmoe_destroy(h)


def test_wait_limit_and_withhold_options_are_validated(q):
    h = q.qmoe_create(_cfg(q))
    try:
        for opt, val in [(q.QMOE_OPT_WAIT_LIMIT_NS, 99999), (q.QMOE_OPT_WAIT_LIMIT_NS, 61 * 10**9),
                         (q.QMOE_OPT_TEST_WITHHOLD, 2), (q.QMOE_OPT_TEST_WITHHOLD, -1), (99, 0),
                         (q.QMOE_OPT_DECODE_TILES, 3), (q.QMOE_OPT_DECODE_TILES, 8), (q.QMOE_OPT_DECODE_TILES, -1)]:
            assert q.lib.qmoe_set_option(h, opt, val) == q.QMOE_INVALID_ARGUMENT
        for opt, val in [(q.QMOE_OPT_WAIT_LIMIT_NS, 10**6), (q.QMOE_OPT_WAIT_LIMIT_NS, 2 * 10**9),
                         (q.QMOE_OPT_TEST_WITHHOLD, 1), (q.QMOE_OPT_TEST_WITHHOLD, 0),
                         (q.QMOE_OPT_DECODE_TILES, 4), (q.QMOE_OPT_DECODE_TILES, 0)]:
            assert q.lib.qmoe_set_option(h, opt, val) == q.QMOE_OK
    finally:
        q.qmoe_destroy(h)


def test_noalloc_status_before_any_noalloc_call(q):
    # no device is current here, or no no-alloc forward has run: never QMOE_OK
    h = q.qmoe_create(_cfg(q))
    try:
        assert q.lib.qmoe_noalloc_read_device_status(h, None) in (q.QMOE_INVALID_ARGUMENT, q.QMOE_CUDA_ERROR)
        assert q.lib.qmoe_noalloc_read_device_status(None, None) == q.QMOE_INVALID_ARGUMENT
    finally:
        q.qmoe_destroy(h)


def test_score_bias_setter_rejects_before_device_work(q):
    h = q.qmoe_create(_cfg(q))
    try:
        assert q.lib.qmoe_set_score_correction_bias(h, 258, None) == q.QMOE_INVALID_ARGUMENT  # misaligned
        assert q.lib.qmoe_set_score_correction_bias(h, None, None) == q.QMOE_OK              # clear: no-op
        assert q.lib.qmoe_set_score_correction_bias(None, None, None) == q.QMOE_INVALID_ARGUMENT
    finally:
        q.qmoe_destroy(h)


def test_status_strings(q):
    for s, name in [(0, b"QMOE_OK"), (1, b"QMOE_INVALID_ARGUMENT"), (2, b"QMOE_NOT_BOUND"),
                    (3, b"QMOE_UNSUPPORTED"), (4, b"QMOE_CUDA_ERROR"), (5, b"QMOE_TIMEOUT"),
                    (6, b"QMOE_OUT_OF_MEMORY")]:
        assert q.lib.qmoe_status_string(s) == name


def test_int8_tier_plan(q):
    # compute_mode INT8_BLOCK: the streaming kernel (path 4), and with K
    # blocks of 128 or more beyond 32 rows per expert the integer tensor-core
    # GEMM (path 5, with the row gather and a token tile of at most 64); the
    # two rounding launches added, and the code buffers in the workspace
    h = q.qmoe_create(_cfg(q, compute_mode=q.COMPUTE_INT8_BLOCK))
    h128 = q.qmoe_create(_cfg(q, compute_mode=q.COMPUTE_INT8_BLOCK, block_size=128))
    hf = q.qmoe_create(_cfg(q))
    ha = q.qmoe_create(_cfg(q, compute_mode=q.COMPUTE_INT8_BLOCK, apply_router_weight_on_input=1))
    try:
        for T in (1, 8, 64, 65, 4096):  # 64-code blocks: the streaming kernel
            assert q.qmoe_path_for(h, T) == q.PATH_INT8
            assert q.qmoe_token_tile_for(h, T) == 0
        for T in (8, 128):
            assert q.qmoe_path_for(h128, T) == q.PATH_INT8
        for T, tile in ((129, 64), (4096, 64)):
            assert q.qmoe_path_for(h128, T) == q.PATH_INT8_TC
            assert q.qmoe_token_tile_for(h128, T) == tile
        assert q.qmoe_launches_for(h, 8) == 6     # route+permute, quantize x, FC1, quantize h, FC2, combine
        assert q.qmoe_launches_for(h, 65) == 7    # routing and permutation apart
        assert q.qmoe_launches_for(h128, 129) == 8  # plus the row gather
        assert q.qmoe_launches_for(ha, 8) == 7    # plus the weighted row gather
        # codes and scales of x [T, H] and h [T*k, I] on top of the float plan
        T, H, I, k, bs = 8, 256, 512, 2, 64
        extra = T * H + T * (H // bs) * 4 + T * k * I + T * k * (I // bs) * 4
        assert q.qmoe_workspace_size(h, T) >= q.qmoe_workspace_size(hf, T) + extra
        q.qmoe_set_option(h, q.QMOE_OPT_PATH, 2)  # the tensor-core GEMM at any T
        assert q.qmoe_path_for(h, 8) == q.PATH_INT8_TC
        q.qmoe_set_option(h, q.QMOE_OPT_PATH, 1)  # the streaming kernel at any T
        assert q.qmoe_path_for(h, 4096) == q.PATH_INT8
        for v in (1, 3):  # 1 and 3 both keep the tier on the streaming kernel
            q.qmoe_set_option(h128, q.QMOE_OPT_PATH, v)
            assert q.qmoe_path_for(h128, 4096) == q.PATH_INT8
        q.qmoe_set_option(h128, q.QMOE_OPT_PATH, -1)
        assert q.qmoe_path_for(h128, 4096) == q.PATH_INT8_TC
    finally:
        q.qmoe_destroy(h)
        q.qmoe_destroy(h128)
        q.qmoe_destroy(hf)
        q.qmoe_destroy(ha)
    hs = q.qmoe_create(_cfg(q, compute_mode=q.COMPUTE_INT8_BLOCK, act_dtype=q.DTYPE_F32,
                            scale_dtype=q.DTYPE_F32))
    assert q.qmoe_path_for(hs, 8) == q.PATH_INT8  # fp32 activations take the tier too
    q.qmoe_destroy(hs)


@pytest.mark.parametrize("args", [
    (1, 64, 8),        # block_size below 16
    (1, 96, 64),       # K not a multiple of block_size
    (1, 64, 48),       # block_size not a power of two
    (-1, 64, 16),      # negative rows
    (1, 0, 16),        # empty rows
])
def test_quantize_entry_rejects_bad_sizes_without_device_work(q, args):
    rows, K, bs = args
    assert q.lib.qmoe_quantize_act_i8(256, q.DTYPE_BF16, rows, K, bs, 256, 256, None) == q.QMOE_INVALID_ARGUMENT


def test_quantize_entry_rejects_bad_dtype_alignment_and_null(q):
    assert q.lib.qmoe_quantize_act_i8(256, q.DTYPE_E8M0, 1, 64, 16, 256, 256, None) == q.QMOE_INVALID_ARGUMENT
    assert q.lib.qmoe_quantize_act_i8(264, q.DTYPE_BF16, 1, 64, 16, 256, 256, None) == q.QMOE_INVALID_ARGUMENT
    assert q.lib.qmoe_quantize_act_i8(256, q.DTYPE_BF16, 1, 64, 16, 258, 256, None) == q.QMOE_INVALID_ARGUMENT
    assert q.lib.qmoe_quantize_act_i8(None, q.DTYPE_BF16, 1, 64, 16, 256, 256, None) == q.QMOE_INVALID_ARGUMENT
    assert q.lib.qmoe_quantize_act_i8(None, q.DTYPE_BF16, 0, 64, 16, None, None, None) == q.QMOE_OK  # no rows


@pytest.mark.parametrize("kw,T,path", [
    (dict(), 8, 1), (dict(), 40, 2), (dict(), 65, 2), (dict(), 4096, 2),
    (dict(compute_mode=1), 8, 4), (dict(compute_mode=1), 300, 4), (dict(compute_mode=1, block_size=128), 300, 5),
    (dict(compute_mode=1, apply_router_weight_on_input=1), 8, 4),
    (dict(apply_router_weight_on_input=1), 8, 1),
    (dict(act_dtype=0, scale_dtype=0), 8, 0), (dict(act_dtype=0, scale_dtype=0), 100, 0),
])
def test_bench_launch_names_match_the_plan(q, kw, T, path):
    # the benchmark's per-kernel labels follow the library's own launch count
    import bench
    h = q.qmoe_create(_cfg(q, **kw))
    try:
        assert q.qmoe_path_for(h, T) == path
        n = q.qmoe_launches_for(h, T)
        names = bench.launch_names(path, n, bool(kw.get("apply_router_weight_on_input")))
        assert len(names) == n
        assert names[-1] == "combine" and names.index("fc1") < names.index("fc2")
        assert ("route_permute" in names) == (T <= 64)
        assert ("quantize_x" in names) == (path in (q.PATH_INT8, q.PATH_INT8_TC))
        assert ("gather" in names) == (path in (q.PATH_TC, q.PATH_TC_DECODE, q.PATH_INT8_TC) or
                                       bool(kw.get("apply_router_weight_on_input")))
    finally:
        q.qmoe_destroy(h)
    with pytest.raises(ValueError):
        bench.launch_names(path, 99, False)


@pytest.mark.parametrize("x,lg,sh,y,ws,status", [
    (16, 16, None, 16, 256, 2),       # well-formed: the binding is checked next
    (24, 16, None, 16, 256, 1),       # x not 16-byte aligned
    (16, 16, 40, 16, 256, 1),         # shared_output not 16-byte aligned
    (16, 16, None, 8, 256, 1),        # y not 16-byte aligned
    (16, 17, None, 16, 256, 1),       # bf16 logits on an odd address
    (16, 16, None, 16, 128, 1),       # workspace not 256-byte aligned
    (None, 16, None, 16, 256, 1),     # x missing
])
def test_forward_argument_checks_precede_the_binding(q, x, lg, sh, y, ws, status):
    h = q.qmoe_create(_cfg(q))
    try:
        assert q.lib.qmoe_forward(h, 4, x, lg, sh, y, ws, 1 << 20, None) == status
        assert q.lib.qmoe_forward(h, -1, x, lg, sh, y, ws, 1 << 20, None) == q.QMOE_INVALID_ARGUMENT
    finally:
        q.qmoe_destroy(h)
