"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Routing indices, the permutation (offsets, permuted token list, inverse) are
compared bit for bit; router weights within a few fp32 ulp; the hidden
activations h and the output y within max-relative error 1e-2 (bf16
activations, fp32 accumulation) or 1e-4 (fp32 activations).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import pytest

from weight_only_quantized_warp_b200 import inputs as gen

from gpu_helpers import boundary_tokens, check_full, check_routing, check_sampled, run_gpu

pytestmark = pytest.mark.gpu


def _cfg(**kw):
    base = dict(T=24, H=320, I=192, E=8, k=2, bits=4, block_size=64, act=gen.ACT_SWIGLU, fusion=2,
                normalize=True, act_dtype=gen.DT_BF16, scale_dtype=gen.DT_BF16)
    base.update(kw)
    return gen.MoEConfig(**base)


def test_tiny_config_fp32(cuda_device):
    cfg, seed, kw = gen.tiny()
    inp = gen.make_inputs(cfg, seed, **kw)
    g = run_gpu(inp)
    assert g.path == 0
    check_full(inp, g)


# Small shapes that span several row tiles, k-groups and CTAs, with ragged
# tails (row tiles not a multiple of 8 warps; segments not a multiple of 8).
CASES = {
    "int4_bs64_fusion2": dict(),
    "int4_bs128_fusion1": dict(H=384, I=640, block_size=128, fusion=1),
    "int4_bs32_swiglu_clamp_bias": dict(block_size=32, fusion=1, alpha=1.702, beta=1.0, limit=7.0,
                                        has_fc1_bias=True, has_fc2_bias=True),
    "int4_bs16": dict(block_size=16),
    "int4_percol": dict(block_size=0),
    "int8_bs128": dict(H=384, I=640, bits=8, block_size=128),
    "int8_bs32": dict(bits=8, block_size=32),
    "int8_bs16": dict(bits=8, block_size=16),
    "int8_percol_fc3_silu_shared": dict(bits=8, block_size=0, fusion=0, has_fc3=True, act=gen.ACT_SILU,
                                        normalize=False, has_shared=True),
    "fc3_with_biases": dict(fusion=0, has_fc3=True, act=gen.ACT_SWIGLU, has_fc1_bias=True,
                            has_fc3_bias=True, has_fc2_bias=True),
    "plain_relu": dict(fusion=0, act=gen.ACT_RELU, has_fc1_bias=True),
    "plain_gelu": dict(fusion=0, act=gen.ACT_GELU),
    "plain_identity": dict(fusion=0, act=gen.ACT_IDENTITY),
    "gated_gelu": dict(fusion=1, act=gen.ACT_GELU),
    "f32_scales_bf16_acts_bs64": dict(scale_dtype=gen.DT_F32),
    "f32_scales_bf16_acts_bs16": dict(scale_dtype=gen.DT_F32, block_size=16),
    "f32_scales_int8_bs16": dict(scale_dtype=gen.DT_F32, bits=8, block_size=16),
    "many_tokens_several_passes": dict(T=200, E=4, k=2),
    "e64_k6": dict(T=40, E=64, k=6, bits=8, block_size=0, fusion=0, has_fc3=True,
                   act=gen.ACT_SILU, normalize=False),
    "k_equals_E": dict(T=9, E=4, k=4),
    "e256_k8": dict(T=20, E=256, k=8, H=128, I=128, block_size=64),
    "one_expert": dict(T=7, E=1, k=1, normalize=False),
    "t1": dict(T=1),
    # shapes the streaming tensor-core kernels take (H, I multiples of 128)
    "k128_int4_bs32_bias": dict(H=256, I=384, block_size=32, fusion=1, has_fc1_bias=True, has_fc2_bias=True),
    "k128_int4_bs16_f32scales": dict(H=256, I=384, block_size=16, scale_dtype=gen.DT_F32),
    "k128_int4_percol": dict(H=256, I=384, block_size=0),
    "k128_int8_bs64_fc3": dict(H=256, I=384, bits=8, block_size=64, fusion=0, has_fc3=True,
                               act=gen.ACT_SILU),
    "k128_int8_percol_relu": dict(H=256, I=384, bits=8, block_size=0, fusion=0, act=gen.ACT_RELU),
    "k128_t32_tile32": dict(H=256, I=384, T=96, E=8, k=2),
    # long K ranges: staged rows near the shared-memory target (fewer token
    # tiles per pass on the streaming path), several tiles and passes, and the
    # zero-point fold's per-column and per-chunk sums over thousands of k
    "long_k_int4_bs128": dict(T=60, E=4, k=2, H=2048, I=1152, block_size=128),
    "long_k_int4_bs32_f32scales": dict(T=60, E=4, k=2, H=2048, I=384, block_size=32,
                                       scale_dtype=gen.DT_F32, has_fc1_bias=True),
    "long_k_int8_percol": dict(T=28, E=4, k=2, H=4096, I=256, bits=8, block_size=0),
    "long_k_one_tile_fold_percol": dict(T=4, E=2, k=1, H=5120, I=256, block_size=0),
    "long_k_one_tile_fold_bs64": dict(T=4, E=2, k=1, H=5120, I=256, block_size=64, has_fc2_bias=True),
    # more than 128 rows per expert: 256-wide token tiles on the tensor-core path
    "wide_tile_int4_bs32_bias": dict(T=300, E=2, k=1, H=256, I=384, block_size=32, fusion=1, alpha=1.702,
                                     beta=1.0, limit=7.0, has_fc1_bias=True, has_fc2_bias=True),
    "wide_tile_int8_percol_fc3_shared": dict(T=520, E=4, k=2, H=256, I=384, bits=8, block_size=0, fusion=0,
                                             has_fc3=True, act=gen.ACT_SILU, normalize=False, has_shared=True),
    "wide_tile_int8_bs128": dict(T=300, E=2, k=1, H=256, I=384, bits=8, block_size=128),
    "wide_tile_int8_bs32_bias": dict(T=300, E=2, k=1, H=256, I=384, bits=8, block_size=32, fusion=1,
                                     has_fc1_bias=True, has_fc2_bias=True),
    "wide_tile_int8_bs16": dict(T=300, E=2, k=1, H=256, I=384, bits=8, block_size=16),
    "wide_tile_int4_bs16": dict(T=300, E=2, k=1, H=256, I=384, block_size=16),
    "wide_tile_int4_bs128_f32scales": dict(T=300, E=2, k=1, H=256, I=384, block_size=128, scale_dtype=gen.DT_F32),
    # routing options of the MoE page
    "grouped_topk": dict(T=40, E=16, k=4, n_group=4, topk_group=2),
    "grouped_topk_one_group_int8": dict(T=33, E=32, k=3, n_group=8, topk_group=1, bits=8, block_size=64),
    "routed_scale_shared": dict(routed_scaling_factor=2.5, has_shared=True, has_fc2_bias=True),
    "weight_on_input_int8_bias": dict(apply_router_weight_on_input=True, bits=8, block_size=32,
                                      has_fc1_bias=True, normalize=False),
    "wide_tile_weight_on_input": dict(T=300, E=2, k=1, H=256, I=384, apply_router_weight_on_input=True,
                                      normalize=False, routed_scaling_factor=0.5),
    "fp32_weight_on_input_scaled": dict(act_dtype=gen.DT_F32, scale_dtype=gen.DT_F32, apply_router_weight_on_input=True,
                                        routed_scaling_factor=0.75, normalize=False, block_size=32),
    # e_score_correction_bias (selection keys fp32(logit + bias)), expert_output_scale, tanh GELU
    "score_bias": dict(T=40, E=16, k=4, has_score_bias=True, normalize=False),
    "score_bias_grouped_eos": dict(T=40, E=16, k=4, n_group=4, topk_group=2, has_score_bias=True,
                                   expert_output_scale=1.75, has_fc2_bias=True),
    "score_bias_wide_tile": dict(T=300, E=2, k=1, H=256, I=384, has_score_bias=True),
    "gelu_tanh_plain_bias": dict(fusion=0, act=gen.ACT_GELU, gelu_mode=1, has_fc1_bias=True),
    "gelu_tanh_gated_int8": dict(fusion=1, act=gen.ACT_GELU, gelu_mode=1, bits=8, block_size=64),
    "gelu_tanh_wide_tile": dict(T=300, E=2, k=1, H=256, I=384, fusion=0, act=gen.ACT_GELU, gelu_mode=1),
    "gelu_tanh_fp32_eos": dict(act_dtype=gen.DT_F32, scale_dtype=gen.DT_F32, fusion=0, act=gen.ACT_GELU,
                               gelu_mode=1, expert_output_scale=0.25, has_shared=True),
    # MXFP4 expert weights (e2m1 codes, E8M0 scale per 32)
    "mxfp4_swiglu_bias": dict(weight_format=gen.WEIGHTS_MXFP4, block_size=32, scale_dtype=gen.DT_E8M0, fusion=1,
                              alpha=1.702, beta=1.0, limit=7.0, has_fc1_bias=True, has_fc2_bias=True),
    "mxfp4_k128": dict(weight_format=gen.WEIGHTS_MXFP4, block_size=32, scale_dtype=gen.DT_E8M0, H=256, I=384),
    "mxfp4_wide_tile": dict(weight_format=gen.WEIGHTS_MXFP4, block_size=32, scale_dtype=gen.DT_E8M0, T=300, E=2,
                            k=1, H=256, I=384),
    "mxfp4_fp32_acts": dict(weight_format=gen.WEIGHTS_MXFP4, block_size=32, scale_dtype=gen.DT_E8M0,
                            act_dtype=gen.DT_F32, has_shared=True),
    "fp32_acts_int8": dict(act_dtype=gen.DT_F32, scale_dtype=gen.DT_F32, bits=8, block_size=32,
                           has_fc1_bias=True, has_fc2_bias=True, has_shared=True),
    "fp32_acts_percol_fc3": dict(act_dtype=gen.DT_F32, scale_dtype=gen.DT_BF16, block_size=0,
                                 fusion=0, has_fc3=True, act=gen.ACT_SILU),
}


PATH_DECODE, PATH_TC, PATH_TC_DECODE = 1, 2, 3


@pytest.mark.parametrize("path", [PATH_DECODE, PATH_TC, PATH_TC_DECODE], ids=["decode", "tc", "tcdecode"])
@pytest.mark.parametrize("name", list(CASES))
def test_parity_small(cuda_device, name, path):
    cfg = _cfg(**CASES[name])
    if cfg.act_dtype == gen.DT_F32 and path != PATH_DECODE:
        pytest.skip("fp32 activations always take the fp32 path")
    inp = gen.make_inputs(cfg, seed=100 + list(CASES).index(name), bias_std=0.1)
    g = run_gpu(inp, path=path)
    if cfg.act_dtype == gen.DT_F32:
        assert g.path == 0
    elif path == PATH_TC_DECODE:
        assert g.path in (PATH_TC_DECODE, PATH_DECODE)
    else:
        assert g.path == path
    check_full(inp, g, name=f"{name}/path{g.path}")


# Every tensor-core kernel instantiation against the oracle: code width x
# scale mode x token tile (16..128 take the kernel with the decoded weights
# in tensor memory, 256 the one with them in shared memory), plus MXFP4.
# The average rows per expert (T * k / E, E = 4, k = 2) picks the tile; the
# segments vary around it, so several tiles and ragged tails occur.
TILE_T = {16: 20, 32: 40, 64: 80, 128: 160, 256: 300}
SCALE_MODES = {"bs16": 16, "bs32": 32, "bs64": 64, "bs128": 128, "percol": 0}


@pytest.mark.parametrize("tile", list(TILE_T))
@pytest.mark.parametrize("scales", list(SCALE_MODES) + ["mxfp4"])
@pytest.mark.parametrize("bits", [4, 8])
def test_tensor_core_instantiations(cuda_device, bits, scales, tile):
    if scales == "mxfp4" and bits == 8:
        pytest.skip("MXFP4 codes are 4-bit")
    kw = dict(T=TILE_T[tile], E=4, k=2, H=256, I=384, bits=bits, fusion=1, has_fc1_bias=True, has_fc2_bias=True)
    if scales == "mxfp4":
        kw.update(weight_format=gen.WEIGHTS_MXFP4, block_size=32, scale_dtype=gen.DT_E8M0)
    else:
        kw.update(block_size=SCALE_MODES[scales])
    cfg = _cfg(**kw)
    inp = gen.make_inputs(cfg, seed=300 + tile + 7 * bits + len(scales), bias_std=0.1)
    g = run_gpu(inp, path=PATH_TC)
    assert g.path == PATH_TC and g.tile == tile
    check_full(inp, g, name=f"tc_int{bits}_{scales}_tile{tile}")


def test_all_tokens_to_one_expert_and_empty_experts(cuda_device):
    cfg = _cfg(T=37, k=1)
    inp = gen.make_inputs(cfg, seed=5)
    lg = np.zeros((cfg.T, cfg.E), dtype=np.float32)
    lg[:, 5] = 3.0
    inp.logits = gen.f32_to_bf16_bits(lg)
    g = run_gpu(inp)
    assert g.offsets.tolist() == [0] * 6 + [37] * 3
    check_full(inp, g)


@pytest.mark.parametrize("groups", [(0, 0), (4, 2), (8, 3)], ids=["plain", "4g2", "8g3"])
def test_logit_ties_break_to_lowest_id(cuda_device, groups):
    cfg = _cfg(T=64, E=16, k=3, n_group=groups[0], topk_group=groups[1])
    inp = gen.make_inputs(cfg, seed=6)
    rng = np.random.default_rng(6)
    lg = rng.integers(-2, 3, size=(cfg.T, cfg.E)).astype(np.float32) * 0.25  # many exact ties
    inp.logits = gen.f32_to_bf16_bits(lg)
    g = run_gpu(inp)
    check_full(inp, g)


@pytest.mark.parametrize("groups", [(0, 0), (4, 2)], ids=["plain", "4g2"])
def test_nan_logits_select_real_experts(cuda_device, groups):
    """NaN logits read as -inf (the oracle's reading): indices stay in range
    and equal the oracle's; rows with a finite logit keep finite outputs."""
    cfg = _cfg(T=40, E=16, k=3, n_group=groups[0], topk_group=groups[1])
    inp = gen.make_inputs(cfg, seed=12)
    rng = np.random.default_rng(12)
    lg = rng.standard_normal((cfg.T, cfg.E)).astype(np.float32)
    lg[rng.random(lg.shape) < 0.3] = np.nan
    lg[0, :] = np.nan             # every logit NaN: weights NaN, indices 0, 1, 2
    lg[1, :] = np.nan
    lg[1, 7] = 1.0                # fewer finite logits than k
    inp.logits = gen.f32_to_bf16_bits(lg)
    g = run_gpu(inp)
    assert ((g.topk_idx >= 0) & (g.topk_idx < cfg.E)).all()
    assert g.topk_idx[0].tolist() == [0, 1, 2]
    check_routing(inp, g)
    import oracle
    from gpu_helpers import TOL_BF16, max_rel
    ref = oracle.forward(inp)["y"]
    assert np.isnan(g.y[0]).all() and np.isnan(ref[0]).all()
    err = max_rel(g.y[1:], ref[1:])
    assert err <= TOL_BF16, f"y max rel err {err:.3e}"


def test_zero_tokens_is_a_noop(cuda_device):
    import torch
    from weight_only_quantized_warp_b200 import qmoe
    cfg = _cfg(T=4)
    inp = gen.make_inputs(cfg, seed=7)
    m = qmoe.QMoE(cfg)
    m.set_weights_from(inp)
    y = torch.full((0, cfg.H), 1.0, dtype=torch.bfloat16, device="cuda")
    x = torch.empty((0, cfg.H), dtype=torch.bfloat16, device="cuda")
    lg = torch.empty((0, cfg.E), dtype=torch.bfloat16, device="cuda")
    m.forward(x, lg, out=y)
    torch.cuda.synchronize()


@pytest.mark.parametrize("path", [PATH_DECODE, PATH_TC, PATH_TC_DECODE], ids=["decode", "tc", "tcdecode"])
def test_repeated_forward_is_bitwise_deterministic(cuda_device, path):
    cfg = _cfg(T=50, bits=4, block_size=128, H=384, I=640)
    inp = gen.make_inputs(cfg, seed=8)
    a = run_gpu(inp, path=path)
    b = run_gpu(inp, repeat=3, path=path)
    np.testing.assert_array_equal(a.y, b.y)
    np.testing.assert_array_equal(a.hidden, b.hidden)


@pytest.mark.parametrize("name", ["mixtral_decode", "sweep_int8_T16"])
def test_dependent_launch_changes_nothing(cuda_device, name):
    """The weight-streaming kernels launched as programmatic dependents (the
    default) give bitwise the same output as plain stream-ordered launches."""
    import torch
    from weight_only_quantized_warp_b200 import qmoe
    cfg, seed, kw = gen.workload(name)
    inp = gen.make_inputs(cfg, seed, **kw)
    m = qmoe.QMoE(cfg, "cuda:0")
    m.set_weights_from(inp)
    x = qmoe.to_device(inp.x, "cuda:0")
    lg = qmoe.to_device(inp.logits, "cuda:0")
    outs = []
    for pdl in (1, 0, 1):
        qmoe.qmoe_set_option(m.handle, qmoe.QMOE_OPT_PDL, pdl)
        for _ in range(3):
            y = m.forward(x, lg)
        torch.cuda.synchronize()
        outs.append(y.clone())
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])


def test_rebind_replaces_the_pack(cuda_device):
    import torch
    from weight_only_quantized_warp_b200 import qmoe
    cfg = _cfg(T=8)
    a = gen.make_inputs(cfg, seed=9)
    b = gen.make_inputs(cfg, seed=10)
    b.x, b.logits = a.x, a.logits
    m = qmoe.QMoE(cfg)
    m.set_weights_from(a)
    m.set_weights_from(b)
    y = m.forward(qmoe.to_device(b.x, "cuda"), qmoe.to_device(b.logits, "cuda"))
    torch.cuda.synchronize()
    import oracle
    from gpu_helpers import max_rel, to_numpy
    assert max_rel(to_numpy(y), oracle.forward(b)["y"]) <= 1e-2


# ------------------------------------------------------------ full-size configs

def _full_size(inp, path, name, per_tile, extra, seed):
    """One full-size forward, then y and h on tokens at every expert segment's
    ends and token-tile boundaries (plus a few random ones) against the
    oracle, token by token."""
    cfg = inp.cfg
    g = run_gpu(inp, path=path)
    tokens = np.arange(cfg.T) if cfg.T <= 8 else boundary_tokens(g, cfg.k, per_tile, extra, seed)
    g = run_gpu(inp, path=path, hidden_tokens=tokens)
    check_sampled(inp, g, tokens, name=f"{name}/path{g.path}", hidden=True)


@pytest.mark.parametrize("path", [None, PATH_DECODE, PATH_TC, PATH_TC_DECODE], ids=["auto", "decode", "tc", "tcdecode"])
@pytest.mark.parametrize("name", ["mixtral_decode", "gpt_oss", "gpt_oss_mxfp4", "deepseek"])
def test_full_size_configs(cuda_device, name, path):
    cfg, seed, kw = gen.workload(name)
    inp = gen.make_inputs(cfg, seed, **kw)
    _full_size(inp, path, name, per_tile=1, extra=4, seed=seed)


# The prefill sweep at full size (H=4096, I=14336, E=8, k=2): every T of both
# code families on the kernels the planner picks, plus the opt-in streaming
# tensor-core path where it applies.
@pytest.mark.parametrize("path", [None, PATH_TC_DECODE], ids=["auto", "tcdecode"])
@pytest.mark.parametrize("bits,T", [(4, 1), (4, 16), (4, 128), (4, 1024), (4, 8192),
                                    (8, 1), (8, 16), (8, 128), (8, 1024), (8, 8192)])
def test_sweep_configs(cuda_device, bits, T, path):
    if path == PATH_TC_DECODE and T > 128:
        pytest.skip("the streaming tensor-core path takes at most 32 rows per expert")
    cfg, seed, kw = gen.sweep(bits, T)
    inp = gen.make_inputs(cfg, seed, **kw)
    _full_size(inp, path, f"sweep_int{bits}_T{T}", per_tile=1, extra=2, seed=seed)
