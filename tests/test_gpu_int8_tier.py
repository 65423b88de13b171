"""GPU parity of the int8 block compute tier (compute_mode INT8_BLOCK: the
streaming integer kernel, path 4, and the integer tensor-core GEMM, path 5)
against the oracle.

The activation rounding is compared bit for bit: codes and fp32 scales of
the standalone entry qmoe_quantize_act_i8 equal the oracle's on the same
rows (both decide in fp32: s = absmax / 127 with an IEEE division, then
rint(v / s) with ties to even), including ties, all-zero blocks and rows, and
tiny magnitudes whose scale is an fp32 subnormal.

The forward is compared like the float tier: routing bit for bit, h within
1e-2 (bf16) or 1e-4 (fp32) of the oracle -- FC1's codes are the same on both
sides, so h differs only by fp32 accumulation -- and y within 1e-2 for both
activation dtypes. The looser y bound for fp32 comes from the arithmetic: FC2
rounds h to int8, and where the kernel's fp32 h and the oracle's exact h fall
on the two sides of a rounding boundary (a few per ten thousand codes when
h differs by ~1e-6 relative) the code moves by one step, which moves an output
by up to s_h * |s_w| * 2^(bits-1), about 1e-3 of it.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from weight_only_quantized_warp_b200 import inputs as gen

from gpu_helpers import TOL_BF16, TOL_F32, check_routing, check_sampled, max_rel, run_gpu

pytestmark = pytest.mark.gpu

PATH_INT8, PATH_INT8_TC = 4, 5
TOL_Y = 1e-2


def _expected_path(cfg, forced=None):
    """The tier's kernel: the tensor-core GEMM for bf16 activations (blocks
    of at least 32 codes) when forced, and by shape with blocks of 128 or more
    beyond 32 rows per expert; the streaming kernel otherwise."""
    tc_ok = cfg.act_dtype == gen.DT_BF16 and cfg.block_size >= 32
    per_expert = -(-max(cfg.T * cfg.k, 1) // cfg.E)
    if forced == 1:
        return PATH_INT8
    if forced == 2:
        return PATH_INT8_TC if tc_ok else PATH_INT8
    return PATH_INT8_TC if tc_ok and per_expert > 32 and cfg.block_size >= 128 else PATH_INT8


def _quant_rows(rng, rows, K, bs, bf16):
    x = (rng.standard_normal((rows, K)) * np.exp(rng.uniform(-4, 4, size=(rows, 1)))).astype(np.float32)
    x[1] = 0.0                                    # an all-zero row
    if K >= 2 * bs:
        x[2, bs:2 * bs] = 0.0                     # an all-zero block
    # ties: v = (m + 1/2) 2^-e with +-127 2^-e in the block, so v / s = m + 1/2 exactly
    m = rng.integers(-126, 126, size=K)
    e = 5
    x[3] = (m + 0.5) * 2.0 ** -e
    x[3, ::bs] = 127 * 2.0 ** -e
    # a tiny row: its scales are fp32 subnormals
    x[4] = x[0] * 1e-37 / np.abs(x[0]).max()
    if bf16:
        return gen.f32_to_bf16_bits(x)
    return x


@pytest.mark.parametrize("dtype", [gen.DT_BF16, gen.DT_F32], ids=["bf16", "f32"])
@pytest.mark.parametrize("K,bs", [(64, 16), (192, 32), (320, 64), (384, 128), (1024, 256), (4096, 1024),
                                  (4096, 4096)])
def test_quantize_entry_is_bit_exact(cuda_device, dtype, K, bs):
    import torch
    from weight_only_quantized_warp_b200 import qmoe
    rng = np.random.default_rng(K + bs)
    rows = 37
    x = _quant_rows(rng, rows, K, bs, dtype == gen.DT_BF16)
    xd = qmoe.to_device(x, "cuda:0")
    q = torch.full((rows, K), 99, dtype=torch.int8, device="cuda:0")
    s = torch.full((rows, K // bs), -1.0, dtype=torch.float32, device="cuda:0")
    qmoe.qmoe_quantize_act_i8(xd, dtype, rows, K, bs, q, s)
    torch.cuda.synchronize()
    qr, sr = oracle.quantize_i8(x, bs)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), sr.view(np.uint32))
    np.testing.assert_array_equal(q.cpu().numpy(), qr)
    ties = np.ones(K, dtype=bool)
    ties[::bs] = False
    assert np.all(qr[3][ties] % 2 == 0)  # every tie went to the even code


def test_quantize_entry_zero_rows_is_a_noop(cuda_device):
    import torch
    from weight_only_quantized_warp_b200 import qmoe
    q = torch.full((1, 64), 7, dtype=torch.int8, device="cuda:0")
    qmoe.qmoe_quantize_act_i8(None, gen.DT_BF16, 0, 64, 16, q, None)
    torch.cuda.synchronize()
    assert int(q.min()) == 7 and int(q.max()) == 7


def _cfg(**kw):
    base = dict(T=24, H=320, I=192, E=8, k=2, bits=4, block_size=64, act=gen.ACT_SWIGLU, fusion=2,
                normalize=True, act_dtype=gen.DT_BF16, scale_dtype=gen.DT_BF16,
                compute_mode=gen.COMPUTE_INT8_BLOCK)
    base.update(kw)
    return gen.MoEConfig(**base)


def _check(inp, g, forced=None):
    c = inp.cfg
    assert g.path == _expected_path(c, forced)
    check_routing(inp, g)
    ref = oracle.forward(inp, want_h=True)
    err = max_rel(g.y, ref["y"])
    assert err <= TOL_Y, f"y max rel err {err:.3e} > {TOL_Y}"
    if c.T > 0:
        tol_h = TOL_BF16 if c.act_dtype == gen.DT_BF16 else TOL_F32
        herr = max_rel(g.hidden[g.inv.reshape(-1)], ref["h"])
        assert herr <= tol_h, f"h max rel err {herr:.3e} > {tol_h}"
    return err


# Shapes spanning several row tiles, k-groups, scale chunks (P = 1, 2, 4, 8,
# and blocks longer than a chunk), CTAs and K-splits, with ragged tails.
CASES = {
    "int4_bs64_fusion2": dict(),
    "int4_bs128_fusion1_clamp_bias": dict(H=384, I=640, block_size=128, fusion=1, alpha=1.702, beta=1.0,
                                          limit=7.0, has_fc1_bias=True, has_fc2_bias=True),
    "int4_bs256": dict(H=512, I=768, block_size=256),
    "int4_bs1024_long_blocks": dict(H=2048, I=1024, block_size=1024),
    "int8_bs32": dict(bits=8, block_size=32),
    "int8_bs128": dict(H=384, I=640, bits=8, block_size=128),
    "int8_bs512_long_blocks": dict(H=1024, I=512, bits=8, block_size=512),
    "int8_fc3_silu_shared": dict(bits=8, fusion=0, has_fc3=True, act=gen.ACT_SILU, normalize=False,
                                 has_shared=True),
    "fc3_with_biases": dict(fusion=0, has_fc3=True, has_fc1_bias=True, has_fc3_bias=True, has_fc2_bias=True),
    "plain_relu": dict(fusion=0, act=gen.ACT_RELU, has_fc1_bias=True),
    "plain_identity_int8": dict(fusion=0, act=gen.ACT_IDENTITY, bits=8),
    "f32_scales": dict(scale_dtype=gen.DT_F32),
    "f32_acts_int4": dict(act_dtype=gen.DT_F32, scale_dtype=gen.DT_F32),
    "f32_acts_int8_bs32": dict(act_dtype=gen.DT_F32, scale_dtype=gen.DT_F32, bits=8, block_size=32),
    "f32_acts_bf16_scales": dict(act_dtype=gen.DT_F32),
    "weight_on_input": dict(apply_router_weight_on_input=True, normalize=False),
    "weight_on_input_f32": dict(apply_router_weight_on_input=True, act_dtype=gen.DT_F32,
                                scale_dtype=gen.DT_F32),
    "grouped_scaled": dict(E=16, k=4, n_group=4, topk_group=2, routed_scaling_factor=2.5),
    "one_token": dict(T=1),
    "five_tokens": dict(T=5),
    "two_tiles_per_expert": dict(T=40),
    "four_tiles_two_passes": dict(T=150),
    "unfused_routing": dict(T=300, E=4),
    "score_bias_gelu_tanh_eos": dict(fusion=1, act=gen.ACT_GELU, gelu_mode=1, has_score_bias=True,
                                     expert_output_scale=0.5, E=16, k=3),
}


@pytest.mark.parametrize("path", [None, 1, 2], ids=["auto", "stream", "tc"])
@pytest.mark.parametrize("name", list(CASES))
def test_int8_tier_parity_small(cuda_device, name, path):
    cfg = _cfg(**CASES[name])
    if path is not None and _expected_path(cfg, path) == _expected_path(cfg):
        pytest.skip("the forced kernel is the one chosen by shape")
    inp = gen.make_inputs(cfg, seed=300 + list(CASES).index(name), bias_std=0.1)
    _check(inp, run_gpu(inp, path=path), forced=path)


def test_int8_tier_zero_rows_and_blocks(cuda_device):
    # tokens whose activations are all zero, and zero blocks, give s = 0, q = 0
    cfg = _cfg(T=16, H=384, I=256, block_size=128, has_fc1_bias=True, has_fc2_bias=True)
    inp = gen.make_inputs(cfg, seed=350, bias_std=0.1)
    x = gen.bf16_bits_to_f32(inp.x).copy()
    x[3] = 0.0
    x[7, 128:256] = 0.0
    inp.x = gen.f32_to_bf16_bits(x)
    _check(inp, run_gpu(inp))


def test_int8_tier_all_tokens_to_one_expert(cuda_device):
    cfg = _cfg(T=40, k=1, E=6)
    inp = gen.make_inputs(cfg, seed=351)
    lg = np.zeros((cfg.T, cfg.E), dtype=np.float32)
    lg[:, 4] = 9.0
    inp.logits = gen.f32_to_bf16_bits(lg)
    _check(inp, run_gpu(inp))


def test_int8_tier_zero_tokens_is_a_noop(cuda_device):
    import torch
    from weight_only_quantized_warp_b200 import qmoe
    cfg = _cfg(T=4)
    inp = gen.make_inputs(cfg, seed=352)
    m = qmoe.QMoE(cfg, "cuda:0")
    m.set_weights_from(inp)
    y = torch.full((1, cfg.H), 3.0, dtype=torch.bfloat16, device="cuda:0")
    m.forward(torch.empty((0, cfg.H), dtype=torch.bfloat16, device="cuda:0"),
              torch.empty((0, cfg.E), dtype=torch.bfloat16, device="cuda:0"), out=y[:0])
    torch.cuda.synchronize()
    assert float(y.float().min()) == 3.0


def test_int8_tier_is_bitwise_deterministic(cuda_device):
    cfg = _cfg(T=33, H=512, I=768, block_size=128)
    inp = gen.make_inputs(cfg, seed=353)
    a = run_gpu(inp)
    b = run_gpu(inp, repeat=3)
    np.testing.assert_array_equal(a.y, b.y)
    np.testing.assert_array_equal(a.hidden, b.hidden)


def test_int8_tier_replays_from_a_cuda_graph(cuda_device):
    import torch
    from weight_only_quantized_warp_b200 import qmoe
    cfg = _cfg(T=12, H=256, I=384, E=4, has_fc1_bias=True, has_fc2_bias=True, has_shared=True)
    first = gen.make_inputs(cfg, 354)
    m = qmoe.QMoE(cfg, "cuda:0")
    m.set_weights_from(first)
    x = qmoe.to_device(first.x, "cuda:0")
    lg = qmoe.to_device(first.logits, "cuda:0")
    sh = qmoe.to_device(first.shared, "cuda:0")
    y = torch.empty_like(x)
    m.workspace(cfg.T)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        m.forward(x, lg, sh, out=y)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        m.forward(x, lg, sh, out=y)
    sx, slg, ssh = gen.make_token_batch(cfg, 355)
    x.copy_(qmoe.to_device(sx, "cuda:0"))
    lg.copy_(qmoe.to_device(slg, "cuda:0"))
    sh.copy_(qmoe.to_device(ssh, "cuda:0"))
    graph.replay()
    torch.cuda.synchronize()
    replayed = y.float().cpu().numpy()
    direct = m.forward(qmoe.to_device(sx, "cuda:0"), qmoe.to_device(slg, "cuda:0"), qmoe.to_device(ssh, "cuda:0"))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(replayed, direct.float().cpu().numpy())
    del graph


@pytest.mark.parametrize("T", [8, 64])
def test_int8_tier_full_size_decode(cuda_device, T):
    cfg, seed, kw = gen.workload("mixtral_decode_i8", T=T)
    inp = gen.make_inputs(cfg, seed, **kw)
    g = run_gpu(inp)
    assert g.path == _expected_path(cfg)
    tokens = np.arange(T) if T <= 8 else np.sort(np.random.default_rng(T).choice(T, 8, replace=False))
    err = check_sampled(inp, g, tokens)
    assert err <= TOL_Y


@pytest.mark.parametrize("bits,T", [(8, 16), (4, 128), (8, 128), (4, 1024), (8, 1024)])
def test_int8_tier_full_size_sweep_shapes(cuda_device, bits, T):
    # the sweep's H=4096, I=14336 shapes on the int8 tier: int8 codes with
    # 128-code blocks and int4 with 64-code blocks, on the streaming kernel
    # (16 tokens) and the integer tensor-core GEMM (32 and 256 rows per expert)
    cfg, seed, kw = gen.sweep(bits, T)
    cfg.compute_mode = gen.COMPUTE_INT8_BLOCK
    inp = gen.make_inputs(cfg, seed, **kw)
    g = run_gpu(inp)
    assert g.path == _expected_path(cfg)
    tokens = np.sort(np.random.default_rng(seed).choice(T, 4 if T < 1024 else 8, replace=False))
    assert check_sampled(inp, g, tokens, name=f"int8_tier_sweep_int{bits}_T{T}/path{g.path}") <= TOL_Y
