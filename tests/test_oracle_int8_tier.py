"""Pins of the oracle's int8 block compute tier.

The "ClikaRT::nn::QMoEWoQ" page (class description) says that a packed block
weight on the int8 block tier rounds the activation to per-block int8 before
the dot, and gives no rounding rule. The oracle reads it as symmetric absmax
rounding over the weight's own K blocks, decided in fp32:
s = absmax / 127, q = clamp(rint(v / s), -127, 127) with ties to even, and the
dot sums s_w * s * (integer dot of centred weight codes and q) over blocks.

The pins below fix that reading from outside the oracle: closed forms of the
rounding (exact scales, ties to even, the all-zero block), the error bound of
round-to-nearest, the special case in which rounding is lossless (the tier's
dot must then equal the float dot of the dequantised weights, which the
dequant pins fix), and the forward's wiring of the pinned pieces.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import pytest

import oracle
from oracle import literal
from weight_only_quantized_warp_b200 import inputs as gen


def _f32(a):
    return np.asarray(a, dtype=np.float32)


def test_rounding_closed_forms_and_ties_to_even():
    bs = 32
    # block 0: absmax 127 -> s = 1 exactly, codes are rint(v) with ties to even
    b0 = np.zeros(bs)
    b0[:9] = [127.0, 63.5, -0.5, 0.5, 1.5, 2.5, -2.5, -127.0, 3.49]
    want0 = [127, 64, 0, 0, 2, 2, -2, -127, 3]
    # block 1: the same values / 8 -> s = 1/8 exactly, the same codes
    b1 = b0 / 8.0
    # block 2: all zero -> s = 0, codes 0
    b2 = np.zeros(bs)
    # block 3: one nonzero value -> it maps to 127, the rest to 0
    b3 = np.zeros(bs)
    b3[5] = -3.0
    x = _f32(np.concatenate([b0, b1, b2, b3]))[None]
    q, s = oracle.quantize_i8(x, bs)
    assert s.dtype == np.float32
    assert s[0, 0] == 1.0 and s[0, 1] == 0.125 and s[0, 2] == 0.0
    assert s[0, 3] == np.float32(3.0) / np.float32(127.0)
    np.testing.assert_array_equal(q[0, :9], want0)
    np.testing.assert_array_equal(q[0, bs:bs + 9], want0)
    assert not q[0, 9:bs].any() and not q[0, 2 * bs:3 * bs].any()
    assert q[0, 3 * bs + 5] == -127 and np.count_nonzero(q[0, 3 * bs:]) == 1


def test_rounding_of_bf16_rows_reads_the_stored_values():
    rng = np.random.default_rng(3)
    v = rng.standard_normal((5, 256)).astype(np.float32)
    bits = gen.f32_to_bf16_bits(v)
    q16, s16 = oracle.quantize_i8(bits, 64)
    q32, s32 = oracle.quantize_i8(gen.bf16_bits_to_f32(bits), 64)
    np.testing.assert_array_equal(q16, q32)
    np.testing.assert_array_equal(s16, s32)


@pytest.mark.parametrize("bs", [32, 64, 128, 1024])
def test_rounding_error_bound_and_code_range(bs):
    rng = np.random.default_rng(bs)
    x = (rng.standard_normal((7, 2048)) * np.exp(rng.uniform(-6, 6, size=(7, 1)))).astype(np.float32)
    x[2, :bs] = 0.0
    q, s = oracle.quantize_i8(x, bs)
    sk = np.repeat(s, bs, axis=1).astype(np.float64)
    err = np.abs(x.astype(np.float64) - sk * q)
    # round to nearest: within half a step (plus the fp32 rounding of v / s)
    assert np.all(err <= sk * 0.5 * (1 + 2.0 ** -20))
    blocks = np.abs(q.reshape(7, -1, bs)).max(axis=2)
    nonzero = np.abs(x.reshape(7, -1, bs)).max(axis=2) > 0
    np.testing.assert_array_equal(blocks[nonzero], 127)
    np.testing.assert_array_equal(blocks[~nonzero], 0)
    assert np.all((np.sign(q) == np.sign(x)) | (q == 0))


def _lossless_rows(rng, rows, K, bs):
    """Rows v = 2^-e * m with integer m in [-127, 127] and +-127 in every block:
    s = 2^-e exactly and the codes are m, so rounding loses nothing."""
    m = rng.integers(-127, 128, size=(rows, K))
    m[:, ::bs] = 127 * rng.choice([-1, 1], size=(rows, K // bs))
    e = rng.integers(2, 9, size=(rows, K // bs))
    return m, np.repeat(np.ldexp(1.0, -e), bs, axis=1) * m


@pytest.mark.parametrize("bits,bs", [(4, 64), (4, 128), (8, 32), (8, 256)])
def test_lossless_rows_make_the_int8_dot_the_float_dot(bits, bs):
    rng = np.random.default_rng(bits * 1000 + bs)
    N, K, rows = 24, 512, 3
    m, x = _lossless_rows(rng, rows, K, bs)
    x = _f32(x)
    q, s = oracle.quantize_i8(x, bs)
    np.testing.assert_array_equal(q, m)
    codes = rng.integers(0, 1 << bits, size=(N, K))
    packed = codes.astype(np.uint8) if bits == 8 else (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    scales = _f32(rng.uniform(0.001, 0.02, size=(N, K // bs)))
    w = oracle.dequant(packed, scales, N, K, bits, bs)
    got = oracle.linear_i8(x, packed, scales, N, K, bits, bs)
    want = x.astype(np.float64) @ w.T
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


@pytest.mark.parametrize("bits,bs", [(4, 64), (8, 128)])
def test_int8_dot_error_bound(bits, bs):
    rng = np.random.default_rng(bits + bs)
    N, K, rows = 16, 1024, 4
    x = _f32(rng.standard_normal((rows, K)))
    codes = rng.integers(0, 1 << bits, size=(N, K))
    packed = codes.astype(np.uint8) if bits == 8 else (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    scales = _f32(rng.uniform(0.001, 0.02, size=(N, K // bs)))
    w = oracle.dequant(packed, scales, N, K, bits, bs)
    _, s = oracle.quantize_i8(x, bs)
    got = oracle.linear_i8(x, packed, scales, N, K, bits, bs)
    want = x.astype(np.float64) @ w.T
    # each activation moves by at most half its block's step
    bound = (np.abs(w)[None, :, :] * (0.5 * np.repeat(s, bs, axis=1))[:, None, :]).sum(axis=2)
    assert np.all(np.abs(got - want) <= bound * (1 + 1e-5) + 1e-12)
    assert np.abs(got - want).max() > 0  # the tier does round


def _tier_cfg(**kw):
    base = dict(T=6, H=128, I=64, E=4, k=2, bits=4, block_size=64, act=gen.ACT_SWIGLU, fusion=1,
                normalize=True, act_dtype=gen.DT_F32, scale_dtype=gen.DT_F32,
                compute_mode=gen.COMPUTE_INT8_BLOCK)
    base.update(kw)
    return gen.MoEConfig(**base)


@pytest.mark.parametrize("fusion,fc3,bits,bs", [(1, False, 4, 64), (2, False, 8, 32), (0, True, 8, 128)])
def test_forward_fc1_on_lossless_inputs_equals_the_float_tier(fusion, fc3, bits, bs):
    cfg = _tier_cfg(fusion=fusion, has_fc3=fc3, bits=bits, block_size=bs, has_fc1_bias=True,
                    has_fc3_bias=fc3, act=gen.ACT_SWIGLU if fusion else gen.ACT_SILU)
    inp = gen.make_inputs(cfg, seed=31, bias_std=0.1)
    rng = np.random.default_rng(31)
    inp.x = _f32(_lossless_rows(rng, cfg.T, cfg.H, bs)[1])
    h8 = oracle.forward(inp, want_h=True)["h"]
    flt = dataclasses.replace(inp, cfg=dataclasses.replace(cfg, compute_mode=gen.COMPUTE_FLOAT))
    hf = oracle.forward(flt, want_h=True)["h"]
    np.testing.assert_allclose(h8, hf, rtol=1e-12, atol=1e-12 * np.abs(hf).max())


@pytest.mark.parametrize("act_dtype", [gen.DT_F32, gen.DT_BF16])
def test_forward_fc2_reads_h_rounded_to_the_activation_dtype(act_dtype):
    # one forced expert with weight 1: y = int8-tier FC2 of round(h) + b2
    cfg = _tier_cfg(k=1, fusion=2, has_fc2_bias=True, act_dtype=act_dtype, scale_dtype=act_dtype)
    inp = gen.make_inputs(cfg, seed=32, bias_std=0.1)
    lg = np.zeros((cfg.T, cfg.E), dtype=np.float32)
    lg[:, 3] = 60.0
    inp.logits = gen.f32_to_bf16_bits(lg) if act_dtype == gen.DT_BF16 else lg
    r = oracle.forward(inp, want_h=True)
    hr = np.vectorize(lambda v: oracle.round_act(v, act_dtype == gen.DT_BF16))(r["h"])
    want = oracle.linear_i8(_f32(hr), inp.fc2_w[3], inp.fc2_s[3], cfg.H, cfg.I, cfg.bits, cfg.block_size)
    want += oracle.to_f64(inp.fc2_b)[3]
    np.testing.assert_allclose(r["y"], want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_round_act_matches_the_bit_level_rounding():
    rng = np.random.default_rng(5)
    v = (rng.standard_normal(4000) * np.exp(rng.uniform(-30, 30, 4000))).astype(np.float32)
    want = gen.bf16_bits_to_f32(gen.f32_to_bf16_bits(v)).astype(np.float64)
    got = np.array([oracle.round_act(float(a), True) for a in v])
    np.testing.assert_array_equal(got, want)
    # ties to even: halfway between 1 and 1 + 2^-7 goes to 1; the next tie goes up
    assert oracle.round_act(1.0 + 2.0 ** -8, True) == 1.0
    assert oracle.round_act(1.0 + 3 * 2.0 ** -8, True) == 1.0 + 2.0 ** -6
    assert oracle.round_act(1.0 + 2.0 ** -30, False) == float(np.float32(1.0 + 2.0 ** -30))


def test_int8_tier_stays_close_to_the_float_tier():
    cfg = _tier_cfg(T=8, H=256, I=128, has_fc1_bias=True, has_fc2_bias=True, has_shared=True)
    inp = gen.make_inputs(cfg, seed=33, bias_std=0.1)
    y8 = oracle.forward(inp)["y"]
    yf = oracle.forward(dataclasses.replace(inp, cfg=dataclasses.replace(cfg, compute_mode=0)))["y"]
    rel = np.abs(y8 - yf).max() / np.abs(yf).max()
    assert 0 < rel < 0.03


LITERAL_TIER_CASES = [
    dict(),
    dict(bits=8, block_size=16, fusion=2, has_fc1_bias=True, has_fc2_bias=True),
    dict(fusion=0, has_fc3=True, act=gen.ACT_SILU, has_fc3_bias=True, has_shared=True),
    dict(act_dtype=gen.DT_BF16, scale_dtype=gen.DT_BF16, k=3, E=5),
    dict(act_dtype=gen.DT_BF16, scale_dtype=gen.DT_BF16, fusion=0, act=gen.ACT_GELU, bits=8),
]


@pytest.mark.parametrize("kw", LITERAL_TIER_CASES, ids=[str(i) for i in range(len(LITERAL_TIER_CASES))])
def test_forward_matches_the_literal_restatement(kw):
    # the Python-float restatement (numpy float32 rounding decisions, integer
    # dots, bf16 rounding by exact scaling) against the C oracle
    cfg = _tier_cfg(**{"T": 4, "H": 32, "I": 16, "block_size": 16, **kw})
    inp = gen.make_inputs(cfg, seed=34, bias_std=0.1)
    a = oracle.forward(inp)
    b = literal.forward(inp)
    np.testing.assert_array_equal(a["topk_idx"], b["topk_idx"])
    np.testing.assert_allclose(a["y"], b["y"], rtol=1e-12, atol=1e-12 * np.abs(b["y"]).max())


def test_literal_rounding_equals_the_oracle_rounding():
    rng = np.random.default_rng(35)
    x = (rng.standard_normal((6, 64)) * np.exp(rng.uniform(-8, 8, size=(6, 1)))).astype(np.float32)
    x[2, :16] = 0.0
    q, s = oracle.quantize_i8(x, 16)
    for r in range(6):
        lq, ls = literal.quantize_row(x[r].astype(np.float64).tolist(), 16)
        np.testing.assert_array_equal(q[r], lq)
        np.testing.assert_array_equal(s[r], np.array(ls, dtype=np.float32))
