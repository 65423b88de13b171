"""Pins of the CPU oracle against what the pages and mathematics fix.

Each test checks the oracle against something other than itself: a
hand-worked example, a closed form, an invariant, a library routine used as
an independent step, or brute force. Together they are chosen so that a
dropped term, a swapped nibble, a wrong zero point, a wrong block index, a
wrong tie-break, a transposed operand or a mis-split gate/up half fails at
least one of them.
"""
from __future__ import annotations

import dataclasses
import itertools
import json
import math
import os

import numpy as np
import pytest
from scipy.special import expit, softmax

import oracle
from oracle import literal
from weight_only_quantized_warp_b200 import inputs as gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _eval(expr: str) -> float:
    return float(eval(expr, {"__builtins__": {}}, {"exp": math.exp, "inf": math.inf}))


# ----------------------------------------------------------------- unpack / dequant

def _pack_codes(q: np.ndarray, bits: int) -> np.ndarray:
    """Test-side packer (vectorised): even k -> low nibble of byte k//2."""
    q = np.asarray(q, dtype=np.uint8)
    if bits == 8:
        return q.copy()
    return (q[..., 0::2] | (q[..., 1::2] << 4)).astype(np.uint8)


def test_golden_dequant_examples():
    for case in _golden("dequant_examples.json")["cases"]:
        row = np.frombuffer(bytes.fromhex(case["bytes_hex_row"]), dtype=np.uint8)
        N, K = case["N"], case["K"]
        w = oracle.dequant(row.reshape(N, -1), np.array(case["scales"], dtype=np.float32),
                           N, K, case["bits"], case["block_size"])
        want = np.zeros(K)
        for kk, v in case["nonzero"].items():
            want[int(kk)] = v
        np.testing.assert_array_equal(w[0], want, err_msg=case["name"])


@pytest.mark.parametrize("bits", [4, 8])
def test_unpack_every_code_every_position(bits):
    # brute force: every code value at every K position parity
    levels = 2 ** bits
    K = 2 * levels
    q = np.zeros((levels, K), dtype=np.int64)
    for c in range(levels):
        q[c] = (np.arange(K) + c) % levels  # each row a different rotation
    got = oracle.unpack(_pack_codes(q, bits), levels, K, bits)
    np.testing.assert_array_equal(got, q)


@pytest.mark.parametrize("bits,bs", [(4, 16), (4, 32), (4, 128), (8, 16), (8, 64), (4, 0), (8, 0)])
def test_dequant_round_trip_exact(bits, bs):
    """Weights W = (q - 2^(b-1)) * 2^-p with a distinct power of two per block
    are exactly representable: pack -> oracle dequant must return W bit for
    bit. A wrong block index picks a different power of two and fails."""
    rng = np.random.default_rng(7)
    N, K = 6, 256
    q = rng.integers(0, 2 ** bits, size=(N, K))
    nb = K // bs if bs else 1
    p = rng.permutation(N * nb).reshape(N, nb) % 20 + 1  # exponents 1..20
    s = np.ldexp(1.0, -p).astype(np.float32)
    blk = (np.arange(K) // bs) if bs else np.zeros(K, dtype=int)
    W = (q - 2 ** (bits - 1)) * s[:, blk].astype(np.float64)
    got = oracle.dequant(_pack_codes(q, bits), s if bs else s[:, 0], N, K, bits, bs)
    np.testing.assert_array_equal(got, W)


# ------------------------------------------------------------------------ MXFP4

def _mx_table():
    g = _golden("mxfp4_codes.json")
    return {c["code"]: _eval(c["value"]) for c in g["codes"]}


def test_mxfp4_code_and_scale_values():
    table = _mx_table()
    for code, v in table.items():
        got = oracle.e2m1(code)
        assert got == v and math.copysign(1.0, got) == math.copysign(1.0, v), code
    for sc in _golden("mxfp4_codes.json")["scales"]:
        assert oracle.to_f64(np.array([sc["byte"]], dtype=np.uint8))[0] == _eval(sc["value"])
    assert np.isnan(oracle.to_f64(np.array([255], dtype=np.uint8))[0])


def test_mxfp4_dequant_of_every_code_at_every_position():
    # codes cycle through all 16 values at every k parity; scales from bytes
    table = _mx_table()
    N, K = 16, 64
    q = (np.arange(N * K).reshape(N, K) * 7 + np.arange(N)[:, None]) % 16
    xb = (120 + (np.arange(N * (K // 32)) % 9)).astype(np.uint8).reshape(N, K // 32)
    want = np.vectorize(table.get)(q) * np.ldexp(1.0, xb.astype(np.int64) - 127)[:, np.arange(K) // 32]
    got = oracle.dequant(_pack_codes(q, 4), xb, N, K, 4, 32, mxfp4=True)
    np.testing.assert_array_equal(got, want)


def test_mxfp4_single_expert_is_the_qlinear_chain():
    # one expert forced (k = 1, renormalised): y = QLinear(act(QLinear(x))) with
    # the weights decoded through the format table, by numpy
    table = _mx_table()
    cfg = gen.MoEConfig(T=5, H=64, I=32, E=3, k=1, bits=4, block_size=32, act=gen.ACT_SWIGLU, fusion=2,
                        normalize=True, act_dtype=gen.DT_F32, scale_dtype=gen.DT_E8M0,
                        has_fc1_bias=True, has_fc2_bias=True, weight_format=gen.WEIGHTS_MXFP4)
    inp = gen.make_inputs(cfg, 41, bias_std=0.1)
    lg = np.full((cfg.T, cfg.E), -30.0, dtype=np.float32)
    lg[:, 1] = 5.0
    inp.logits = lg
    def deq(w, sc, N, K):
        q = oracle.unpack(w, N, K, 4)
        return np.vectorize(table.get)(q) * np.ldexp(1.0, sc.astype(np.int64) - 127)[:, np.arange(K) // 32]
    W1 = deq(inp.fc1_w[1], inp.fc1_s[1], 2 * cfg.I, cfg.H)
    W2 = deq(inp.fc2_w[1], inp.fc2_s[1], cfg.H, cfg.I)
    x = inp.x.astype(np.float64)
    a = x @ W1.T + inp.fc1_b[1].astype(np.float64)
    g, u = a[:, :cfg.I], a[:, cfg.I:]
    h = g * expit(g) * u
    y = h @ W2.T + inp.fc2_b[1].astype(np.float64)
    np.testing.assert_allclose(oracle.forward(inp)["y"], y, rtol=1e-12, atol=1e-12 * np.abs(y).max())


# ----------------------------------------------------------------------- routing

def test_golden_routing_examples():
    for case in _golden("routing_examples.json")["cases"]:
        lg = np.array([case["logits"]], dtype=np.float32)
        idx, w = oracle.route(lg, case["k"], case["normalize"])
        assert idx[0].tolist() == case["sel"], case
        np.testing.assert_allclose(w[0], [_eval(s) for s in case["weights"]], rtol=1e-15)


@pytest.mark.parametrize("E,k", [(4, 1), (4, 2), (5, 3), (6, 2), (6, 6), (8, 4)])
def test_routing_brute_force_with_ties(E, k):
    rng = np.random.default_rng(E * 10 + k)
    # values from a small set so ties are frequent
    lg = rng.integers(-2, 3, size=(200, E)).astype(np.float32) * 0.5
    idx, w = oracle.route(lg, k, True)
    for t in range(lg.shape[0]):
        row = lg[t].astype(np.float64).tolist()
        assert idx[t].tolist() == literal.select_experts(row, k)
        best = max(sum(row[e] for e in s) for s in itertools.combinations(range(E), k))
        assert math.isclose(sum(row[e] for e in idx[t]), best, rel_tol=0, abs_tol=0)


def test_nan_logits_read_as_negative_infinity():
    """A NaN logit loses to every number and ties resolve by id, so every
    selected index names an expert; its softmax term is exp(-inf) = 0."""
    rng = np.random.default_rng(11)
    E, k = 6, 3
    lg = rng.standard_normal((300, E))
    nan_mask = rng.random((300, E)) < 0.4
    lg[nan_mask] = np.nan
    lg[0, :] = np.nan                       # no finite logit at all
    lg[1, :] = np.nan
    lg[1, 4] = 0.5                          # one finite logit
    lg = lg.astype(np.float32)
    for normalize in (True, False):
        idx, w = oracle.route(lg, k, normalize)
        assert ((idx >= 0) & (idx < E)).all()
        for t in range(lg.shape[0]):
            row = lg[t].astype(np.float64)
            assert idx[t].tolist() == literal.select_experts(row.tolist(), k)
            finite = np.flatnonzero(~np.isnan(row))
            # finite logits first (value desc, id asc), then NaN ids ascending
            want = sorted(finite.tolist(), key=lambda e: (-row[e], e))[:k]
            want += [e for e in range(E) if np.isnan(row[e])][:k - len(want)]
            assert idx[t].tolist() == want
            if len(finite) == 0:
                assert np.isnan(w[t]).all()
                continue
            p = np.zeros(E)
            p[finite] = softmax(row[finite])
            ref = p[idx[t]]
            if normalize:
                ref = ref / ref.sum()
            np.testing.assert_allclose(w[t], ref, rtol=1e-14, atol=0)
    # grouped selection ignores NaN members when scoring a group
    lg = np.array([[np.nan, -5.0, 1.0, 0.5, np.nan, np.nan, 0.0, -1.0]])
    # group scores: {0,1} -5, {2,3} 1, {4,5} -inf (all NaN), {6,7} 0
    idx, _ = oracle.route(lg, 3, True, 4, 2)
    assert idx[0].tolist() == [2, 3, 6]
    idx, _ = oracle.route(lg, 5, True, 4, 3)
    assert idx[0].tolist() == [2, 3, 6, 7, 1]
    idx, _ = oracle.route(lg, 8, True, 4, 4)
    assert idx[0].tolist() == [2, 3, 6, 7, 1, 0, 4, 5]


def test_k_equals_E_is_the_softmax():
    rng = np.random.default_rng(3)
    E = 7
    lg = (rng.standard_normal((50, E)) * 3).astype(np.float32)
    for normalize in (True, False):
        idx, w = oracle.route(lg, E, normalize)
        ref = softmax(lg.astype(np.float64), axis=1)
        order = np.lexsort((np.tile(np.arange(E), (50, 1)), -lg), axis=1)
        np.testing.assert_array_equal(idx, order)
        np.testing.assert_allclose(w, np.take_along_axis(ref, idx, axis=1), rtol=1e-14)


def test_unnormalised_weights_are_softmax_probabilities():
    rng = np.random.default_rng(4)
    lg = rng.standard_normal((40, 8)).astype(np.float32)
    idx, w = oracle.route(lg, 2, False)
    p = softmax(lg.astype(np.float64), axis=1)
    np.testing.assert_allclose(w, np.take_along_axis(p, idx, axis=1), rtol=1e-14)
    idx2, w2 = oracle.route(lg, 2, True)
    np.testing.assert_array_equal(idx, idx2)
    np.testing.assert_allclose(w2.sum(axis=1), 1.0, rtol=1e-15)


# ------------------------------------------- e_score_correction_bias (QMoEWoQ pages)

def test_golden_score_bias_examples():
    for case in _golden("routing_bias.json")["cases"]:
        lg = np.array([case["logits"]], dtype=np.float32)
        idx, w = oracle.route(lg, case["k"], case["normalize"], score_bias=np.array(case["bias"], dtype=np.float32))
        assert idx[0].tolist() == case["sel"], case
        np.testing.assert_allclose(w[0], [_eval(s) for s in case["weights"]], rtol=1e-14)


@pytest.mark.parametrize("E,G,TG,k", [(8, 0, 0, 2), (16, 0, 0, 5), (16, 4, 2, 4), (32, 8, 3, 6)])
def test_score_bias_against_float32_keys(E, G, TG, k):
    """Selection = top-k of numpy float32(logit) + float32(bias) (IEEE single
    additions), groups scored by their largest key; weights = the unbiased
    softmax restricted to the selection."""
    rng = np.random.default_rng(E * 3 + k)
    lg = rng.standard_normal((150, E)).astype(np.float32)
    b = (rng.standard_normal(E) * 0.7).astype(np.float32)
    keys = lg + b                      # float32 + float32 -> float32
    for normalize in (True, False):
        idx, w = oracle.route(lg, k, normalize, G, TG, score_bias=b)
        p = softmax(lg.astype(np.float64), axis=1)
        for t in range(lg.shape[0]):
            allowed = np.ones(E, dtype=bool)
            if G > 1:
                gs = keys[t].reshape(G, E // G).max(axis=1)
                order = sorted(range(G), key=lambda g: (-gs[g], g))[:TG]
                allowed = np.isin(np.arange(E) // (E // G), order)
            cand = [e for e in range(E) if allowed[e]]
            want = sorted(cand, key=lambda e: (-keys[t, e], e))[:k]
            assert idx[t].tolist() == want
            ref = p[t, want]
            if normalize:
                ref = ref / ref.sum()
            np.testing.assert_allclose(w[t], ref, rtol=1e-14)
    # a zero bias changes nothing
    i0, w0 = oracle.route(lg, k, True, G, TG)
    i1, w1 = oracle.route(lg, k, True, G, TG, score_bias=np.zeros(E, dtype=np.float32))
    np.testing.assert_array_equal(i0, i1)
    np.testing.assert_array_equal(w0, w1)


# ------------------------------------------------- gelu_mode, expert_output_scale

def test_gelu_tanh_form_against_torch():
    """The tanh form of GELU equals torch's gelu(approximate="tanh") in fp64,
    stays within 1e-3 of the erf form, and keeps gelu(a) - gelu(-a) = a."""
    import torch
    a = np.linspace(-8.0, 8.0, 641)
    ref = torch.nn.functional.gelu(torch.from_numpy(a), approximate="tanh").numpy()
    got = np.array([oracle.plain_act(5, v) for v in a])
    np.testing.assert_allclose(got, ref, rtol=1e-14, atol=1e-15)
    erf = np.array([oracle.plain_act(gen.ACT_GELU, v) for v in a])
    assert np.abs(got - erf).max() < 1e-3
    neg = np.array([oracle.plain_act(5, -v) for v in a])
    np.testing.assert_allclose(got - neg, a, rtol=0, atol=1e-14)
    # gated use: act(g) * u with the same form
    assert oracle.gated_act(5, 1.25, -0.5, 0.0, 0.0, math.inf) == oracle.plain_act(5, 1.25) * -0.5


def test_gelu_mode_selects_the_form_in_the_forward():
    cfg = _tiny_cfg(T=5, fusion=0, act=gen.ACT_GELU, has_fc1_bias=True)
    inp = gen.make_inputs(cfg, seed=23, bias_std=0.1)
    y_erf = oracle.forward(inp, want_h=True)
    inp_t = dataclasses.replace(inp, cfg=dataclasses.replace(cfg, gelu_mode=1))
    y_tanh = oracle.forward(inp_t, want_h=True)
    assert not np.array_equal(y_erf["h"], y_tanh["h"])
    np.testing.assert_allclose(y_tanh["h"], y_erf["h"], rtol=0, atol=1e-3 * np.abs(y_erf["h"]).max() + 1e-3)


def test_expert_output_scale_scales_every_expert_output():
    """eos multiplies each expert output (with its fc2 bias) before the
    router weighting: y - shared scales by eos, the same as
    routed_scaling_factor, and a forced single expert gives eos times the
    two-layer QLinear chain."""
    cfg = _tiny_cfg(T=6, has_fc2_bias=True, has_shared=True)
    inp = gen.make_inputs(cfg, seed=24, bias_std=0.1)
    sh = oracle.to_f64(inp.shared)
    y1 = oracle.forward(inp)["y"]
    y3 = oracle.forward(dataclasses.replace(inp, cfg=dataclasses.replace(cfg, expert_output_scale=3.0)))["y"]
    r3 = oracle.forward(dataclasses.replace(inp, cfg=dataclasses.replace(cfg, routed_scaling_factor=3.0)))["y"]
    np.testing.assert_allclose(y3 - sh, 3.0 * (y1 - sh), rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(y3, r3, rtol=1e-14, atol=1e-14)
    # 0 reads as 1
    y0 = oracle.forward(dataclasses.replace(inp, cfg=dataclasses.replace(cfg, expert_output_scale=0.0)))["y"]
    np.testing.assert_array_equal(y0, y1)


# -------------------------------------------------------- routing options (MoE page)

def test_golden_grouped_routing_examples():
    for case in _golden("routing_grouped.json")["cases"]:
        lg = np.array([case["logits"]], dtype=np.float64)  # the decimal values exactly
        idx, w = oracle.route(lg, case["k"], case["normalize"], case["n_group"], case["topk_group"])
        assert idx[0].tolist() == case["sel"], case
        np.testing.assert_allclose(w[0], [_eval(s) for s in case["weights"]], rtol=1e-14)


@pytest.mark.parametrize("E,G,TG,k", [(8, 4, 2, 3), (16, 4, 1, 4), (32, 8, 3, 6), (64, 8, 4, 6), (12, 3, 2, 5)])
def test_grouped_routing_against_numpy_sorts(E, G, TG, k):
    # an independent statement with numpy primitives: group maxima by a
    # reshape, kept groups and the final choice by lexicographic sorts
    rng = np.random.default_rng(E + G + TG + k)
    lg = (rng.integers(-3, 4, size=(300, E)) * 0.5).astype(np.float32)  # many ties
    idx, _ = oracle.route(lg, k, True, G, TG)
    for t in range(lg.shape[0]):
        row = lg[t].astype(np.float64)
        gmax = row.reshape(G, E // G).max(axis=1)
        kept = np.lexsort((np.arange(G), -gmax))[:TG]
        allowed = np.isin(np.arange(E) // (E // G), kept)
        cand = np.nonzero(allowed)[0]
        order = cand[np.lexsort((cand, -row[cand]))]
        np.testing.assert_array_equal(idx[t], order[:k])


def test_all_groups_kept_is_plain_top_k():
    rng = np.random.default_rng(7)
    lg = rng.standard_normal((100, 16)).astype(np.float32)
    for normalize in (True, False):
        i0, w0 = oracle.route(lg, 4, normalize)
        i1, w1 = oracle.route(lg, 4, normalize, 4, 4)
        np.testing.assert_array_equal(i0, i1)
        np.testing.assert_array_equal(w0, w1)


def _small(**kw):
    base = dict(T=6, H=64, I=64, E=4, k=2, bits=4, block_size=32, act=gen.ACT_SWIGLU, fusion=1,
                normalize=True, act_dtype=gen.DT_F32, scale_dtype=gen.DT_F32, has_shared=True)
    base.update(kw)
    return gen.MoEConfig(**base)


def test_routed_scaling_factor_scales_only_the_routed_sum():
    # without a shared output, scaling by a power of two is exact
    cfg = _small(has_shared=False)
    inp = gen.make_inputs(cfg, 31)
    y1 = oracle.forward(inp)["y"]
    inp.cfg = dataclasses.replace(cfg, routed_scaling_factor=2.0)
    np.testing.assert_array_equal(oracle.forward(inp)["y"], 2.0 * y1)
    # the shared output is added after the scaling, unscaled
    cfg = _small()
    inp = gen.make_inputs(cfg, 31)
    y1 = oracle.forward(inp)["y"]
    inp.cfg = dataclasses.replace(cfg, routed_scaling_factor=0.25)
    sh = oracle.to_f64(inp.shared)
    np.testing.assert_allclose(oracle.forward(inp)["y"], 0.25 * (y1 - sh) + sh, rtol=0,
                               atol=1e-14 * np.abs(y1).max())


def test_router_weight_on_input_with_one_expert_and_renormalised_weight_changes_nothing():
    # k = 1 with renormalisation: the weight is exactly 1 wherever it is applied
    cfg = _small(k=1, has_fc1_bias=True, has_fc2_bias=True)
    inp = gen.make_inputs(cfg, 32)
    y0 = oracle.forward(inp)["y"]
    inp.cfg = dataclasses.replace(cfg, apply_router_weight_on_input=True)
    np.testing.assert_array_equal(oracle.forward(inp)["y"], y0)


def test_router_weight_on_input_of_a_linear_ffn_equals_weight_on_output():
    # identity activation, no biases: the FFN is linear, so w * FFN(x) = FFN(w * x)
    cfg = _small(act=gen.ACT_IDENTITY, fusion=0, k=2, normalize=False)
    inp = gen.make_inputs(cfg, 33)
    y0 = oracle.forward(inp)["y"]
    inp.cfg = dataclasses.replace(cfg, apply_router_weight_on_input=True)
    y1 = oracle.forward(inp)["y"]
    np.testing.assert_allclose(y1, y0, rtol=0, atol=1e-12 * np.abs(y0).max())
    # with a non-linear activation the two placements differ
    cfg = _small(k=2, normalize=False)
    inp = gen.make_inputs(cfg, 33)
    y0 = oracle.forward(inp)["y"]
    inp.cfg = dataclasses.replace(cfg, apply_router_weight_on_input=True)
    assert np.abs(oracle.forward(inp)["y"] - y0).max() > 1e-6 * np.abs(y0).max()


# ------------------------------------------------------------------- permutation

@pytest.mark.parametrize("T,E,k", [(1, 4, 2), (37, 8, 2), (64, 64, 6), (100, 5, 5)])
def test_permutation_invariants(T, E, k):
    rng = np.random.default_rng(T + E)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    idx, _ = oracle.route(lg, k, True)
    offsets, perm, inv = oracle.permute(idx, E)
    counts = np.bincount(idx.ravel(), minlength=E)
    np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]))
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        np.testing.assert_array_equal(seg, np.sort(np.nonzero((idx == e).any(axis=1))[0]))
    for t in range(T):
        for j in range(k):
            p = inv[t, j]
            assert perm[p] == t
            assert offsets[idx[t, j]] <= p < offsets[idx[t, j] + 1]
    assert sorted(inv.ravel().tolist()) == list(range(T * k))


def test_permutation_empty_and_single_expert():
    idx = np.zeros((5, 1), dtype=np.int32) + 2
    offsets, perm, inv = oracle.permute(idx, 4)
    assert offsets.tolist() == [0, 0, 0, 5, 5]
    assert perm.tolist() == [0, 1, 2, 3, 4]
    offsets, perm, inv = oracle.permute(np.zeros((0, 2), dtype=np.int32), 3)
    assert offsets.tolist() == [0, 0, 0, 0]


# -------------------------------------------------------------------- activations

def test_swiglu_without_limit_is_silu_gate_times_up():
    rng = np.random.default_rng(5)
    for g, u in rng.standard_normal((100, 2)) * 4:
        got = oracle.gated_act(gen.ACT_SWIGLU, g, u, 1.0, 0.0, math.inf)
        assert math.isclose(got, g * expit(g) * u, rel_tol=1e-14, abs_tol=1e-300)
        # alpha 0 reads as 1; limit 0 reads as no clamp
        assert oracle.gated_act(gen.ACT_SWIGLU, g, u, 0.0, 0.0, 0.0) == got
        assert math.isclose(oracle.gated_act(gen.ACT_SILU, g, u, 9.0, 9.0, 1.0), got,
                            rel_tol=1e-14, abs_tol=1e-300)


def test_swiglu_clamp_invariances():
    a, b, L = 1.702, 1.0, 7.0
    f = lambda g, u: oracle.gated_act(gen.ACT_SWIGLU, g, u, a, b, L)  # noqa: E731
    assert f(10.0, 2.0) == f(7.0, 2.0)        # gate clamped from above
    assert f(-10.0, 2.0) != f(-7.0, 2.0)      # gate not clamped from below
    assert f(3.0, 9.0) == f(3.0, 7.0)         # up clamped from above
    assert f(3.0, -9.0) == f(3.0, -7.0)       # ... and from below
    assert f(3.0, 6.5) != f(3.0, 7.0)
    # beta shifts the up branch: h(beta=1) - h(beta=0) = g' * sigmoid(a g')
    d = f(2.0, 0.5) - oracle.gated_act(gen.ACT_SWIGLU, 2.0, 0.5, a, 0.0, L)
    assert math.isclose(d, 2.0 * expit(a * 2.0), rel_tol=1e-14)


def test_plain_activations():
    # standard normal CDF at 1 (tabulated): 0.8413447460685429
    assert math.isclose(oracle.plain_act(gen.ACT_GELU, 1.0), 0.8413447460685429, rel_tol=1e-14)
    for v in (-3.0, -0.5, 0.0, 0.7, 2.5):
        assert math.isclose(oracle.plain_act(gen.ACT_GELU, v) - oracle.plain_act(gen.ACT_GELU, -v),
                            v, rel_tol=1e-13, abs_tol=1e-15)
        assert oracle.plain_act(gen.ACT_RELU, v) == max(v, 0.0)
        assert oracle.plain_act(gen.ACT_IDENTITY, v) == v
        assert math.isclose(oracle.plain_act(gen.ACT_SILU, v), v * expit(v), rel_tol=1e-14,
                            abs_tol=1e-300)
    # gated forms multiply the gate activation by up
    assert math.isclose(oracle.gated_act(gen.ACT_GELU, 1.0, 3.0, 0, 0, 0), 3 * 0.8413447460685429,
                        rel_tol=1e-14)
    assert oracle.gated_act(gen.ACT_RELU, -1.0, 3.0, 0, 0, 0) == 0.0


# ----------------------------------------------------------------- whole forward

def _tiny_cfg(**kw):
    base = dict(T=6, H=32, I=16, E=4, k=2, bits=4, block_size=16, act=gen.ACT_SWIGLU, fusion=1,
                normalize=True, act_dtype=gen.DT_F32, scale_dtype=gen.DT_F32)
    base.update(kw)
    return gen.MoEConfig(**base)


def test_golden_one_token_forward():
    d = _golden("forward_one_token.json")
    c = d["config"]
    cfg = gen.MoEConfig(T=1, H=2, I=1, E=2, k=1, bits=8, block_size=0, act=c["act"], fusion=2,
                        alpha=1.0, beta=0.0, limit=math.inf, normalize=True,
                        act_dtype=gen.DT_F32, scale_dtype=gen.DT_F32)
    f32 = lambda a: np.array(a, dtype=np.float32)  # noqa: E731
    inp = gen.MoEInputs(cfg, x=f32(d["x"]), logits=f32(d["logits"]),
                        fc1_w=np.array(d["fc1_codes"], dtype=np.uint8), fc1_s=f32(d["fc1_scales"]),
                        fc2_w=np.array(d["fc2_codes"], dtype=np.uint8), fc2_s=f32(d["fc2_scales"]))
    y = oracle.forward(inp)["y"]
    np.testing.assert_allclose(y[0], [_eval(s) for s in d["y_no_bias_no_shared"]], rtol=1e-15)
    cfg.has_fc2_bias = cfg.has_shared = True
    inp.fc2_b, inp.shared = f32(d["fc2_bias"]), f32(d["shared"])
    y = oracle.forward(inp)["y"]
    np.testing.assert_allclose(y[0], [_eval(s) for s in d["y_with_bias_and_shared"]], rtol=1e-15)


def _dense(inp, which, e):
    c = inp.cfg
    w = getattr(inp, which + "_w")[e]
    s = getattr(inp, which + "_s")[e]
    N = w.shape[0]
    K = w.shape[1] * 8 // c.bits
    return oracle.dequant(w, s, N, K, c.bits, c.block_size)


def _ffn_numpy(inp, e, x64):
    """One expert as two QLinear layers, y = x @ dequant(W).T + b (numpy matmul)."""
    c = inp.cfg
    b = lambda a, n: np.zeros(n) if a is None else oracle.to_f64(a)[e]  # noqa: E731
    a1 = x64 @ _dense(inp, "fc1", e).T + b(inp.fc1_b, c.n1)
    if c.fusion == 1:
        g, u = a1[:, 0::2], a1[:, 1::2]
    elif c.fusion == 2:
        g, u = a1[:, :c.I], a1[:, c.I:]
    elif c.has_fc3:
        g, u = a1, x64 @ _dense(inp, "fc3", e).T + b(inp.fc3_b, c.I)
    else:
        g, u = a1, None
    if u is None:
        h = np.vectorize(lambda v: oracle.plain_act(c.act, v))(g)
    else:
        h = np.vectorize(lambda gg, uu: oracle.gated_act(c.act, gg, uu, c.alpha, c.beta, c.limit))(g, u)
    return h @ _dense(inp, "fc2", e).T + b(inp.fc2_b, c.H)


@pytest.mark.parametrize("fusion,fc3", [(1, False), (2, False), (0, True)])
def test_k_equals_E_is_the_dense_softmax_mixture(fusion, fc3):
    cfg = _tiny_cfg(k=4, E=4, fusion=fusion, has_fc3=fc3, act=gen.ACT_SWIGLU if fusion else gen.ACT_SILU,
                    has_fc1_bias=True, has_fc2_bias=True, has_fc3_bias=fc3, alpha=1.702, beta=1.0,
                    limit=7.0)
    inp = gen.make_inputs(cfg, seed=11, bias_std=0.1)
    y = oracle.forward(inp)["y"]
    x64 = oracle.to_f64(inp.x)
    p = softmax(oracle.to_f64(inp.logits), axis=1)
    ref = sum(p[:, [e]] * _ffn_numpy(inp, e, x64) for e in range(cfg.E))
    np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("bits,bs", [(4, 32), (8, 0), (8, 16)])
def test_single_forced_expert_is_a_qlinear_chain(bits, bs):
    cfg = _tiny_cfg(k=1, bits=bits, block_size=bs, fusion=2, has_fc1_bias=True, has_fc2_bias=True)
    inp = gen.make_inputs(cfg, seed=12)
    lg = np.zeros((cfg.T, cfg.E), dtype=np.float32)
    lg[:, 2] = 50.0
    inp.logits = lg
    y = oracle.forward(inp)["y"]
    ref = _ffn_numpy(inp, 2, oracle.to_f64(inp.x))
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-13)


def test_fusion_layouts_of_one_logical_weight_agree():
    """The same gate/up rows stored as fusion 1, fusion 2 and fc1+fc3 give the
    same y bit for bit (same sums in the same order)."""
    cfg2 = _tiny_cfg(fusion=2, has_fc1_bias=True)
    base = gen.make_inputs(cfg2, seed=13)
    I = cfg2.I
    gate_w, up_w = base.fc1_w[:, :I], base.fc1_w[:, I:]
    gate_s, up_s = base.fc1_s[:, :I], base.fc1_s[:, I:]
    gate_b, up_b = base.fc1_b[:, :I], base.fc1_b[:, I:]
    y2 = oracle.forward(base)["y"]

    inter = lambda a, b: np.stack([a, b], axis=2).reshape(a.shape[0], 2 * I, *a.shape[2:])  # noqa: E731
    i1 = dataclasses.replace(base, cfg=dataclasses.replace(cfg2, fusion=1),
                             fc1_w=inter(gate_w, up_w), fc1_s=inter(gate_s, up_s),
                             fc1_b=inter(gate_b, up_b))
    y1 = oracle.forward(i1)["y"]
    i0 = dataclasses.replace(base, cfg=dataclasses.replace(cfg2, fusion=0, has_fc3=True,
                                                           has_fc3_bias=True, act=gen.ACT_SWIGLU),
                             fc1_w=gate_w.copy(), fc1_s=gate_s.copy(), fc1_b=gate_b.copy(),
                             fc3_w=up_w.copy(), fc3_s=up_s.copy(), fc3_b=up_b.copy())
    y0 = oracle.forward(i0)["y"]
    np.testing.assert_array_equal(y1, y2)
    np.testing.assert_array_equal(y0, y2)


def test_shared_zero_equals_absent_and_bias_is_weighted():
    cfg = _tiny_cfg(has_fc2_bias=True)
    inp = gen.make_inputs(cfg, seed=14)
    r = oracle.forward(inp)
    y_bias = r["y"]
    inp0 = dataclasses.replace(inp, fc2_b=np.zeros_like(inp.fc2_b))
    y_nob = oracle.forward(inp0)["y"]
    b2 = oracle.to_f64(inp.fc2_b)
    want = sum(r["topk_w"][:, [j]] * b2[r["topk_idx"][:, j]] for j in range(cfg.k))
    np.testing.assert_allclose(y_bias - y_nob, want, rtol=1e-9, atol=1e-15)
    inpz = dataclasses.replace(inp, shared=np.zeros((cfg.T, cfg.H), dtype=np.float32))
    np.testing.assert_array_equal(oracle.forward(inpz)["y"], y_bias)


LITERAL_CASES = [
    dict(),
    dict(fusion=2, bits=8, block_size=0, normalize=False),
    dict(fusion=0, has_fc3=True, act=gen.ACT_SILU, has_fc3_bias=True, has_fc1_bias=True),
    dict(fusion=0, act=gen.ACT_GELU, has_fc1_bias=True),
    dict(fusion=0, act=gen.ACT_RELU),
    dict(fusion=0, act=gen.ACT_IDENTITY, bits=8, block_size=16),
    dict(alpha=1.702, beta=1.0, limit=0.5, has_fc1_bias=True, has_fc2_bias=True, has_shared=True),
    dict(act_dtype=gen.DT_BF16, scale_dtype=gen.DT_BF16, k=3, E=5),
    dict(has_score_bias=True, k=3, E=6, normalize=False),
    dict(fusion=0, act=gen.ACT_GELU, gelu_mode=1, has_fc1_bias=True, expert_output_scale=1.5, has_fc2_bias=True),
    dict(fusion=1, act=gen.ACT_GELU, gelu_mode=1, has_score_bias=True, expert_output_scale=0.5),
]


@pytest.mark.parametrize("kw", LITERAL_CASES, ids=[str(i) for i in range(len(LITERAL_CASES))])
def test_whole_forward_matches_literal_restatement(kw):
    cfg = _tiny_cfg(T=4, H=32, I=16, **kw)
    inp = gen.make_inputs(cfg, seed=21, bias_std=0.1)
    a = oracle.forward(inp)
    b = literal.forward(inp)
    np.testing.assert_array_equal(a["topk_idx"], b["topk_idx"])
    np.testing.assert_allclose(a["topk_w"], b["topk_w"], rtol=1e-13)
    np.testing.assert_allclose(a["y"], b["y"], rtol=1e-12, atol=1e-12 * np.abs(b["y"]).max())


def test_sampled_tokens_equal_rows_of_full_run():
    cfg = _tiny_cfg(T=9, has_shared=True)
    inp = gen.make_inputs(cfg, seed=22)
    full = oracle.forward(inp)["y"]
    sub = oracle.forward(inp, tokens=[8, 0, 3])["y"]
    np.testing.assert_array_equal(sub, full[[8, 0, 3]])
