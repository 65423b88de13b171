"""A second, deliberately literal statement of the whole forward (tiny shapes).

TEST INFRASTRUCTURE ONLY. It exists to cross-check ``qmoe_oracle.c`` by brute
force: routing enumerates every k-subset of experts, weights are rebuilt
element by element from their bytes, and every expert is run token by token
with Python floats (fp64). Use it for T, H, I, E of a few dozen at most.

Definitions followed are the same passages as the C oracle: the "QMoE"
operator page (layouts, pack_size, block_size, swiglu_fusion, activation
attributes, k, normalize_routing_weights), the "MoE" page summary (top-k,
gated FFN, weighted combine), the "QLinearWoQ" summary (x @ dequant(W).T + b)
and "ClikaRT::nn::QMoEWoQ" forward() (shared_output folds into the combine),
plus its class description's int8 block tier (compute_mode 1: per-block
int8 rounding of each expert input row, decided with numpy float32 scalars,
and integer dots per block), the routing bias of set_weights
(e_score_correction_bias: selection on float32 logit + bias, weights from the
unbiased logits), expert_output_scale and the tanh form of GELU. Grouped
routing, the router weight on the input, routed scaling and MXFP4 are left to
the C oracle.
"""
from __future__ import annotations

import itertools
import math

import numpy as np

from .binding import to_f64


def _code(byte_row, k, bits):
    if bits == 8:
        return int(byte_row[k])
    b = int(byte_row[k // 2])
    return b & 15 if k % 2 == 0 else b >> 4


def dense_weight(packed, scales, N, K, bits, bs):
    """[N][K] list of Python floats."""
    z = 2 ** (bits - 1)
    W = []
    for n in range(N):
        row = []
        for k in range(K):
            s = scales[n][k // bs] if bs > 0 else scales[n]
            row.append((_code(packed[n], k, bits) - z) * float(s))
        W.append(row)
    return W


def _nan_as_neg_inf(logits_row):
    return [-math.inf if math.isnan(v) else v for v in logits_row]


def select_experts(logits_row, k):
    """Brute force: the k-subset with the largest logit sum; among equal sums
    the lexicographically smallest sorted id tuple. Returned in list order
    (logit descending, id ascending). A NaN logit reads as -inf; for the
    subset sums -inf stands as a finite value below every finite logit, so
    subsets of -inf members still compare."""
    vals = _nan_as_neg_inf(logits_row)
    E = len(vals)
    floor = min([v for v in vals if math.isfinite(v)] + [0.0]) - 1e6
    key = [v if v != -math.inf else floor for v in vals]
    best, best_sum = None, None
    for sub in itertools.combinations(range(E), k):
        s = sum(key[e] for e in sub)
        if best_sum is None or s > best_sum:
            best, best_sum = sub, s
    return sorted(best, key=lambda e: (-key[e], e))


def route_weights(logits_row, sel, normalize):
    logits_row = _nan_as_neg_inf(logits_row)
    m = max(logits_row)
    ex = [math.exp(v - m) for v in logits_row]
    p = [v / sum(ex) for v in ex]
    w = [p[e] for e in sel]
    if normalize:
        tot = sum(w)
        w = [v / tot for v in w]
    return w


def round_act(v, bf16):
    """v rounded to the activation dtype: fp32 by numpy's conversion; bf16 by
    keeping 8 significant bits (round half to even, Python's round on an
    exactly scaled float)."""
    if not bf16:
        return float(np.float32(v))
    if v == 0.0 or not math.isfinite(v):
        return v
    ex = math.frexp(v)[1]
    lsb = max(ex - 8, -133)
    return math.ldexp(round(math.ldexp(v, -lsb)), lsb)


def quantize_row(v, bs):
    """Int8 block tier ("ClikaRT::nn::QMoEWoQ" class description, read as
    symmetric absmax rounding decided in fp32): per block of bs values,
    s = absmax / 127 and q = rint(v / s) clamped to +-127, with numpy float32
    scalars for every decision."""
    codes, scales = [], []
    for b in range(len(v) // bs):
        blk = [np.float32(a) for a in v[b * bs:(b + 1) * bs]]
        amax = max(abs(a) for a in blk)
        s = np.float32(amax) / np.float32(127.0)
        scales.append(float(s))
        for a in blk:
            q = 0 if s == 0 else int(np.rint(a / s))
            codes.append(max(-127, min(127, q)))
    return codes, scales


def dot_i8(packed_row, scales_row, K, bits, bs, codes, xs):
    """sum over blocks of s_w * s_x * (integer dot of centred codes)."""
    z = 2 ** (bits - 1)
    tot = 0.0
    for b in range(K // bs):
        d = sum((_code(packed_row, k, bits) - z) * codes[k] for k in range(b * bs, (b + 1) * bs))
        tot += float(scales_row[b]) * xs[b] * d
    return tot


def _gelu(a, tanh_form):
    if tanh_form:
        return 0.5 * a * (1 + math.tanh(math.sqrt(2 / math.pi) * (a + 0.044715 * a ** 3)))
    return 0.5 * a * (1 + math.erf(a / math.sqrt(2)))


def activation(act, g, u, alpha, beta, limit, gated, gelu_tanh=False):
    sig = lambda v: 1.0 / (1.0 + math.exp(-v))  # noqa: E731
    if not gated:
        a = g
        return {0: max(a, 0.0), 1: _gelu(a, gelu_tanh), 2: a * sig(a), 4: a}[act]
    if act == 3:
        al = 1.0 if alpha == 0 else alpha
        if math.isfinite(limit) and limit > 0:
            g = min(g, limit)
            u = max(-limit, min(limit, u))
        return (u + beta) * g * sig(al * g)
    base = {0: max(g, 0.0), 1: _gelu(g, gelu_tanh), 2: g * sig(g), 4: g}[act]
    return base * u


def forward(inp):
    c = inp.cfg
    x = to_f64(inp.x)
    lg = to_f64(inp.logits)
    sh = to_f64(inp.shared)
    fused = c.fusion in (1, 2)
    gated = fused or c.has_fc3
    N1 = (2 if fused else 1) * c.I

    def scl(a):
        return to_f64(a).tolist()

    def bias(a, e):
        return [0.0] * 10**6 if a is None else to_f64(a)[e].tolist()

    W1 = [dense_weight(inp.fc1_w[e], scl(inp.fc1_s)[e], N1, c.H, c.bits, c.block_size)
          for e in range(c.E)]
    W2 = [dense_weight(inp.fc2_w[e], scl(inp.fc2_s)[e], c.H, c.I, c.bits, c.block_size)
          for e in range(c.E)]
    W3 = ([dense_weight(inp.fc3_w[e], scl(inp.fc3_s)[e], c.I, c.H, c.bits, c.block_size)
           for e in range(c.E)] if c.has_fc3 else None)

    i8 = getattr(c, "compute_mode", 0) == 1
    bf16 = np.asarray(inp.x).dtype == np.uint16
    S1, S2 = scl(inp.fc1_s), scl(inp.fc2_s)
    S3 = scl(inp.fc3_s) if c.has_fc3 else None

    gt = int(getattr(c, "gelu_mode", 0)) == 1
    eos = float(getattr(c, "expert_output_scale", 1.0) or 1.0)
    sbias = getattr(inp, "score_bias", None)
    y = np.zeros((c.T, c.H))
    sels, wts = [], []
    for t in range(c.T):
        row = lg[t].tolist()
        if sbias is None:
            sel = select_experts(row, c.k)
        else:
            # selection keys: one float32 addition of logit and bias (numpy's
            # IEEE single precision); the weights use the unbiased logits
            keys = [float(np.float32(v) + np.float32(b)) for v, b in zip(np.asarray(lg[t], dtype=np.float32),
                                                                       np.asarray(sbias, dtype=np.float32))]
            sel = select_experts(keys, c.k)
        w = route_weights(row, sel, c.normalize)
        sels.append(sel)
        wts.append(w)
        xt = x[t].tolist()
        for j, e in enumerate(sel):
            b1, b2, b3 = bias(inp.fc1_b, e), bias(inp.fc2_b, e), bias(inp.fc3_b, e)
            if i8:
                qx, sx = quantize_row(xt, c.block_size)
                a = [dot_i8(inp.fc1_w[e][n], S1[e][n], c.H, c.bits, c.block_size, qx, sx) + b1[n]
                     for n in range(N1)]
            else:
                a = [sum(xt[kk] * W1[e][n][kk] for kk in range(c.H)) + b1[n] for n in range(N1)]
            h = []
            for i in range(c.I):
                if not gated:
                    h.append(activation(c.act, a[i], None, c.alpha, c.beta, c.limit, False, gt))
                    continue
                if c.fusion == 1:
                    g, u = a[2 * i], a[2 * i + 1]
                elif c.fusion == 2:
                    g, u = a[i], a[c.I + i]
                else:
                    g = a[i]
                    if i8:
                        u = dot_i8(inp.fc3_w[e][i], S3[e][i], c.H, c.bits, c.block_size, qx, sx) + b3[i]
                    else:
                        u = sum(xt[kk] * W3[e][i][kk] for kk in range(c.H)) + b3[i]
                h.append(activation(c.act, g, u, c.alpha, c.beta, c.limit, True, gt))
            if i8:
                qh, sh_ = quantize_row([round_act(v, bf16) for v in h], c.block_size)
            for m in range(c.H):
                if i8:
                    o = dot_i8(inp.fc2_w[e][m], S2[e][m], c.I, c.bits, c.block_size, qh, sh_) + b2[m]
                else:
                    o = sum(h[i] * W2[e][m][i] for i in range(c.I)) + b2[m]
                y[t, m] += w[j] * (eos * o)
        if sh is not None:
            y[t] += sh[t]
    return dict(y=y, topk_idx=np.array(sels, dtype=np.int32), topk_w=np.array(wts))
