"""Seeded synthetic inputs for the weight-only-quantized MoE forward.

This module only draws numbers. It holds none of the operator's arithmetic:
no unpacking, no dequantisation, no routing and no FFN. Both the CUDA path
and the CPU oracle receive the arrays it returns, and each side interprets
them on its own.

Tensor shapes follow the QMoE operator page (graiphic.io, "QMoE", input
list):

* ``fc1_w``  ``[E, fusion*I, H/pack]`` uint8, ``pack = 8/bits``
* ``fc1_s``  ``[E, fusion*I, H/bs]`` (``bs > 0``) or ``[E, fusion*I]`` (``bs == 0``)
* ``fc2_w``  ``[E, H, I/pack]`` uint8, scales ``[E, H, I/bs]`` or ``[E, H]``
* ``fc3_w``  ``[E, I, H/pack]`` uint8 (optional), scales likewise
* biases ``[E, rows]`` in the activation dtype (optional)
* ``x`` ``[T, H]``, ``router_logits`` ``[T, E]``, ``shared`` ``[T, H]``

bf16 tensors are carried as ``np.uint16`` bit patterns, fp32 ones as
``np.float32``. Packed weight bytes are drawn uniformly over 0..255, so every
nibble (int4) or byte (int8) code is uniform over its range whatever order the
two nibbles of a byte are read in.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

ACT_RELU, ACT_GELU, ACT_SILU, ACT_SWIGLU, ACT_IDENTITY = 0, 1, 2, 3, 4
DT_F32, DT_BF16, DT_E8M0 = 0, 1, 2
WEIGHTS_INT, WEIGHTS_MXFP4 = 0, 1
COMPUTE_FLOAT, COMPUTE_INT8_BLOCK = 0, 1
ACT_NAMES = {"relu": ACT_RELU, "gelu": ACT_GELU, "silu": ACT_SILU,
             "swiglu": ACT_SWIGLU, "identity": ACT_IDENTITY}


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); return bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounding = 0x7FFF + ((u >> 16) & 1)
    return ((u + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass
class MoEConfig:
    """Counts and attributes of one QMoE operator instance."""
    T: int
    H: int
    I: int
    E: int
    k: int
    bits: int = 4
    block_size: int = 0
    act: int = ACT_SWIGLU
    fusion: int = 1
    alpha: float = 0.0
    beta: float = 0.0
    limit: float = math.inf
    normalize: bool = True
    act_dtype: int = DT_BF16
    scale_dtype: int = DT_BF16
    has_fc1_bias: bool = False
    has_fc2_bias: bool = False
    has_fc3: bool = False
    has_fc3_bias: bool = False
    has_shared: bool = False
    # routing options of the MoE page: grouped top-k (n_group <= 1: none),
    # scaling of the routed sum (0 reads as 1), router weight on the input
    n_group: int = 0
    topk_group: int = 0
    routed_scaling_factor: float = 1.0
    apply_router_weight_on_input: bool = False
    # WEIGHTS_MXFP4: e2m1 codes with one E8M0 scale byte per 32 codes
    weight_format: int = WEIGHTS_INT
    # COMPUTE_INT8_BLOCK: the activations are rounded per K block to int8
    compute_mode: int = COMPUTE_FLOAT
    # MoE page options: a multiplier of every expert output (0 reads as 1)
    # and the GELU form (0 erf, 1 tanh); set_weights' e_score_correction_bias
    # ([E] fp32, drawn when has_score_bias)
    expert_output_scale: float = 1.0
    gelu_mode: int = 0
    has_score_bias: bool = False

    @property
    def gated(self) -> bool:
        return self.fusion in (1, 2) or self.has_fc3

    @property
    def n1(self) -> int:
        """Rows of fc1: fusion_size * inter_size."""
        return (2 if self.fusion in (1, 2) else 1) * self.I


@dataclasses.dataclass
class MoEInputs:
    cfg: MoEConfig
    x: np.ndarray
    logits: np.ndarray
    fc1_w: np.ndarray
    fc1_s: np.ndarray
    fc2_w: np.ndarray
    fc2_s: np.ndarray
    fc1_b: Optional[np.ndarray] = None
    fc2_b: Optional[np.ndarray] = None
    fc3_w: Optional[np.ndarray] = None
    fc3_s: Optional[np.ndarray] = None
    fc3_b: Optional[np.ndarray] = None
    shared: Optional[np.ndarray] = None
    score_bias: Optional[np.ndarray] = None   # [E] float32


def _store(a: np.ndarray, dtype: int) -> np.ndarray:
    a = np.asarray(a, dtype=np.float32)
    return f32_to_bf16_bits(a) if dtype == DT_BF16 else np.ascontiguousarray(a)


def _weights(rng, E, N, K, bits):
    return rng.integers(0, 256, size=(E, N, K * bits // 8), dtype=np.uint8)


def _scales(rng, cfg: MoEConfig, E, N, K, exact_range: bool):
    shape = (E, N, K // cfg.block_size) if cfg.block_size > 0 else (E, N)
    if cfg.weight_format == WEIGHTS_MXFP4:
        # E8M0 exponent bytes around 0.05 * sqrt(64 / K) / 2 (e2m1 magnitudes
        # average about 2), spread over four powers of two
        centre = 127 + int(round(math.log2(0.025 * math.sqrt(64.0 / K))))
        return rng.integers(centre - 2, centre + 2, size=shape, dtype=np.int64).astype(np.uint8)
    s = rng.uniform(0.01, 0.05, size=shape)
    if not exact_range:
        # keep activations O(1): sqrt(64/K) for the reduction length and
        # 8/2^(bits-1) so int8 codes (|q-z| <= 128) match int4 magnitudes
        s = s * math.sqrt(64.0 / K) * (8.0 / 2 ** (cfg.bits - 1))
    return _store(s, cfg.scale_dtype)


def zipf_gumbel_logits(rng, T: int, E: int, s: float) -> np.ndarray:
    """Logits whose top-1 expert follows a Zipf(s) law over a seeded ranking.

    ``l[t, e] = log(pi_rank(e)) + Gumbel(0, 1)`` with ``pi_r ~ r^-s``; the
    Gumbel-max property makes the argmax distributed exactly as ``pi``.
    """
    ranks = rng.permutation(E) + 1
    pi = ranks.astype(np.float64) ** (-s)
    pi /= pi.sum()
    return np.log(pi)[None, :] + rng.gumbel(0.0, 1.0, size=(T, E))


def make_inputs(cfg: MoEConfig, seed: int, logits: str = "normal",
                logit_std: float = 1.0, tiny_scales: bool = False,
                bias_std: float = 0.02) -> MoEInputs:
    """Draw one seeded input set for ``cfg``.

    ``logits`` is ``"normal"`` (N(0, logit_std)), ``"uniform"`` (U(0,1)) or
    ``"zipf"`` (Zipf s=1.1 over experts via Gumbel-max).
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    T, H, I, E = cfg.T, cfg.H, cfg.I, cfg.E
    x = _store(rng.standard_normal((T, H)), cfg.act_dtype)
    if logits == "normal":
        lg = rng.standard_normal((T, E)) * logit_std
    elif logits == "uniform":
        lg = rng.uniform(0.0, 1.0, size=(T, E))
    elif logits == "zipf":
        lg = zipf_gumbel_logits(rng, T, E, 1.1)
    else:
        raise ValueError(logits)
    lg = _store(lg, cfg.act_dtype)
    n1 = cfg.n1
    fc1_w = _weights(rng, E, n1, H, cfg.bits)
    fc1_s = _scales(rng, cfg, E, n1, H, tiny_scales)
    fc2_w = _weights(rng, E, H, I, cfg.bits)
    fc2_s = _scales(rng, cfg, E, H, I, tiny_scales)
    inp = MoEInputs(cfg, x, lg, fc1_w, fc1_s, fc2_w, fc2_s)
    if cfg.has_fc3:
        inp.fc3_w = _weights(rng, E, I, H, cfg.bits)
        inp.fc3_s = _scales(rng, cfg, E, I, H, tiny_scales)
    if cfg.has_fc1_bias:
        inp.fc1_b = _store(rng.standard_normal((E, n1)) * bias_std, cfg.act_dtype)
    if cfg.has_fc2_bias:
        inp.fc2_b = _store(rng.standard_normal((E, H)) * bias_std, cfg.act_dtype)
    if cfg.has_fc3 and cfg.has_fc3_bias:
        inp.fc3_b = _store(rng.standard_normal((E, I)) * bias_std, cfg.act_dtype)
    if cfg.has_shared:
        inp.shared = _store(rng.standard_normal((T, H)), cfg.act_dtype)
    if cfg.has_score_bias:
        inp.score_bias = (rng.standard_normal(E) * 0.5).astype(np.float32)
    return inp


def make_token_batch(cfg: MoEConfig, seed: int, logits: str = "normal",
                     logit_std: float = 1.0, **_unused):
    """Draw only the per-token tensors ``(x, router_logits, shared)`` for
    ``cfg`` from their own seeded generator, with the same distributions as
    :func:`make_inputs` (``shared`` is None unless ``cfg.has_shared``)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    T, H, E = cfg.T, cfg.H, cfg.E
    x = _store(rng.standard_normal((T, H)), cfg.act_dtype)
    if logits == "normal":
        lg = rng.standard_normal((T, E)) * logit_std
    elif logits == "uniform":
        lg = rng.uniform(0.0, 1.0, size=(T, E))
    elif logits == "zipf":
        lg = zipf_gumbel_logits(rng, T, E, 1.1)
    else:
        raise ValueError(logits)
    shared = _store(rng.standard_normal((T, H)), cfg.act_dtype) if cfg.has_shared else None
    return x, _store(lg, cfg.act_dtype), shared


# ---------------------------------------------------------------------------
# Named workloads. Each is (config, seed, generator keyword arguments).
# ---------------------------------------------------------------------------

def tiny():
    cfg = MoEConfig(T=16, H=64, I=128, E=4, k=2, bits=4, block_size=32,
                    act=ACT_SWIGLU, fusion=1, limit=math.inf, normalize=True,
                    act_dtype=DT_F32, scale_dtype=DT_F32)
    return cfg, 1, dict(logits="normal", logit_std=1.0, tiny_scales=True)


def tiny_i8():
    """The tiny shape on the int8 block compute tier (64-code blocks)."""
    cfg = MoEConfig(T=16, H=128, I=128, E=4, k=2, bits=4, block_size=64,
                    act=ACT_SWIGLU, fusion=1, limit=math.inf, normalize=True,
                    act_dtype=DT_F32, scale_dtype=DT_F32, compute_mode=COMPUTE_INT8_BLOCK)
    return cfg, 6, dict(logits="normal", logit_std=1.0, tiny_scales=True)


def mixtral_decode(T: int = 8):
    cfg = MoEConfig(T=T, H=4096, I=14336, E=8, k=2, bits=4, block_size=128,
                    act=ACT_SWIGLU, fusion=2, normalize=True,
                    act_dtype=DT_BF16, scale_dtype=DT_BF16)
    return cfg, 2, dict(logits="normal", logit_std=2.0)


def gpt_oss(T: int = 1024):
    cfg = MoEConfig(T=T, H=2880, I=2880, E=32, k=4, bits=4, block_size=32,
                    act=ACT_SWIGLU, fusion=1, alpha=1.702, beta=1.0, limit=7.0,
                    normalize=True, act_dtype=DT_BF16, scale_dtype=DT_BF16,
                    has_fc1_bias=True, has_fc2_bias=True)
    return cfg, 3, dict(logits="normal", logit_std=1.0)


def gpt_oss_mxfp4(T: int = 1024):
    """The gpt-oss-like shape with MXFP4 expert weights (e2m1 codes, one E8M0
    scale per 32), the checkpoint format the QMoEWoQ page names."""
    cfg = MoEConfig(T=T, H=2880, I=2880, E=32, k=4, bits=4, block_size=32,
                    act=ACT_SWIGLU, fusion=1, alpha=1.702, beta=1.0, limit=7.0,
                    normalize=True, act_dtype=DT_BF16, scale_dtype=DT_E8M0,
                    has_fc1_bias=True, has_fc2_bias=True, weight_format=WEIGHTS_MXFP4)
    return cfg, 5, dict(logits="normal", logit_std=1.0)


def mixtral_decode_i8(T: int = 8):
    """The decode shape of mixtral_decode on the int8 block compute tier."""
    cfg, seed, kw = mixtral_decode(T)
    cfg.compute_mode = COMPUTE_INT8_BLOCK
    return cfg, seed, kw


def deepseek(T: int = 4096):
    cfg = MoEConfig(T=T, H=2048, I=1408, E=64, k=6, bits=8, block_size=0,
                    act=ACT_SILU, fusion=0, has_fc3=True, normalize=False,
                    act_dtype=DT_BF16, scale_dtype=DT_BF16, has_shared=True)
    return cfg, 4, dict(logits="zipf")


SWEEP_T = (1, 16, 128, 1024, 8192)


def sweep(bits: int, T: int):
    bs = 64 if bits == 4 else 128
    cfg = MoEConfig(T=T, H=4096, I=14336, E=8, k=2, bits=bits, block_size=bs,
                    act=ACT_SWIGLU, fusion=2, normalize=True,
                    act_dtype=DT_BF16, scale_dtype=DT_BF16)
    seed = (10 if bits == 4 else 20) + SWEEP_T.index(T)
    return cfg, seed, dict(logits="uniform")


WORKLOADS = {
    "tiny": tiny,
    "tiny_i8": tiny_i8,
    "mixtral_decode": mixtral_decode,
    "mixtral_decode_i8": mixtral_decode_i8,
    "gpt_oss": gpt_oss,
    "gpt_oss_mxfp4": gpt_oss_mxfp4,
    "deepseek": deepseek,
}


def workload(name: str, **kw):
    """Return ``(cfg, seed, gen_kwargs)`` for a named workload."""
    if name.startswith("sweep_i8tier_int"):
        # sweep_i8tier_int4_T1024: the sweep shape on the int8 block compute tier
        bits = int(name[len("sweep_i8tier_int")])
        cfg, seed, gkw = sweep(bits, int(name.split("_T")[1]))
        cfg.compute_mode = COMPUTE_INT8_BLOCK
        return cfg, seed, gkw
    if name.startswith("sweep_int"):
        # sweep_int4_T128
        bits = int(name[len("sweep_int")])
        T = int(name.split("_T")[1])
        return sweep(bits, T)
    return WORKLOADS[name](**kw)


def make_workload(name: str, **kw) -> MoEInputs:
    cfg, seed, gkw = workload(name, **kw)
    return make_inputs(cfg, seed, **gkw)
