"""Seeded synthetic inputs for the gated delta rule.

This module only draws random numbers and rounds them to the storage dtype; it
holds none of the method's arithmetic, and it is the one module that both the
CUDA path's callers and the CPU oracle's callers share.

Named workloads (sizes and value distributions of the problem statement):

==============  ==========================================================
tiny_fp32       B=1, H=2, T=256, d_k=d_v=64, chunk 64, fp32, S0 = 0
gdn_prefill     B=4, H=16, T=4096, d=128, bf16, scalar gate, S0 ~ N(0, 0.01)
kda_prefill     B=2, H=32, T=8192, d=128, bf16, per-channel gate, S0 = 0
decode          N=256 sequences, H=32, d=128, bf16 tokens, fp32 state
                S ~ N(0, 0.1), 1000 steps
varlen_prefill  16 packed sequences, sum T = 65536, lengths uniform in
                [1024, 7168], H=16, d=128, bf16, scalar gate, S0 = 0
gdp_prefill     Gated DeltaProduct, n_h = 2 substeps per token: B=4, H=16,
                T=2048 (4096 virtual steps), d=128, bf16, scalar gate,
                S0 ~ N(0, 0.01)
frame_prefill   implicit frame-level update: B=1, H=16, 16 frames of n=1024
                tokens (T=16384), d=128, bf16, per-channel decay per frame,
                writing strength gamma = (d_k / n) e^z, z ~ N(0, 1)
gdn2_prefill    Gated DeltaNet-2 (erase gate b per key channel, write gate w
                per value channel, b, w = sigmoid(N(0, 1))): B=2, H=16,
                T=4096, d=128, bf16, per-channel decay, S0 = 0
==============  ==========================================================

N(0, x) is read as mean 0, variance x.  Draw order for prefill: q, k, v,
beta logits, gate noise, S0, then sequence lengths.  q and k are Gaussian,
L2-normalised per token; v ~ N(0, 1); beta = sigmoid(N(0, 1)); the log-decay
g = -softplus(N(0, 1)) * gate_scale.  All draws are fp32 from numpy's PCG64,
then rounded (round-to-nearest-even) to the storage dtype, so the arrays
returned hold exactly the values the device sees.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

BASE_SEED = 20261202


@dataclasses.dataclass(frozen=True)
class PrefillConfig:
    name: str
    B: int
    T: int
    H: int
    d_k: int
    d_v: int
    chunk: int
    dtype: str            # "bf16" or "f32": storage of q, k, v and out
    gate: str             # "scalar" or "channel"
    gate_scale: float     # g = -softplus(N(0,1)) * gate_scale
    s0_var: float         # 0 -> S0 = 0 (None); else S0 ~ N(0, s0_var)
    n_seq: int = 0        # > 0: packed variable-length batch (B = 1)
    len_lo: int = 0
    len_hi: int = 0
    seed_index: int = 0
    n_h: int = 1          # Householder substeps per token (> 1: Gated DeltaProduct)
    variant: str = ""     # "gdn2": Gated DeltaNet-2 (erase and write gates instead of beta)

    @property
    def tokens(self) -> int:
        return self.B * self.T

    def replace(self, **kw) -> "PrefillConfig":
        return dataclasses.replace(self, **kw)


@dataclasses.dataclass(frozen=True)
class DecodeConfig:
    name: str
    N: int
    H: int
    d_k: int
    d_v: int
    dtype: str
    gate: str
    gate_scale: float
    s_var: float
    steps: int
    seed_index: int = 3

    def replace(self, **kw) -> "DecodeConfig":
        return dataclasses.replace(self, **kw)


PREFILL = {
    "tiny_fp32": PrefillConfig("tiny_fp32", 1, 256, 2, 64, 64, 64, "f32", "scalar", 0.1, 0.0,
                               seed_index=0),
    "gdn_prefill": PrefillConfig("gdn_prefill", 4, 4096, 16, 128, 128, 64, "bf16", "scalar", 0.1,
                                 0.01, seed_index=1),
    "kda_prefill": PrefillConfig("kda_prefill", 2, 8192, 32, 128, 128, 64, "bf16", "channel", 0.05,
                                 0.0, seed_index=2),
    "varlen_prefill": PrefillConfig("varlen_prefill", 1, 65536, 16, 128, 128, 64, "bf16", "scalar",
                                    0.1, 0.0, n_seq=16, len_lo=1024, len_hi=7168, seed_index=4),
    "gdp_prefill": PrefillConfig("gdp_prefill", 4, 2048, 16, 128, 128, 64, "bf16", "scalar", 0.1,
                                 0.01, seed_index=5, n_h=2),
    "gdn2_prefill": PrefillConfig("gdn2_prefill", 2, 4096, 16, 128, 128, 64, "bf16", "channel", 0.05,
                                  0.0, seed_index=6, variant="gdn2"),
    # the Gated DeltaNet and per-channel workloads at the other chunk sizes
    # (16: tensor cores; 128: CUDA cores)
    "gdn_prefill_c16": PrefillConfig("gdn_prefill_c16", 4, 4096, 16, 128, 128, 16, "bf16",
                                     "scalar", 0.1, 0.01, seed_index=1),
    "kda_prefill_c16": PrefillConfig("kda_prefill_c16", 2, 8192, 32, 128, 128, 16, "bf16",
                                     "channel", 0.05, 0.0, seed_index=2),
    "gdn_prefill_c128": PrefillConfig("gdn_prefill_c128", 4, 4096, 16, 128, 128, 128, "bf16",
                                      "scalar", 0.1, 0.01, seed_index=1),
}
DECODE = {
    "decode": DecodeConfig("decode", 256, 32, 128, 128, "bf16", "scalar", 0.1, 0.1, 1000),
    # the same step with the per-key-channel (KDA) decay
    "kda_decode": DecodeConfig("kda_decode", 256, 32, 128, 128, "bf16", "channel", 0.05, 0.1,
                               1000, seed_index=8),
}


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round fp32 values to ``dtype`` (``bf16`` by round-to-nearest-even on
    the bit pattern, ``f32`` unchanged); returns fp32 holding the rounded
    values."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "f32":
        return x
    if dtype != "bf16":
        raise ValueError(dtype)
    bits = x.view(np.uint32).astype(np.uint64)
    bits = (bits + 0x7FFF + ((bits >> 16) & 1)) >> 16
    return (bits.astype(np.uint32) << 16).view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The upper 16 bits of fp32 values that are already bf16-representable."""
    return (np.ascontiguousarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _l2_rows(x: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1, keepdims=True))
    return (x / n).astype(np.float32)


def _softplus(x: np.ndarray) -> np.ndarray:
    return np.logaddexp(0.0, x.astype(np.float64)).astype(np.float32)


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return (1.0 / (1.0 + np.exp(-x.astype(np.float64)))).astype(np.float32)


def varlen_lengths(rng: np.random.Generator, n_seq: int, total: int, lo: int, hi: int) -> np.ndarray:
    """n_seq - 1 lengths uniform in [lo, hi]; the last one takes the
    remainder and the draw repeats (same generator) until it is in range."""
    for _ in range(100000):
        head = rng.integers(lo, hi + 1, size=n_seq - 1)
        last = total - int(head.sum())
        if lo <= last <= hi:
            return np.concatenate([head, [last]]).astype(np.int64)
    raise RuntimeError("could not draw sequence lengths")


@dataclasses.dataclass
class PrefillInputs:
    cfg: PrefillConfig
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    g: np.ndarray
    beta: np.ndarray
    S0: Optional[np.ndarray]
    cu_seqlens: Optional[np.ndarray]

    @property
    def n_seq(self) -> int:
        return self.cfg.B if self.cu_seqlens is None else len(self.cu_seqlens) - 1


def prefill_inputs(cfg: PrefillConfig, seed: Optional[int] = None,
                   s0_var: Optional[float] = None) -> PrefillInputs:
    """Draw one prefill batch for ``cfg`` (seed defaults to the workload's)."""
    if seed is None:
        seed = BASE_SEED + cfg.seed_index
    rng = np.random.default_rng(seed)
    B, T, H, dk, dv = cfg.B, cfg.T, cfg.H, cfg.d_k, cfg.d_v
    f32 = np.float32
    q = _l2_rows(rng.standard_normal((B, T, H, dk), dtype=f32))
    k = _l2_rows(rng.standard_normal((B, T, H, dk), dtype=f32))
    v = rng.standard_normal((B, T, H, dv), dtype=f32)
    beta = _sigmoid(rng.standard_normal((B, T, H), dtype=f32))
    gshape = (B, T, H, dk) if cfg.gate == "channel" else (B, T, H)
    g = (-_softplus(rng.standard_normal(gshape, dtype=f32)) * f32(cfg.gate_scale)).astype(f32)
    n_seq = cfg.n_seq if cfg.n_seq > 0 else B
    var = cfg.s0_var if s0_var is None else s0_var
    S0 = None
    if var > 0:
        S0 = (rng.standard_normal((n_seq, H, dv, dk), dtype=f32) * f32(np.sqrt(var))).astype(f32)
    cu = None
    if cfg.n_seq > 0:
        if B != 1:
            raise ValueError("packed batches have B = 1")
        lens = varlen_lengths(rng, cfg.n_seq, T, cfg.len_lo, cfg.len_hi)
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return PrefillInputs(cfg, round_to(q, cfg.dtype), round_to(k, cfg.dtype),
                         round_to(v, cfg.dtype), g, beta, S0, cu)


def product_inputs(cfg: PrefillConfig, seed: Optional[int] = None,
                   s0_var: Optional[float] = None) -> PrefillInputs:
    """Draw one Gated DeltaProduct batch: as :func:`prefill_inputs`, with k
    ``[B, T, n_h, H, d_k]``, v ``[B, T, n_h, H, d_v]`` and beta
    ``[B, T, n_h, H]`` (one key, value and step size per substep); q and g stay
    one per token.  Same draw order, each substep's k normalised on its own."""
    if seed is None:
        seed = BASE_SEED + cfg.seed_index
    rng = np.random.default_rng(seed)
    B, T, H, dk, dv, nh = cfg.B, cfg.T, cfg.H, cfg.d_k, cfg.d_v, cfg.n_h
    f32 = np.float32
    q = _l2_rows(rng.standard_normal((B, T, H, dk), dtype=f32))
    k = _l2_rows(rng.standard_normal((B, T, nh, H, dk), dtype=f32))
    v = rng.standard_normal((B, T, nh, H, dv), dtype=f32)
    beta = _sigmoid(rng.standard_normal((B, T, nh, H), dtype=f32))
    gshape = (B, T, H, dk) if cfg.gate == "channel" else (B, T, H)
    g = (-_softplus(rng.standard_normal(gshape, dtype=f32)) * f32(cfg.gate_scale)).astype(f32)
    n_seq = cfg.n_seq if cfg.n_seq > 0 else B
    var = cfg.s0_var if s0_var is None else s0_var
    S0 = None
    if var > 0:
        S0 = (rng.standard_normal((n_seq, H, dv, dk), dtype=f32) * f32(np.sqrt(var))).astype(f32)
    cu = None
    if cfg.n_seq > 0:
        if B != 1:
            raise ValueError("packed batches have B = 1")
        lens = varlen_lengths(rng, cfg.n_seq, T, cfg.len_lo, cfg.len_hi)
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return PrefillInputs(cfg, round_to(q, cfg.dtype), round_to(k, cfg.dtype),
                         round_to(v, cfg.dtype), g, beta, S0, cu)


@dataclasses.dataclass
class Gdn2Inputs:
    cfg: PrefillConfig
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    g: np.ndarray
    b: np.ndarray          # erase gate [B, T, H, d_k]
    w: np.ndarray          # write gate [B, T, H, d_v]
    S0: Optional[np.ndarray]
    cu_seqlens: Optional[np.ndarray]

    @property
    def n_seq(self) -> int:
        return self.cfg.B if self.cu_seqlens is None else len(self.cu_seqlens) - 1


def gdn2_inputs(cfg: PrefillConfig, seed: Optional[int] = None,
                s0_var: Optional[float] = None) -> Gdn2Inputs:
    """Draw one Gated DeltaNet-2 batch: as :func:`prefill_inputs`, with the
    scalar beta replaced by an erase gate b (per key channel) and a write gate
    w (per value channel), each sigmoid(N(0, 1)).  Draw order: q, k, v, b
    logits, w logits, gate noise, S0, lengths."""
    if seed is None:
        seed = BASE_SEED + cfg.seed_index
    rng = np.random.default_rng(seed)
    B, T, H, dk, dv = cfg.B, cfg.T, cfg.H, cfg.d_k, cfg.d_v
    f32 = np.float32
    q = _l2_rows(rng.standard_normal((B, T, H, dk), dtype=f32))
    k = _l2_rows(rng.standard_normal((B, T, H, dk), dtype=f32))
    v = rng.standard_normal((B, T, H, dv), dtype=f32)
    b = _sigmoid(rng.standard_normal((B, T, H, dk), dtype=f32))
    w = _sigmoid(rng.standard_normal((B, T, H, dv), dtype=f32))
    gshape = (B, T, H, dk) if cfg.gate == "channel" else (B, T, H)
    g = (-_softplus(rng.standard_normal(gshape, dtype=f32)) * f32(cfg.gate_scale)).astype(f32)
    n_seq = cfg.n_seq if cfg.n_seq > 0 else B
    var = cfg.s0_var if s0_var is None else s0_var
    S0 = None
    if var > 0:
        S0 = (rng.standard_normal((n_seq, H, dv, dk), dtype=f32) * f32(np.sqrt(var))).astype(f32)
    cu = None
    if cfg.n_seq > 0:
        if B != 1:
            raise ValueError("packed batches have B = 1")
        lens = varlen_lengths(rng, cfg.n_seq, T, cfg.len_lo, cfg.len_hi)
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return Gdn2Inputs(cfg, round_to(q, cfg.dtype), round_to(k, cfg.dtype), round_to(v, cfg.dtype),
                      g, b, w, S0, cu)


@dataclasses.dataclass(frozen=True)
class FrameConfig:
    name: str
    B: int
    T: int
    H: int
    d_k: int
    d_v: int
    n: int                # tokens per frame
    dtype: str
    gate: str             # "scalar" or "channel" (one decay per frame)
    gate_scale: float
    s0_var: float
    seed_index: int = 7

    @property
    def frames(self) -> int:
        return (self.T + self.n - 1) // self.n

    def replace(self, **kw) -> "FrameConfig":
        return dataclasses.replace(self, **kw)


FRAME = {
    "frame_prefill": FrameConfig("frame_prefill", 1, 16384, 16, 128, 128, 1024, "bf16", "channel",
                                 0.05, 0.0),
}


@dataclasses.dataclass
class FrameInputs:
    cfg: FrameConfig
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    g: np.ndarray          # per frame [B, F, H] or [B, F, H, d_k]
    gamma: np.ndarray      # per token [B, T, H]
    S0: Optional[np.ndarray]


def frame_inputs(cfg: FrameConfig, seed: Optional[int] = None,
                 s0_var: Optional[float] = None) -> FrameInputs:
    """Draw one batch for the implicit frame-level update.  Draw order: q, k, v,
    writing-strength logits z, gate noise, S0.  gamma = (d_k / n) e^z: the
    page's overall scale s = d_k / n, at which the old state and a frame take
    about half each."""
    if seed is None:
        seed = BASE_SEED + cfg.seed_index
    rng = np.random.default_rng(seed)
    B, T, H, dk, dv = cfg.B, cfg.T, cfg.H, cfg.d_k, cfg.d_v
    f32 = np.float32
    q = _l2_rows(rng.standard_normal((B, T, H, dk), dtype=f32))
    k = _l2_rows(rng.standard_normal((B, T, H, dk), dtype=f32))
    v = rng.standard_normal((B, T, H, dv), dtype=f32)
    z = rng.standard_normal((B, T, H), dtype=f32)
    gamma = (np.exp(z.astype(np.float64)) * (dk / cfg.n)).astype(f32)
    F = cfg.frames
    gshape = (B, F, H, dk) if cfg.gate == "channel" else (B, F, H)
    g = (-_softplus(rng.standard_normal(gshape, dtype=f32)) * f32(cfg.gate_scale)).astype(f32)
    var = cfg.s0_var if s0_var is None else s0_var
    S0 = None
    if var > 0:
        S0 = (rng.standard_normal((B, H, dv, dk), dtype=f32) * f32(np.sqrt(var))).astype(f32)
    return FrameInputs(cfg, round_to(q, cfg.dtype), round_to(k, cfg.dtype), round_to(v, cfg.dtype),
                       g, gamma, S0)


@dataclasses.dataclass
class DecodeInputs:
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    g: np.ndarray
    beta: np.ndarray


def decode_state(cfg: DecodeConfig, seed: Optional[int] = None) -> np.ndarray:
    """Initial decode state S ~ N(0, s_var), fp32 [N, H, d_v, d_k]."""
    if seed is None:
        seed = BASE_SEED + cfg.seed_index
    rng = np.random.default_rng([seed, 0x5])
    S = rng.standard_normal((cfg.N, cfg.H, cfg.d_v, cfg.d_k), dtype=np.float32)
    return (S * np.float32(np.sqrt(cfg.s_var))).astype(np.float32)


def decode_token(cfg: DecodeConfig, step: int, seed: Optional[int] = None) -> DecodeInputs:
    """The new token of every sequence at decode step ``step`` (regenerated
    from (seed, step), so any step can be redrawn on its own)."""
    if seed is None:
        seed = BASE_SEED + cfg.seed_index
    rng = np.random.default_rng([seed, 0x7, step])
    N, H, dk, dv = cfg.N, cfg.H, cfg.d_k, cfg.d_v
    f32 = np.float32
    q = _l2_rows(rng.standard_normal((N, H, dk), dtype=f32))
    k = _l2_rows(rng.standard_normal((N, H, dk), dtype=f32))
    v = rng.standard_normal((N, H, dv), dtype=f32)
    beta = _sigmoid(rng.standard_normal((N, H), dtype=f32))
    gshape = (N, H, dk) if cfg.gate == "channel" else (N, H)
    g = (-_softplus(rng.standard_normal(gshape, dtype=f32)) * f32(cfg.gate_scale)).astype(f32)
    return DecodeInputs(round_to(q, cfg.dtype), round_to(k, cfg.dtype), round_to(v, cfg.dtype),
                        g, beta)
