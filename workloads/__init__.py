"""Seeded synthetic inputs for the five attention workloads.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests. It draws random numbers and rounds them to the storage dtype;
it holds none of the quantized-attention arithmetic.

Recipe (all draws are numpy ``default_rng`` float32 normals, rounded with
round-to-nearest-even to the config's dtype):

* Per-(kv head, channel) K gains ``g``: ``lognormal(0, sigma)`` from the model
  seed, or 1 when the config has no gains.
* Outlier channels: a fixed channel list (tiny config) or ``round(frac * D)``
  distinct channels per kv head drawn from the model seed; their gain is
  multiplied by ``outlier_factor``.
* Q, K, V: standard normal. K is multiplied by its gains before rounding.
  Each (batch, head) slice has its own seed so any slice can be regenerated on
  its own (the oracle only ever needs the slices it samples).
* Calibration batch: 512 fresh tokens (batch 1) from the calibration seed, same
  gains and outlier channels as the evaluation tensors.

Seeds: model = 1000 + i, data = i, calibration = 100 + i for config i = 1..5.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

__all__ = ["Config", "CONFIGS", "get", "k_gains", "q_slice", "k_slice", "rope_tables",
           "v_slice", "qcal_slice", "kcal_slice", "full", "calib_full",
           "round_to_dtype", "to_bits"]

_KIND = {"q": 1, "k": 2, "v": 3, "qcal": 4, "kcal": 5}


@dataclass(frozen=True)
class Config:
    index: int
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nkv: int
    D: int
    causal: bool
    dtype: str                      # "fp16" or "bf16"
    gain_sigma: float | None        # lognormal sigma of the K channel gains
    outlier_channels: tuple | None  # fixed outlier channels (same for every kv head)
    outlier_frac: float             # else: fraction of channels per kv head
    outlier_factor: float
    smooth: str                     # "self" (from the tensors), "calib" (512-token batch) or "off"
    alpha: float = 0.5
    calib_tokens: int = 512
    modes: tuple = ("p_reorder",)
    desc: str = ""

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def seed_model(self) -> int:
        return 1000 + self.index

    @property
    def seed_data(self) -> int:
        return self.index

    @property
    def seed_calib(self) -> int:
        return 100 + self.index

    def flops(self) -> float:
        """Algorithmic attention FLOPs: 4*B*Hq*Nq*Nkv*D, halved when causal."""
        f = 4.0 * self.B * self.Hq * self.Nq * self.Nkv * self.D
        return f / 2 if self.causal else f

    def replace(self, **kw) -> "Config":
        d = {k: getattr(self, k) for k in self.__dataclass_fields__}
        d.update(kw)
        return Config(**d)


CONFIGS = [
    Config(1, "tiny_h1_n256_d64", 1, 1, 1, 256, 256, 64, False, "fp16",
           None, (3, 17, 40, 61), 0.0, 20.0, "self",
           modes=("p_reorder", "high_precision_l"),
           desc="tiny single-head check, non-causal, fp16"),
    Config(2, "qwen3_8b_prefill_n4096", 1, 32, 8, 4096, 4096, 128, True, "bf16",
           1.0, None, 0.02, 15.0, "calib",
           modes=("p_reorder", "high_precision_l"),
           desc="Qwen3-8B-shaped causal prefill, GQA 32/8, D=128"),
    Config(3, "gemma2_9b_prefill_n8192", 1, 16, 8, 8192, 8192, 256, True, "bf16",
           0.5, None, 0.0, 1.0, "calib",
           desc="Gemma2-9B-shaped causal prefill, GQA 16/8, D=256"),
    Config(4, "llama31_8b_prefill_n16384", 2, 32, 8, 16384, 16384, 128, True, "bf16",
           1.0, None, 0.0, 1.0, "off",
           desc="Llama3.1-8B-shaped long causal prefill, Smooth-QK off"),
    Config(5, "decode_chunk_b64_q16_kv8192", 64, 32, 8, 16, 8192, 128, False, "bf16",
           None, None, 0.01, 10.0, "calib",
           modes=("p_reorder", "high_precision_l"),
           desc="batched decode-style chunk, 16 queries over 8192 cached keys"),
]


def get(i_or_name) -> Config:
    for c in CONFIGS:
        if c.index == i_or_name or c.name == i_or_name:
            return c
    raise KeyError(i_or_name)


def round_to_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values to bf16 / fp16 (nearest-even) and return them as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "fp16":
        return x.astype(np.float16).astype(np.float32)
    if dtype == "bf16":
        u = x.view(np.uint32)
        r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
        return r.view(np.float32)
    if dtype == "fp32":
        return x
    raise ValueError(dtype)


def to_bits(x: np.ndarray, dtype: str) -> np.ndarray:
    """Storage bits (uint16) of float32 values that are already exact in ``dtype``."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "fp16":
        return x.astype(np.float16).view(np.uint16)
    if dtype == "bf16":
        return (x.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    raise ValueError(dtype)


def _rng(*key) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(k) for k in key]))


def k_gains(cfg: Config) -> np.ndarray:
    """Per-(kv head, channel) K gains, float32 [Hkv, D], outliers included."""
    rng = _rng(cfg.seed_model, 7)
    if cfg.gain_sigma is None:
        g = np.ones((cfg.Hkv, cfg.D), np.float32)
    else:
        g = rng.lognormal(0.0, cfg.gain_sigma, size=(cfg.Hkv, cfg.D)).astype(np.float32)
    if cfg.outlier_channels is not None:
        g[:, list(cfg.outlier_channels)] *= np.float32(cfg.outlier_factor)
    elif cfg.outlier_frac > 0:
        n = int(round(cfg.outlier_frac * cfg.D))
        for h in range(cfg.Hkv):
            ch = rng.choice(cfg.D, size=n, replace=False)
            g[h, ch] *= np.float32(cfg.outlier_factor)
    return g


def _normal(seed, kind, b, h, n, d) -> np.ndarray:
    return _rng(seed, _KIND[kind], b, h).standard_normal((n, d), dtype=np.float32)


def q_slice(cfg: Config, b: int, h: int) -> np.ndarray:
    """Q[b, h] as float32 [Nq, D] holding exact dtype values."""
    return round_to_dtype(_normal(cfg.seed_data, "q", b, h, cfg.Nq, cfg.D), cfg.dtype)


def k_slice(cfg: Config, b: int, g: int, gains: np.ndarray | None = None) -> np.ndarray:
    if gains is None:
        gains = k_gains(cfg)
    x = _normal(cfg.seed_data, "k", b, g, cfg.Nkv, cfg.D) * gains[g][None, :]
    return round_to_dtype(x, cfg.dtype)


def v_slice(cfg: Config, b: int, g: int) -> np.ndarray:
    return round_to_dtype(_normal(cfg.seed_data, "v", b, g, cfg.Nkv, cfg.D), cfg.dtype)


def qcal_slice(cfg: Config, h: int) -> np.ndarray:
    return round_to_dtype(_normal(cfg.seed_calib, "qcal", 0, h, cfg.calib_tokens, cfg.D), cfg.dtype)


def kcal_slice(cfg: Config, g: int, gains: np.ndarray | None = None) -> np.ndarray:
    if gains is None:
        gains = k_gains(cfg)
    x = _normal(cfg.seed_calib, "kcal", 0, g, cfg.calib_tokens, cfg.D) * gains[g][None, :]
    return round_to_dtype(x, cfg.dtype)


def full(cfg: Config):
    """Full Q [B,Hq,Nq,D], K and V [B,Hkv,Nkv,D] as float32 (exact dtype values).

    Only for configs that fit comfortably in host memory; large configs are
    built slice by slice by the callers.
    """
    gains = k_gains(cfg)
    q = np.empty((cfg.B, cfg.Hq, cfg.Nq, cfg.D), np.float32)
    k = np.empty((cfg.B, cfg.Hkv, cfg.Nkv, cfg.D), np.float32)
    v = np.empty((cfg.B, cfg.Hkv, cfg.Nkv, cfg.D), np.float32)
    for b in range(cfg.B):
        for h in range(cfg.Hq):
            q[b, h] = q_slice(cfg, b, h)
        for g in range(cfg.Hkv):
            k[b, g] = k_slice(cfg, b, g, gains)
            v[b, g] = v_slice(cfg, b, g)
    return q, k, v


def calib_full(cfg: Config):
    """Calibration tensors (Qcal [1,Hq,T,D], Kcal [1,Hkv,T,D]) for the config's smoothing mode.

    ``smooth == "self"`` calibrates on the evaluation tensors themselves;
    ``"calib"`` on the separate 512-token batch; ``"off"`` returns None.
    """
    if cfg.smooth == "off":
        return None
    if cfg.smooth == "self":
        q, k, _ = full(cfg)
        return q, k
    gains = k_gains(cfg)
    qc = np.stack([qcal_slice(cfg, h) for h in range(cfg.Hq)])[None]
    kc = np.stack([kcal_slice(cfg, g, gains) for g in range(cfg.Hkv)])[None]
    return qc, kc


def rope_tables(n_pos: int, D: int, base: float = 10000.0):
    """Caller-side RoPE tables for the fused RoPE option: cos and sin of
    pos * base^(-2d/D) for d < D/2, evaluated in float64 and rounded to float32
    ([n_pos, D/2] each), the usual frequency schedule of rotary embeddings."""
    inv = base ** (-np.arange(0, D // 2, dtype=np.float64) * 2.0 / D)
    ang = np.arange(n_pos, dtype=np.float64)[:, None] * inv[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
