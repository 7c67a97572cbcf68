"""Seeded synthetic inputs for the MoE-layer forward, and the workload table.

This module is the only code shared by the CUDA path's tests/benchmark and the
CPU oracle.  It draws random numbers and shapes them onto value grids; it holds
none of the layer's arithmetic (no routing, no capacity, no expert math).

Workloads (sizes from the five MoE workloads the library is measured on):

  name              T      d     E    k   F      F_s   score          renorm scale  capacity factor
  c1_tiny          256     64    8    2   128    -     softmax        yes    1      1.25 (token-order drop)
  c2_handbook     8192   2048   64    8   1024   -     softmax        yes    1      none
  c3_fine_grained 16384  4096  256    8   512    2048  sigmoid+bias   yes    2.5    none
  c4_coarse       16384  4096    8    2   14336  -     softmax        yes    1      none
  c5_stress       32768  7168  896   16   256    -     sqrt(softplus) yes    1      1.0 (token-order drop)

Value grids (chosen so that every fp32 partial sum of the router dot product
is an exact multiple of a power of two below 2**24 grid units, hence exact in
any summation order):
  * bf16 workloads: x = round(8*N(0,1))/8 clipped to [-4, 4];
    Wg = round(1024*N(0,0.02))/1024 with the integer clipped to [-64, 64];
    |x*Wg| <= 2048 * 2**-13, so |sum| < 7168*2048 < 2**24 units of 2**-13.
    Per-expert logit offsets are rounded to the same 2**-13 grid.
    Expert weights: N(0,0.02) rounded to bf16 (no grid needed).
  * c1_tiny (fp32 everywhere): x = round(256*N(0,1))/256 clipped to [-4,4],
    every weight round(256*N(0,0.02))/256 with the integer clipped to [-32,32];
    |sum| <= 64*1024*32 = 2**21 units of 2**-16.
  * c3_fine_grained: per-expert logit offset N(0,0.5) (skews the load), and a
    selection-only bias U(-0.1, 0.1) in fp32.
  * c5_stress: Zipf(s=1.2) offset  o[e] = -1.2*ln(r_e), r a seeded random
    permutation of 1..E, so hotness is decoupled from the expert index.

Every tensor has its own random stream, numpy default_rng([seed, stream]); each
expert's weights have their own stream too, so any expert can be regenerated
alone and big weight sets can be generated in parallel.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, replace
from typing import Optional

import numpy as np

SCORES = ("softmax", "sigmoid", "sqrt_softplus")


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int
    d: int
    E: int
    k: int
    F: int
    F_s: int = 0                  # shared-expert width, 0 = no shared expert
    score: str = "softmax"
    renormalize: bool = True
    scale: float = 1.0
    capacity_factor: Optional[float] = None   # None = no dropping
    act: str = "bf16"             # "bf16" or "f32": activation/weight storage type
    logit_offset: Optional[str] = None        # None | "normal0.5" | "zipf1.2"
    select_bias: Optional[str] = None         # None | "uniform0.1"

    def with_(self, **kw) -> "MoEConfig":
        return replace(self, **kw)


CONFIGS = {
    "c1_tiny": MoEConfig("c1_tiny", T=256, d=64, E=8, k=2, F=128, score="softmax",
                         capacity_factor=1.25, act="f32"),
    "c2_handbook": MoEConfig("c2_handbook", T=8192, d=2048, E=64, k=8, F=1024,
                             score="softmax"),
    "c3_fine_grained": MoEConfig("c3_fine_grained", T=16384, d=4096, E=256, k=8, F=512,
                                 F_s=2048, score="sigmoid", scale=2.5,
                                 logit_offset="normal0.5", select_bias="uniform0.1"),
    "c4_coarse": MoEConfig("c4_coarse", T=16384, d=4096, E=8, k=2, F=14336,
                           score="softmax"),
    "c5_stress": MoEConfig("c5_stress", T=32768, d=7168, E=896, k=16, F=256,
                           score="sqrt_softplus", capacity_factor=1.0,
                           logit_offset="zipf1.2"),
}

# stream ids
_S_X, _S_WG, _S_OFF, _S_BIAS, _S_SHARED = 1, 2, 3, 4, 5
_S_WNOISE, _S_NOISE, _S_TOKEN_ID = 6, 7, 8
_S_EXPERT_BASE = 1000


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.default_rng([seed, stream])


def _to_bf16_values(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (torch's cast), returned as float32."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def gen_x(cfg: MoEConfig, seed: int = 0, T: Optional[int] = None) -> np.ndarray:
    T = cfg.T if T is None else T
    z = _rng(seed, _S_X).standard_normal((T, cfg.d), dtype=np.float32)
    if cfg.act == "f32":
        return np.clip(np.rint(z * 256.0), -1024, 1024).astype(np.float32) / 256.0
    return np.clip(np.rint(z * 8.0), -32, 32).astype(np.float32) / 8.0


def gen_router(cfg: MoEConfig, seed: int = 0):
    """Router weight Wg [d, E] fp32, logit offset [E] or None, selection bias [E] or None."""
    z = _rng(seed, _S_WG).standard_normal((cfg.d, cfg.E), dtype=np.float32) * 0.02
    if cfg.act == "f32":
        Wg = np.clip(np.rint(z * 256.0), -32, 32).astype(np.float32) / 256.0
    else:
        Wg = np.clip(np.rint(z * 1024.0), -64, 64).astype(np.float32) / 1024.0
    off = None
    if cfg.logit_offset == "normal0.5":
        o = _rng(seed, _S_OFF).standard_normal(cfg.E) * 0.5
        off = (np.rint(o * 8192.0) / 8192.0).astype(np.float32)
    elif cfg.logit_offset == "zipf1.2":
        r = _rng(seed, _S_OFF).permutation(cfg.E) + 1          # ranks 1..E
        o = -1.2 * np.log(r.astype(np.float64))
        off = (np.rint(o * 8192.0) / 8192.0).astype(np.float32)
    elif cfg.logit_offset is not None:
        raise ValueError(cfg.logit_offset)
    bias = None
    if cfg.select_bias == "uniform0.1":
        bias = _rng(seed, _S_BIAS).uniform(-0.1, 0.1, cfg.E).astype(np.float32)
    elif cfg.select_bias is not None:
        raise ValueError(cfg.select_bias)
    return Wg, off, bias


def gen_noise_router(cfg: MoEConfig, seed: int = 0) -> np.ndarray:
    """Noise-router weight W_noise [d, E] fp32 on the router's grid (exact fp32 logits)."""
    z = _rng(seed, _S_WNOISE).standard_normal((cfg.d, cfg.E), dtype=np.float32) * 0.02
    if cfg.act == "f32":
        return np.clip(np.rint(z * 256.0), -32, 32).astype(np.float32) / 256.0
    return np.clip(np.rint(z * 1024.0), -64, 64).astype(np.float32) / 1024.0


def gen_noise(cfg: MoEConfig, seed: int = 0, T: Optional[int] = None) -> np.ndarray:
    """Standard normal draws [T, E] fp32 for noisy top-k gating."""
    T = cfg.T if T is None else T
    return _rng(seed, _S_NOISE).standard_normal((T, cfg.E), dtype=np.float32)


def gen_token_ids(cfg: MoEConfig, seed: int = 0, T: Optional[int] = None, vocab: int = 32768,
                  s: float = 1.0) -> np.ndarray:
    """Token ids [T] int32 with text-like (Zipf) frequencies: rank r of the vocabulary drawn with
    probability proportional to r^-s, ranks mapped to ids by a seeded permutation."""
    T = cfg.T if T is None else T
    rng = _rng(seed, _S_TOKEN_ID)
    p = np.arange(1, vocab + 1, dtype=np.float64) ** -s
    ranks = rng.choice(vocab, size=T, p=p / p.sum())
    return rng.permutation(vocab)[ranks].astype(np.int32)


def _weights(cfg: MoEConfig, rng: np.random.Generator, shape) -> np.ndarray:
    z = rng.standard_normal(shape, dtype=np.float32) * 0.02
    if cfg.act == "f32":
        return np.clip(np.rint(z * 256.0), -32, 32).astype(np.float32) / 256.0
    return _to_bf16_values(z)


def gen_expert(cfg: MoEConfig, e: int, seed: int = 0):
    """Expert e's weights: W_gu [2F, d] (rows 0..F-1 gate, F..2F-1 up), W_dn [d, F]."""
    rng = _rng(seed, _S_EXPERT_BASE + e)
    W_gu = _weights(cfg, rng, (2 * cfg.F, cfg.d))
    W_dn = _weights(cfg, rng, (cfg.d, cfg.F))
    return W_gu, W_dn


def gen_shared(cfg: MoEConfig, seed: int = 0):
    """Shared expert weights W_gu [2F_s, d], W_dn [d, F_s], or None."""
    if cfg.F_s <= 0:
        return None
    rng = _rng(seed, _S_SHARED)
    return _weights(cfg, rng, (2 * cfg.F_s, cfg.d)), _weights(cfg, rng, (cfg.d, cfg.F_s))


def gen_experts(cfg: MoEConfig, seed: int = 0, threads: Optional[int] = None):
    """All experts stacked: W_gu [E, 2F, d], W_dn [E, d, F] (float32 arrays)."""
    W_gu = np.empty((cfg.E, 2 * cfg.F, cfg.d), np.float32)
    W_dn = np.empty((cfg.E, cfg.d, cfg.F), np.float32)

    def one(e):
        W_gu[e], W_dn[e] = gen_expert(cfg, e, seed)

    threads = threads or min(16, os.cpu_count() or 1)
    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(one, range(cfg.E)))
    return W_gu, W_dn


def gen_experts_torch(cfg: MoEConfig, seed: int = 0, threads: Optional[int] = None):
    """All experts as host torch tensors in the storage dtype (bf16 or fp32):
    W_gu [E, 2F, d], W_dn [E, d, F].  Same values as gen_expert(cfg, e, seed)."""
    import torch
    dt = torch.float32 if cfg.act == "f32" else torch.bfloat16
    W_gu = torch.empty((cfg.E, 2 * cfg.F, cfg.d), dtype=dt)
    W_dn = torch.empty((cfg.E, cfg.d, cfg.F), dtype=dt)

    def one(e):
        a, b = gen_expert(cfg, e, seed)
        W_gu[e].copy_(torch.from_numpy(a))      # values are already exact in dt
        W_dn[e].copy_(torch.from_numpy(b))

    threads = threads or min(16, os.cpu_count() or 1)
    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(one, range(cfg.E)))
    return W_gu, W_dn


def small_config(name: str = "small", **kw) -> MoEConfig:
    """A small bf16 configuration for quick tests (overridable)."""
    base = dict(name=name, T=300, d=128, E=16, k=4, F=128, score="softmax")
    base.update(kw)
    return MoEConfig(**base)


def fits_exact_fp32(cfg: MoEConfig) -> bool:
    """True when the router grid keeps every partial sum of x.Wg below 2**24 units."""
    if cfg.act == "f32":
        return cfg.d * 1024 * 32 < 2 ** 24
    return cfg.d * 32 * 64 + 8192 * 16 < 2 ** 24


__all__ = ["MoEConfig", "CONFIGS", "SCORES", "gen_x", "gen_router", "gen_expert", "gen_experts",
           "gen_shared", "gen_noise_router", "gen_noise", "gen_token_ids", "small_config", "fits_exact_fp32"]
