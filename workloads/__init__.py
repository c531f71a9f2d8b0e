"""Seeded synthetic workloads for the MoE layer forward.

This module only *generates inputs*: shapes, seeds and value distributions.
It holds none of the layer's arithmetic (no routing, no top-k, no dispatch, no
expert math), so both the CPU oracle and the CUDA library can take their
inputs from it without sharing any of the method.

Shapes follow the layers the pages name as shape donors (Qwen3-30B-A3B,
Qwen3-235B-A22B decode, gpt-oss-120b); no trained weights are used anywhere.

Recipe (all draws from ``torch.Generator`` on the requested device):

* ``x ~ N(0, 1)`` ``[T, d]``
* ``w_router ~ N(0, 0.02)`` ``[E, d]`` (the gate ``nn.Linear(d, E)`` weight,
  i.e. ``W_r^T`` of a ``W_r[d, E]``)
* ``w1, w3 ~ N(0, 1/sqrt(d))`` ``[E, h, d]``; ``w2 ~ N(0, 1/sqrt(h))``
  ``[E, d, h]`` -- the ``[out, in]`` stacked layout of the hyper_parallel
  ``GroupedExperts`` module; the second argument of ``N`` is the standard
  deviation, as in ``torch.nn.init.normal_``.
* values are drawn in fp32 and rounded once (round-to-nearest-even) to the
  layer dtype; the oracle reads the rounded values exactly.
* Zipf-skewed routing: a per-expert logit bias ``b_e = ln p_e`` with
  ``p_e`` proportional to ``rank(e)^-1.2`` under a seeded random ranking of the
  experts.  It is carried *inside* the router contraction: the last feature of
  every token is set to 1 and the last column of ``w_router`` to ``b_e``, so
  ``x . w_router[e] = (unbiased logit) + b_e`` and no bias argument is needed.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

__all__ = [
    "MoEConfig", "CONFIGS", "config", "make_layer", "make_logits",
    "make_rank_counts", "zipf_bias", "SEED_X", "SEED_WR", "SEED_W1",
    "SEED_W3", "SEED_W2",
]

# Per-tensor seed offsets: each tensor has its own stream, so any tensor can
# be regenerated alone.
SEED_X, SEED_WR, SEED_W1, SEED_W3, SEED_W2, SEED_BIAS, SEED_LOGITS = range(7)


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    dtype: str          # "f32" or "bf16"
    T: int
    d: int
    E: int
    top_k: int
    h: int
    seed: int
    renormalize: bool = True
    zipf_s: Optional[float] = None   # Zipf exponent of the routing skew, or None
    ep_ranks: int = 1                # simulated EP ranks (R == G); 1 = no regroup
    router_std: float = 0.02

    @property
    def N(self) -> int:
        return self.T * self.top_k

    @property
    def local_experts(self) -> int:
        return self.E // self.ep_ranks

    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def gemm_flops(self) -> int:
        """Algorithmic flops of the routed experts: 3 GEMMs of 2*d*h per copy."""
        return 6 * self.d * self.h * self.N


CONFIGS = [
    MoEConfig("tiny_fp32_T256_d128_E8_k2_h256", "f32", 256, 128, 8, 2, 256, seed=0),
    MoEConfig("qwen3_30b_a3b_T4096_d2048_E128_k8_h768", "bf16", 4096, 2048, 128, 8, 768, seed=1),
    MoEConfig("qwen3_30b_a3b_zipf_T16384_d2048_E128_k8_h768", "bf16", 16384, 2048, 128, 8, 768,
              seed=2, zipf_s=1.2),
    MoEConfig("qwen3_235b_a22b_decode_T64_d4096_E128_k8_h1536", "bf16", 64, 4096, 128, 8, 1536,
              seed=3),
    MoEConfig("gpt_oss_120b_ep8_T8192_d2880_E128_k4_h2880", "bf16", 8192, 2880, 128, 4, 2880,
              seed=4, ep_ranks=8),
]


def config(i_or_name) -> MoEConfig:
    if isinstance(i_or_name, int):
        return CONFIGS[i_or_name]
    for c in CONFIGS:
        if c.name == i_or_name:
            return c
    raise KeyError(i_or_name)


def _gen(device, seed: int, which: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000 + which)
    return g


def _normal(shape, std, dtype, device, gen, chunk_rows=None):
    """N(0, std) drawn in fp32, rounded once to ``dtype``."""
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(shape[0], -1)
    step = chunk_rows or shape[0]
    for r0 in range(0, shape[0], step):
        r1 = min(shape[0], r0 + step)
        tmp = torch.randn((r1 - r0, flat.shape[1]), generator=gen, device=device,
                          dtype=torch.float32)
        tmp.mul_(std)
        flat[r0:r1].copy_(tmp)
    return out


def zipf_bias(E: int, s: float, seed: int) -> np.ndarray:
    """Per-expert logit bias ln p_e, p_e ~ rank(e)^-s under a seeded ranking.

    Returned in float64; the layer stores it rounded to the layer dtype.
    """
    rng = np.random.default_rng(seed * 1000 + SEED_BIAS)
    rank = rng.permutation(E) + 1
    logp = -s * np.log(rank.astype(np.float64))
    logp -= np.log(np.exp(logp).sum())
    return logp


def make_layer(cfg: MoEConfig, device="cpu", T: Optional[int] = None,
               experts: bool = True):
    """Return dict of x, w_router, w1, w3, w2 for ``cfg`` on ``device``.

    ``T`` overrides the token count (the expert weights do not depend on it).
    """
    T = cfg.T if T is None else T
    dt = cfg.torch_dtype()
    x = _normal((T, cfg.d), 1.0, dt, device, _gen(device, cfg.seed, SEED_X))
    wr = _normal((cfg.E, cfg.d), cfg.router_std, dt, device,
                 _gen(device, cfg.seed, SEED_WR))
    if cfg.zipf_s is not None:
        b = torch.from_numpy(zipf_bias(cfg.E, cfg.zipf_s, cfg.seed)).to(torch.float32)
        wr[:, cfg.d - 1] = b.to(device=device, dtype=dt)
        x[:, cfg.d - 1] = 1.0
    out = {"x": x, "w_router": wr}
    if experts:
        ch = max(1, (1 << 26) // (cfg.h * cfg.d))   # ~256 MB fp32 per draw
        out["w1"] = _normal((cfg.E, cfg.h, cfg.d), 1.0 / math.sqrt(cfg.d), dt, device,
                            _gen(device, cfg.seed, SEED_W1), ch)
        out["w3"] = _normal((cfg.E, cfg.h, cfg.d), 1.0 / math.sqrt(cfg.d), dt, device,
                            _gen(device, cfg.seed, SEED_W3), ch)
        out["w2"] = _normal((cfg.E, cfg.d, cfg.h), 1.0 / math.sqrt(cfg.h), dt, device,
                            _gen(device, cfg.seed, SEED_W2), ch)
    return out


def make_logits(T: int, E: int, top_k: int, seed: int, std: float = 1.0,
                min_gap: float = 1e-3) -> np.ndarray:
    """fp32 router scores ``[T, E]`` whose k-th and (k+1)-th largest differ by
    at least ``min_gap`` in every row (rows failing that are redrawn).

    With such scores the selected set is stable under any rounding smaller
    than ``min_gap / 2``.
    """
    rng = np.random.default_rng(seed * 1000 + SEED_LOGITS)
    L = (rng.standard_normal((T, E)) * std).astype(np.float32)
    if top_k >= E:
        return L
    for _ in range(1000):
        srt = -np.sort(-L.astype(np.float64), axis=1)
        bad = (srt[:, top_k - 1] - srt[:, top_k]) < min_gap
        if not bad.any():
            return L
        L[bad] = (rng.standard_normal((int(bad.sum()), E)) * std).astype(np.float32)
    raise RuntimeError("could not draw logits with the requested top-k gap")


def make_rank_counts(G: int, R: int, L: int, rows: int, seed: int) -> np.ndarray:
    """counts_rm ``[G, R, L]`` ~ Multinomial(rows, uniform over G*R*L) (int32)."""
    rng = np.random.default_rng(seed * 1000 + 77)
    c = rng.multinomial(rows, np.full(G * R * L, 1.0 / (G * R * L)))
    return c.reshape(G, R, L).astype(np.int32)
