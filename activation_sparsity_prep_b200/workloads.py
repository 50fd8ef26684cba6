"""Seeded synthetic inputs for the SharQ hot path.

This module draws random numbers and rounds them to bf16; it holds none of
the method's arithmetic (no norm, mask, scale or quantisation).  Both the
CUDA path and the CPU oracle receive the arrays built here, so the two sides
always see the same bits.

The pages motivate SharQ with activations whose input-dependent outliers
dominate FP4 block scales (SharQ paper, Abstract).  No dataset or trained
weight is used; the distributions below stand in for them:

* ``normal_outlier``   X ~ N(0,1) with a few seeded whole-column outliers
* ``laplace_outlier``  X ~ Laplace(0,1) with round(0.005 K) seeded columns,
                       each scaled by U[20,100]
* ``student_t``        X = t(nu=3) per element times a per-token scale
                       s ~ LogNormal(0, 0.5)
* weights              W ~ N(0, 0.02)

Generator seeding: ``numpy.random.default_rng([cfg, tensor_id + 16*linear])``
with tensor_id 0 = X, 1 = W, 2 = outlier channels, 3 = outlier factors,
4 = routing, 5 = per-token scales.  Values are drawn in float64, cast to
float32 and rounded to bf16 with round-to-nearest-even.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional, Tuple

import numpy as np

TID_X, TID_W, TID_CH, TID_FAC, TID_ROUTE, TID_TOKSCALE = 0, 1, 2, 3, 4, 5

_W_CHUNK_ROWS = 2048


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return the raw
    uint16 bit patterns.  Inputs must be finite."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen raw bf16 bit patterns to float32 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _rng(cfg: int, tensor_id: int, linear: int) -> np.random.Generator:
    return np.random.default_rng([cfg, tensor_id + 16 * linear])


def activation(dist: str, cfg: int, linear: int, M: int, K: int,
               n_outlier: Optional[int] = None) -> np.ndarray:
    """Activation tensor X [M, K] as bf16 bits (uint16)."""
    if dist == "normal_outlier":
        x = _rng(cfg, TID_X, linear).standard_normal((M, K))
        cnt = 4 if n_outlier is None else n_outlier
        ch = _rng(cfg, TID_CH, linear).choice(K, size=cnt, replace=False)
        x[:, ch] *= 50.0
    elif dist == "laplace_outlier":
        x = _rng(cfg, TID_X, linear).laplace(0.0, 1.0, size=(M, K))
        cnt = int(round(0.005 * K)) if n_outlier is None else n_outlier
        ch = _rng(cfg, TID_CH, linear).choice(K, size=cnt, replace=False)
        fac = _rng(cfg, TID_FAC, linear).uniform(20.0, 100.0, size=cnt)
        x[:, ch] *= fac[None, :]
    elif dist == "student_t":
        x = _rng(cfg, TID_X, linear).standard_t(3.0, size=(M, K))
        s = _rng(cfg, TID_TOKSCALE, linear).lognormal(0.0, 0.5, size=(M, 1))
        x *= s
    else:
        raise ValueError(f"unknown activation distribution {dist!r}")
    return f32_to_bf16_bits(x.astype(np.float32))


def weight(cfg: int, linear: int, N: int, K: int, std: float = 0.02) -> np.ndarray:
    """Weight W [N, K] ~ N(0, std) as bf16 bits, drawn in row chunks of
    2048 (one stream, so the result does not depend on available memory)."""
    g = _rng(cfg, TID_W, linear)
    out = np.empty((N, K), dtype=np.uint16)
    for r0 in range(0, N, _W_CHUNK_ROWS):
        r1 = min(N, r0 + _W_CHUNK_ROWS)
        w = g.standard_normal((r1 - r0, K)) * std
        out[r0:r1] = f32_to_bf16_bits(w.astype(np.float32))
    return out


def gamma_ones(K: int) -> np.ndarray:
    """RMSNorm weight of all ones (bf16 1.0 = 0x3F80)."""
    return np.full((K,), 0x3F80, dtype=np.uint16)


def gamma_random(cfg: int, linear: int, K: int) -> np.ndarray:
    """A non-trivial RMSNorm weight ~ U[0.5, 1.5] for coverage tests."""
    g = _rng(cfg, 7, linear).uniform(0.5, 1.5, size=K)
    return f32_to_bf16_bits(g.astype(np.float32))


def beta_random(cfg: int, linear: int, K: int) -> np.ndarray:
    """A LayerNorm bias ~ N(0, 0.1) (stands in for an adaLN shift)."""
    b = _rng(cfg, 6, linear).normal(0.0, 0.1, size=K)
    return f32_to_bf16_bits(b.astype(np.float32))


def routing(cfg: int, T: int, E: int, topk: int) -> np.ndarray:
    """Uniform random top-k routing: [T, topk] distinct expert ids per token."""
    g = _rng(cfg, TID_ROUTE, 0)
    keys = g.random((T, E))
    return np.argsort(keys, axis=1, kind="stable")[:, :topk].astype(np.int32)


def group_by_expert(experts: np.ndarray, E: int) -> Tuple[np.ndarray, np.ndarray]:
    """Dispatch order for a grouped linear.

    Returns ``row_index`` [T*topk] (the token row each dispatched row reads,
    grouped by expert, tokens ascending inside a group) and ``offsets`` [E+1]
    (group boundaries)."""
    T, topk = experts.shape
    flat_e = experts.reshape(-1)
    flat_t = np.repeat(np.arange(T, dtype=np.int32), topk)
    order = np.lexsort((flat_t, flat_e))
    row_index = flat_t[order].astype(np.int32)
    counts = np.bincount(flat_e, minlength=E)
    offsets = np.zeros(E + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    return row_index, offsets


# ---------------------------------------------------------------------------
# Workload registry: shapes follow the model families named on the pages
# (Llama-3.1-8B, Qwen2.5-7B, Qwen3-30B-A3B, and the Wan2.2 video DiT for the
# LayerNorm form); weights are random.
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class Linear:
    name: str
    K: int
    N: int
    norm: bool          # fused norm on the input (RMSNorm: gamma = 1, eps = 1e-6)
    index: int          # linear index used in the seeds
    layernorm: bool = False   # LayerNorm with gamma ~ U[0.5, 1.5] and beta ~ N(0, 0.1)


@dataclass(frozen=True)
class Workload:
    name: str
    cfg: int
    dist: str
    linears: Tuple[Linear, ...]
    Ms: Tuple[int, ...] = ()
    moe: Optional[Dict[str, int]] = None
    n_outlier: Optional[int] = None
    sweep: Tuple[Tuple[str, int, int], ...] = ()   # (fmt, n, m)


EPS = 1e-6

WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload(
        "tiny", 1, "normal_outlier",
        (Linear("tiny", 256, 256, True, 0),), Ms=(16,)),
    # a small SwiGLU MLP (gate+up 256 -> 2 x 256, down 256 -> 256) for the
    # producer-fused path's quick checks
    "tiny_mlp": Workload(
        "tiny_mlp", 7, "laplace_outlier",
        (Linear("gate_up", 256, 512, True, 0),
         Linear("down", 256, 256, False, 1)),
        Ms=(16,)),
    "llama8b": Workload(
        "llama8b", 2, "laplace_outlier",
        (Linear("qkv", 4096, 6144, True, 0),
         Linear("o", 4096, 4096, False, 1),
         Linear("gate_up", 4096, 28672, True, 2),
         Linear("down", 14336, 4096, False, 3)),
        Ms=(1, 16, 128, 2048)),
    "qwen7b": Workload(
        "qwen7b", 3, "student_t",
        (Linear("qkv", 3584, 4608, True, 0),
         Linear("gate_up", 3584, 37888, True, 1),
         Linear("down", 18944, 3584, False, 2)),
        Ms=(4096,)),
    "qwen3moe": Workload(
        "qwen3moe", 4, "laplace_outlier",
        (Linear("gate_up", 2048, 1536, True, 0),
         Linear("down", 768, 2048, False, 1)),
        moe={"T": 4096, "E": 128, "topk": 8}),
    "sweep": Workload(
        "sweep", 5, "laplace_outlier",
        (Linear("gate_up", 4096, 14336, True, 0),),
        Ms=(16384,),
        sweep=tuple((f, n, m) for f in ("nvfp4", "mxfp4")
                    for (n, m) in ((2, 4), (1, 4), (4, 8)))),
    # Wan2.2-T2V-A14B-shaped DiT block (hidden 5120, FFN 13824): LayerNorm
    # (gamma = 1 + scale, beta = shift, as adaLN modulation gives) in front of
    # the fused q/k/v and the FFN up projection; 8192 video tokens.
    "wan_dit": Workload(
        "wan_dit", 6, "laplace_outlier",
        (Linear("qkv", 5120, 15360, True, 0, layernorm=True),
         Linear("o", 5120, 5120, False, 1),
         Linear("ffn_up", 5120, 13824, True, 2, layernorm=True),
         Linear("ffn_down", 13824, 5120, False, 3)),
        Ms=(8192,)),
}


def linear_inputs(wl: Workload, lin: Linear, M: int) -> Dict[str, np.ndarray]:
    """X, W, gamma (or None), beta (or None) and the norm kind ("rms" or
    "layernorm") for one linear of a workload at M rows."""
    X = activation(wl.dist, wl.cfg, lin.index, M, lin.K, wl.n_outlier)
    W = weight(wl.cfg, lin.index, lin.N, lin.K)
    if lin.layernorm:
        return {"X": X, "W": W, "gamma": gamma_random(wl.cfg, lin.index, lin.K),
                "beta": beta_random(wl.cfg, lin.index, lin.K), "norm": "layernorm"}
    g = gamma_ones(lin.K) if lin.norm else None
    return {"X": X, "W": W, "gamma": g, "beta": None, "norm": "rms"}
