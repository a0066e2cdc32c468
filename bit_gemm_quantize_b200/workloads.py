"""Seeded synthetic inputs for the W4A8 Integer-Scale linear layer.

This module only draws random numbers and lays them out; it holds none of the
quantization arithmetic, so the CPU oracle and the CUDA path can both be fed
from it without sharing any of the method.

Shapes and distributions follow the workloads the Integer Scale summary page
measures (section 5.2, Fig. 5a / Fig. 6: K=4096, N=22016, batch sweep; section
5.3: Mixtral 8x7B experts) with LLaMA-style hidden sizes.  Real activations
and weights are not available, so:

* X ~ N(0, 1) per element, with round(outlier_frac * K) "outlier channels"
  (columns of X, chosen without replacement) multiplied by ``outlier_scale``,
  which mimics the channel outliers that per-token quantization has to absorb;
* W ~ N(0, 0.02) per element, drawn in fp32 (weights are quantized from fp32
  even when X is bf16);
* MoE routing: every token picks two distinct experts uniformly at random.

Draw order from one ``numpy.random.Generator(PCG64(seed))``: X, then W, then
the outlier channel indices, then the routing.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

__all__ = [
    "LinearWorkload",
    "MoEWorkload",
    "make_linear",
    "make_moe",
    "route_rows",
    "to_bf16_bits",
    "bf16_bits_to_f32",
    "SWEEP_M",
    "CONFIGS",
]

# FFN up-projection batch sweep of the pages' kernel comparison (K=4096, N=22016).
SWEEP_M = (1, 8, 32, 128, 512, 1024)


@dataclass
class LinearWorkload:
    x: np.ndarray  # [M, K] float32 (already rounded to bf16 when x_dtype == "bf16")
    w: np.ndarray  # [K, N] float32
    x_dtype: str  # "f32" or "bf16"
    outlier_cols: np.ndarray  # int64 indices into K
    seed: int

    @property
    def M(self) -> int:
        return self.x.shape[0]

    @property
    def K(self) -> int:
        return self.x.shape[1]

    @property
    def N(self) -> int:
        return self.w.shape[1]


@dataclass
class MoEWorkload:
    x: np.ndarray  # [T, K] float32 (bf16-rounded)
    w: list  # E arrays [K, N] float32
    experts: np.ndarray  # [T, topk] int64, distinct per token
    outlier_cols: np.ndarray
    seed: int


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even on the dropped half."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> fp32 (exact widening)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _outlier_count(K: int, frac: float) -> int:
    return int(round(frac * K))


def make_linear(
    M: int,
    K: int,
    N: int,
    *,
    x_dtype: str = "bf16",
    seed: int = 0,
    outlier_frac: float = 0.005,
    n_outliers: Optional[int] = None,
    outlier_scale: float = 30.0,
    w_std: float = 0.02,
) -> LinearWorkload:
    """One linear layer's synthetic activations and weights."""
    if x_dtype not in ("f32", "bf16"):
        raise ValueError(f"x_dtype must be 'f32' or 'bf16', got {x_dtype!r}")
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal((M, K), dtype=np.float32)
    w = (rng.standard_normal((K, N), dtype=np.float32) * np.float32(w_std)).astype(np.float32)
    n_out = _outlier_count(K, outlier_frac) if n_outliers is None else int(n_outliers)
    cols = np.sort(rng.choice(K, size=n_out, replace=False)) if n_out > 0 else np.zeros(0, np.int64)
    if n_out > 0:
        x[:, cols] *= np.float32(outlier_scale)
    if x_dtype == "bf16":
        x = bf16_bits_to_f32(to_bf16_bits(x))
    return LinearWorkload(x=x, w=w, x_dtype=x_dtype, outlier_cols=cols.astype(np.int64), seed=seed)


def make_moe(
    tokens: int,
    K: int,
    N: int,
    experts: int,
    *,
    topk: int = 2,
    seed: int = 0,
    outlier_frac: float = 0.005,
    outlier_scale: float = 30.0,
    w_std: float = 0.02,
) -> MoEWorkload:
    """A mixture-of-experts layer: per-expert weights plus top-k routing."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal((tokens, K), dtype=np.float32)
    ws = [
        (rng.standard_normal((K, N), dtype=np.float32) * np.float32(w_std)).astype(np.float32)
        for _ in range(experts)
    ]
    n_out = _outlier_count(K, outlier_frac)
    cols = np.sort(rng.choice(K, size=n_out, replace=False)) if n_out > 0 else np.zeros(0, np.int64)
    if n_out > 0:
        x[:, cols] *= np.float32(outlier_scale)
    x = bf16_bits_to_f32(to_bf16_bits(x))
    route = np.stack([rng.choice(experts, size=topk, replace=False) for _ in range(tokens)]).astype(np.int64)
    return MoEWorkload(x=x, w=ws, experts=route, outlier_cols=cols.astype(np.int64), seed=seed)


def route_rows(experts: np.ndarray, n_experts: int):
    """Layout of the routed rows of a top-k routing [T, topk]: rows grouped by
    expert (expert 0 first), tokens ascending within an expert.

    Returns (row_index int32 [R]: the token of each routed row,
    offsets int64 [E+1]: the rows of expert e are offsets[e] .. offsets[e+1]-1).
    """
    experts = np.asarray(experts, np.int64)
    T, topk = experts.shape
    token = np.repeat(np.arange(T, dtype=np.int64), topk)
    expert = experts.reshape(-1)
    order = np.lexsort((token, expert))  # by expert, then token
    row_index = token[order].astype(np.int32)
    counts = np.bincount(expert, minlength=n_experts).astype(np.int64)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    return row_index, offsets


# The five workloads, by what they are.  Each entry: dict of keyword arguments.
CONFIGS = {
    "tiny": dict(M=16, K=1024, N=1024, x_dtype="f32", n_outliers=4, outlier_scale=20.0, out="f32"),
    "decode": dict(Ms=(1, 4, 16), K=4096, N=4096, x_dtype="bf16", outlier_scale=30.0, out="f16"),
    "ffn_up_sweep": dict(Ms=SWEEP_M, K=4096, N=22016, x_dtype="bf16", outlier_scale=30.0, out="f16"),
    "prefill": dict(shapes=((4096, 4096, 11008), (4096, 11008, 4096)), x_dtype="bf16", out="f16"),
    "moe": dict(tokens=2048, K=4096, N=14336, experts=8, topk=2, out="f16"),
}
