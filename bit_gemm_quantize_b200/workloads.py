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

Every layer drawn here is checked against the int32 accumulator bound before
it is returned (``assert_int32_bound``): the kernels and the oracle both
accumulate sum_g S[g,n] * P_g[m,n] in 32 bits, so a generated weight matrix
whose integer scales could push that sum past 2^31 for some input is refused
with ``ValueError``.  The check is a conservative upper bound computed from
the raw weights (largest |w| per group, never a quantized code or scale), so
it feeds no value to either side.
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
    "int32_bound_upper",
    "assert_int32_bound",
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


def int32_bound_upper(w: np.ndarray, group: int = 128, alpha: Optional[int] = 1024, qmax_w: int = 7,
                      qmax_x: int = 127) -> float:
    """An upper bound on qmax_x * qmax_w * group * max_n sum_g |S[g,n]| for the
    integer scales S = round(s_g * alpha), s_g = max_{k in g}|w[k,n]| / qmax_w,
    derived from the raw weights alone (fp64): each S is at most
    amax * alpha / qmax_w inflated by 2^-20 (fp32 rounding of the scale) plus
    1/2 (rounding to an integer).  alpha=None bounds the searched amplifier
    (the smallest power of two lifting the smallest positive scale to 1) by
    the next power of two above the reciprocal of a deflated smallest scale."""
    w = np.asarray(w)
    K, N = w.shape
    if K % group:
        raise ValueError("K must be a multiple of group")
    # largest |w| per (group, column): exact in the input precision, widened after
    amax = np.abs(w.reshape(K // group, group, N)).max(axis=1).astype(np.float64)  # [G, N]
    if alpha is None:
        pos = amax[amax > 0]
        if pos.size == 0:
            return 0.0
        s_lo = pos.min() / qmax_w * (1.0 - 2.0 ** -20)
        alpha = 1.0 if s_lo >= 1.0 else 2.0 ** np.ceil(np.log2(1.0 / s_lo))
    s_up = amax * float(alpha) / qmax_w * (1.0 + 2.0 ** -20) + 0.5
    s_up[amax == 0] = 0.0
    return float(qmax_x) * qmax_w * group * float(s_up.sum(axis=0).max(initial=0.0))


def assert_int32_bound(w: np.ndarray, group: int = 128, alpha: Optional[int] = 1024, qmax_w: int = 7,
                       qmax_x: int = 127) -> None:
    """Refuse (ValueError) weights whose integer-scale accumulators could leave
    int32 for some input (the worst case of int32_bound_upper)."""
    b = int32_bound_upper(w, group, alpha, qmax_w, qmax_x)
    if b >= 2.0 ** 31:
        raise ValueError(f"weights break the int32 accumulator bound: worst case {b:.3e} >= 2^31 "
                         f"(group {group}, alpha {alpha})")


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
    group: int = 128,
    alpha: Optional[int] = 1024,
    check_bound: bool = True,
) -> LinearWorkload:
    """One linear layer's synthetic activations and weights.  The weights are
    checked against the int32 accumulator bound for (group, alpha) unless
    check_bound is False (alpha=None: the searched amplifier)."""
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
    if check_bound and K % group == 0:
        assert_int32_bound(w, group, alpha)
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
    group: int = 128,
    alpha: Optional[int] = None,
) -> MoEWorkload:
    """A mixture-of-experts layer: per-expert weights plus top-k routing.  The
    amplifier is one per layer (alpha=None: searched over every expert's
    scales), so the int32 bound is checked for each expert with the bound on
    the layer's amplifier."""
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
    if K % group == 0:
        a_layer = alpha
        if alpha is None:  # one amplifier bound for the whole layer: from all experts' weights
            a_layer = _searched_alpha_upper(ws, group)
        for w in ws:
            assert_int32_bound(w, group, a_layer)
    return MoEWorkload(x=x, w=ws, experts=route, outlier_cols=cols.astype(np.int64), seed=seed)


def _searched_alpha_upper(ws, group: int, qmax_w: int = 7) -> int:
    """Upper bound on the amplifier searched over several weight matrices."""
    lo = np.inf
    for w in ws:
        w = np.asarray(w)
        K, N = w.shape
        amax = np.abs(w.reshape(K // group, group, N)).max(axis=1).astype(np.float64)
        pos = amax[amax > 0]
        if pos.size:
            lo = min(lo, pos.min() / qmax_w * (1.0 - 2.0 ** -20))
    if not np.isfinite(lo) or lo >= 1.0:
        return 1
    return int(2.0 ** np.ceil(np.log2(1.0 / lo)))


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
