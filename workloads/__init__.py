"""Seeded synthetic inputs for the W4A16 group-wise GEMM and its grouped-expert form.

This module is shared by the CPU oracle's tests and by the CUDA path's tests and
benchmark. It only draws random numbers and arranges them; it holds none of the
method's arithmetic (no packing, no dequantisation, no products).

Tensor roles and shapes follow the Int4GroupwiseGemmPluginV2 page (class
description: activations [b, seq, K] fp16, scales [ceil(K/G), N] fp16, output
[b, seq, N] fp16; constructor: N = columns, K = rows of the weight matrix,
groupSize = G). The int4 codes are signed values in [-8, 7].

Distributions (one seeded numpy PCG64 generator per case):
  A  ~ N(0, 1) drawn in float32, rounded to float16
  q  ~ uniform integers in [-8, 7]
  s  ~ uniform in [0.002, 0.02] drawn in float32, rounded to float16
Grouped-expert case (Int4MoePlugin page, constructor: numExperts, topK,
hiddenSize, moeInterSize, quantizationGroupSize): each token draws topK distinct
experts uniformly; the (token, slot) pairs are stably sorted by expert, which
gives the gathered activation rows and the [E+1] prefix offsets.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import numpy as np

S_LOW, S_HIGH = 0.002, 0.02


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def n_groups(K: int, G: int) -> int:
    return -(-K // G)


@dataclasses.dataclass
class DenseCase:
    name: str
    M: int
    K: int
    N: int
    G: int
    seed: int
    A: np.ndarray  # [M, K] float16
    q: np.ndarray  # [K, N] int8 in [-8, 7]
    S: np.ndarray  # [ceil(K/G), N] float16


@dataclasses.dataclass
class GroupedCase:
    name: str
    E: int
    top_k: int
    tokens: int
    K: int
    N: int
    G: int
    seed: int
    A_tokens: np.ndarray      # [tokens, K] float16
    experts: np.ndarray       # [tokens, top_k] int32, distinct per token
    order: np.ndarray         # [tokens*top_k] int64: flat (token*top_k + slot) index of each gathered row
    A: np.ndarray             # [rows, K] float16, rows gathered per expert
    offsets: np.ndarray       # [E+1] int32 prefix offsets into A's rows
    q: np.ndarray             # [E, K, N] int8
    S: np.ndarray             # [E, ceil(K/G), N] float16

    @property
    def total_rows(self) -> int:
        return int(self.offsets[-1])


def dense(M: int, K: int, N: int, G: int, seed: int, name: str = "dense",
          a_scale: float = 1.0) -> DenseCase:
    """One dense case with the distributions stated in the module docstring."""
    g = _rng(seed)
    A = (g.standard_normal((M, K), dtype=np.float32) * np.float32(a_scale)).astype(np.float16)
    q = g.integers(-8, 8, size=(K, N), dtype=np.int8)
    S = g.uniform(S_LOW, S_HIGH, size=(n_groups(K, G), N)).astype(np.float32).astype(np.float16)
    return DenseCase(name, M, K, N, G, seed, A, q, S)


def grouped(E: int, top_k: int, tokens: int, K: int, N: int, G: int, seed: int,
            name: str = "grouped", empty_experts: Optional[List[int]] = None) -> GroupedCase:
    """Top-k routing of `tokens` tokens over E experts, rows gathered per expert.

    `empty_experts` (test aid) lists experts that no token may pick.
    """
    g = _rng(seed)
    A_tokens = g.standard_normal((tokens, K), dtype=np.float32).astype(np.float16)
    allowed = np.array([e for e in range(E) if not empty_experts or e not in empty_experts])
    if top_k > len(allowed):
        raise ValueError("top_k exceeds the number of selectable experts")
    experts = np.stack([g.choice(allowed, size=top_k, replace=False) for _ in range(tokens)]).astype(np.int32)
    flat = experts.reshape(-1)
    order = np.argsort(flat, kind="stable")
    counts = np.bincount(flat, minlength=E)
    offsets = np.zeros(E + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    A = A_tokens[order // top_k]
    q = g.integers(-8, 8, size=(E, K, N), dtype=np.int8)
    S = g.uniform(S_LOW, S_HIGH, size=(E, n_groups(K, G), N)).astype(np.float32).astype(np.float16)
    return GroupedCase(name, E, top_k, tokens, K, N, G, seed, A_tokens, experts,
                       order.astype(np.int64), np.ascontiguousarray(A), offsets, q, S)


def dense8(M: int, K: int, N: int, G: int, seed: int, name: str = "dense8") -> DenseCase:
    """A W8A16 case: activations as in `dense`, signed 8-bit codes uniform over
    [-128, 127], scales uniform over [S_LOW, S_HIGH] / 16, so that the weights q*s
    span about the same range as the int4 cases'."""
    g = _rng(seed)
    A = g.standard_normal((M, K), dtype=np.float32).astype(np.float16)
    q = g.integers(-128, 128, size=(K, N), dtype=np.int8)
    S = (g.uniform(S_LOW, S_HIGH, size=(n_groups(K, G), N)) / 16).astype(np.float32).astype(np.float16)
    return DenseCase(name, M, K, N, G, seed, A, q, S)


@dataclasses.dataclass
class MoeCase:
    name: str
    tokens: int
    E: int
    top_k: int
    H: int
    I: int
    G: int
    seed: int
    X: np.ndarray         # [tokens, H] float16 hidden states
    logits: np.ndarray    # [tokens, E] float16 router logits
    q_up: np.ndarray      # [E, H, I] int8 codes of the up projections
    S_up: np.ndarray      # [E, ceil(H/G), I] float16
    q_down: np.ndarray    # [E, I, H] int8 codes of the down projections
    S_down: np.ndarray    # [E, ceil(I/G), H] float16


def moe(tokens: int, E: int, top_k: int, H: int, I: int, G: int, seed: int, name: str = "moe") -> MoeCase:
    """A mixture-of-experts layer case (Int4MoePlugin page, constructor: numExperts,
    topK, hiddenSize, moeInterSize, quantizationGroupSize): hidden states and router
    logits ~ N(0, 1) rounded to fp16; per-expert codes and scales as in `dense`."""
    g = _rng(seed)
    X = g.standard_normal((tokens, H), dtype=np.float32).astype(np.float16)
    logits = g.standard_normal((tokens, E), dtype=np.float32).astype(np.float16)
    q_up = g.integers(-8, 8, size=(E, H, I), dtype=np.int8)
    S_up = g.uniform(S_LOW, S_HIGH, size=(E, n_groups(H, G), I)).astype(np.float32).astype(np.float16)
    q_down = g.integers(-8, 8, size=(E, I, H), dtype=np.int8)
    S_down = g.uniform(S_LOW, S_HIGH, size=(E, n_groups(I, G), H)).astype(np.float32).astype(np.float16)
    return MoeCase(name, tokens, E, top_k, H, I, G, seed, X, logits, q_up, S_up, q_down, S_down)


# The five workload families and their sizes, with a fixed seed per config.
CONFIGS: Dict[str, dict] = {
    "tiny":        dict(kind="dense", M=4, K=512, N=512, G=128, seed=0),
    "decode_m1":   dict(kind="dense", M=1, K=4096, N=4096, G=128, seed=1),
    "decode_m16":  dict(kind="dense", M=16, K=4096, N=4096, G=128, seed=11),
    "mlp_up":      dict(kind="dense", M=8, K=4096, N=14336, G=128, seed=2),
    "mlp_down":    dict(kind="dense", M=8, K=14336, N=4096, G=128, seed=21),
    "mlp_up_g64":  dict(kind="dense", M=8, K=4096, N=14336, G=64, seed=22),
    "prefill":     dict(kind="dense", M=2048, K=4096, N=4096, G=128, seed=3),
    "grouped":     dict(kind="grouped", E=8, top_k=2, tokens=512, K=4096, N=14336, G=128, seed=4),
    # the whole mixture-of-experts layer around the grouped product (up 4096 -> 14336,
    # down 14336 -> 4096), routed by its own logits
    "moe_layer":   dict(kind="moe", E=8, top_k=2, tokens=512, H=4096, I=14336, G=128, seed=6),
    # the same layer at a decode batch of 4 tokens (8 gathered rows)
    "moe_decode":  dict(kind="moe", E=8, top_k=2, tokens=4, H=4096, I=14336, G=128, seed=9),
    # the 8-bit code variant (W8A16) at the decode and prefill sizes
    "w8_decode_m16": dict(kind="dense8", M=16, K=4096, N=4096, G=128, seed=7),
    "w8_prefill":    dict(kind="dense8", M=2048, K=4096, N=4096, G=128, seed=8),
}


def make(name: str):
    cfg = dict(CONFIGS[name])
    kind = cfg.pop("kind")
    if kind == "dense":
        return dense(name=name, **cfg)
    if kind == "moe":
        return moe(name=name, **cfg)
    if kind == "dense8":
        return dense8(name=name, **cfg)
    return grouped(name=name, **cfg)
