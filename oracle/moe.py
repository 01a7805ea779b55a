"""CPU oracle for the INT4 mixture-of-experts layer — TEST INFRASTRUCTURE ONLY.

Only `tests/`, `__graft_entry__.smoke()` and `bench.py`'s CPU-baseline leg may
use this module. It follows the Int4 Moe Plugin page (constructor parameters
numExperts, topK, hiddenSize, moeInterSize, activationType,
quantizationGroupSize). The page names the layer's parameters but not its
steps; the steps below are the plainest reading of them, each written out
plainly (fp64 arithmetic, one rounding to fp16 where a step produces fp16):

  1. route     each token's topK experts by router logit (ties: the lower
               expert index first); their weights are the softmax of the
               selected logits;
  2. dispatch  the (token, slot) pairs grouped by expert, stable in
               (token, slot) order: gathered row r holds token order[r] // topK;
               offsets[e] .. offsets[e+1] are expert e's rows;
  3. up        h = fp16(x_gathered @ dequant(W_up[e])) per expert
               (hiddenSize -> moeInterSize, the grouped W4A16 GEMM);
  4. activate  a = fp16(act(h)), act the elementwise activationType;
  5. down      y = fp16(a @ dequant(W_down[e])) per expert
               (moeInterSize -> hiddenSize);
  6. combine   out[t] = fp16(sum over slots j of weight[t, j] * y[row of (t, j)]).

The GEMM steps call the C oracle (`oracle.load()`); everything else is numpy in
float64. Parity pins: tests/test_moe_oracle.py.
"""
from __future__ import annotations

import math
from typing import Dict, List, Sequence

import numpy as np
from scipy.special import erf

# Activation codes (the elementwise activations of the activationType parameter
# that this layer implements; the same codes in include/w4a16.h).
ACT_IDENTITY = 0
ACT_RELU = 1
ACT_GELU_ERF = 2
ACT_GELU_TANH = 3
ACTIVATIONS = {"identity": ACT_IDENTITY, "relu": ACT_RELU, "gelu_erf": ACT_GELU_ERF, "gelu_tanh": ACT_GELU_TANH}


def route(logits: np.ndarray, top_k: int):
    """Step 1 (topK): ids [T, k] int32 (descending logit, ties -> lower index) and
    weights [T, k] float64 (softmax over the selected logits)."""
    lg = np.asarray(logits, dtype=np.float16).astype(np.float64)
    T, E = lg.shape
    if not 1 <= top_k <= E:
        raise ValueError("top_k must be in [1, E]")
    ids = np.zeros((T, top_k), dtype=np.int32)
    w = np.zeros((T, top_k), dtype=np.float64)
    for t in range(T):
        # stable sort on the negated logit: equal logits keep ascending expert order
        order = sorted(range(E), key=lambda e: (-lg[t, e], e))[:top_k]
        ids[t] = order
        sel = np.array([lg[t, e] for e in order])
        ex = np.exp(sel - sel.max())
        w[t] = ex / ex.sum()
    return ids, w


def dispatch(ids: np.ndarray, num_experts: int):
    """Step 2: order [T*k] (flat index t*k + j of each gathered row), offsets [E+1]
    int32, pos [T, k] (gathered row of slot j of token t)."""
    T, k = ids.shape
    flat = ids.reshape(-1)
    order = np.array(sorted(range(T * k), key=lambda i: (int(flat[i]), i)), dtype=np.int64)
    counts = np.bincount(flat, minlength=num_experts)
    offsets = np.zeros(num_experts + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    pos = np.zeros(T * k, dtype=np.int64)
    pos[order] = np.arange(T * k)
    return order, offsets, pos.reshape(T, k)


def activation(h: np.ndarray, act: int) -> np.ndarray:
    """Step 4: a = fp16(act(h)) evaluated in float64 on the fp16 values of h."""
    x = np.asarray(h, dtype=np.float16).astype(np.float64)
    if act == ACT_IDENTITY:
        y = x
    elif act == ACT_RELU:
        y = np.maximum(x, 0.0)
    elif act == ACT_GELU_ERF:
        y = 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))
    elif act == ACT_GELU_TANH:
        y = 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))
    else:
        raise ValueError(f"unknown activation {act}")
    return y.astype(np.float16)


def combine(y: np.ndarray, weights: np.ndarray, pos: np.ndarray) -> np.ndarray:
    """Step 6: out[t] = fp16(sum_j weights[t, j] * y[pos[t, j]]) in float64, slot order."""
    yy = np.asarray(y, dtype=np.float16).astype(np.float64)
    T, k = pos.shape
    acc = np.zeros((T, yy.shape[1]), dtype=np.float64)
    for j in range(k):
        acc += weights[:, j:j + 1] * yy[pos[:, j]]
    return acc.astype(np.float16)


def moe_layer(o, X: np.ndarray, logits: np.ndarray, wp_up: Sequence[np.ndarray], S_up: Sequence[np.ndarray],
              wp_down: Sequence[np.ndarray], S_down: Sequence[np.ndarray], top_k: int, G: int,
              act: int) -> Dict[str, np.ndarray]:
    """Steps 1-6 for tokens X [T, H] fp16 and router logits [T, E] fp16, with canonical
    packed weights W_up[e] [H, I] and W_down[e] [I, H] and their fp16 scales.
    Returns every intermediate (ids, weights, order, offsets, pos, x_gathered, h, a, y, out)."""
    X = np.asarray(X, dtype=np.float16)
    T, H = X.shape
    E = len(wp_up)
    I = wp_up[0].shape[1]
    ids, w = route(logits, top_k)
    order, offsets, pos = dispatch(ids, E)
    xg = np.ascontiguousarray(X[order // top_k])
    h = o.grouped_gemm(xg, list(wp_up), list(S_up), offsets, H, G)
    a = activation(h, act)
    y = o.grouped_gemm(a, list(wp_down), list(S_down), offsets, I, G)
    out = combine(y, w, pos)
    return {"ids": ids, "weights": w, "order": order, "offsets": offsets, "pos": pos, "x_gathered": xg,
            "h": h, "a": a, "y": y, "out": out}
