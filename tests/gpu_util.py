"""Helpers shared by the GPU parity tests: device copies of seeded cases and the
element-wise tolerance |gpu - ref| <= 1e-2 + 5e-3 * |ref|."""
from __future__ import annotations

import numpy as np
import torch

import weight_only_int4_wise_b200 as w

ATOL = 1e-2
RTOL = 5e-3
SENTINEL = 0x7BAD  # a finite fp16 bit pattern the product never writes into a guard band


def dev(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def within_tolerance(got: np.ndarray, ref: np.ndarray):
    g = got.astype(np.float64)
    r = ref.astype(np.float64)
    err = np.abs(g - r)
    bound = ATOL + RTOL * np.abs(r)
    ok = bool(np.all(np.isfinite(g)) and np.all(err <= bound))
    rel = err / np.maximum(np.abs(r), 1e-6)
    return ok, float(err.max(initial=0.0)), float(rel.max(initial=0.0))


def guarded_output(rows: int, cols: int, pad: int = 64):
    """An fp16 [rows, cols] view in the middle of a buffer whose both ends hold a sentinel."""
    flat = torch.full((pad + rows * cols + pad,), 0, dtype=torch.int16, device="cuda")
    flat.fill_(SENTINEL)
    view = flat[pad:pad + rows * cols].view(torch.float16).view(rows, cols)
    return flat, view, pad


def guards_intact(flat: torch.Tensor, pad: int, n: int) -> bool:
    h = flat.cpu().numpy().view(np.uint16)
    return bool(np.all(h[:pad] == SENTINEL) and np.all(h[pad + n:] == SENTINEL))


def device_weights(q: np.ndarray):
    """Pack and repack int8 codes on the GPU; returns (canonical, tiled) device tensors."""
    return w.prepare_weights(dev(q))
