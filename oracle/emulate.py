"""Rounding-contract emulation of the two elementwise stages, in numpy fp32.

TEST INFRASTRUCTURE ONLY (same rule as ``oracle.muon``): never imported by
the product path.

The momentum and update stages are elementwise and their result is fixed
bit for bit once the order of the fp32 operations and the rounding of each
stored value are fixed.  The contract the library states for them is:

momentum (per element, all fp32, round-to-nearest-even, no fused multiply-add):
    t    = mu * buf
    buf' = t + g                      -> stored (bf16 RNE for bf16 tensors)
    x0   = g + mu * buf'  (Nesterov)  using the fp32 buf' (not the stored one)
    x0   = buf'           (otherwise)
    -> stored (bf16 RNE for bf16 tensors)

update (per element):
    decay = 1 - lr * wd               (fp32)
    scale = fl32(lr * 0.2 * sqrt(max(rows, cols)))  (computed in double, rounded once)
    p'    = p * decay - scale * O     (each product rounded, then the difference)

The arithmetic follows the DMuon Training Guide hyperparameter table (momentum,
nesterov and lr rows); the rounding points are the library's own contract.
"""
from __future__ import annotations

import math

import numpy as np


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even), returned as fp32.

    Done on the bit pattern: add 0x7FFF plus the lowest kept bit, then clear
    the low 16 bits.  NaNs are kept quiet.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    out = r.view(np.float32).copy()
    nan = np.isnan(x)
    if nan.any():
        out[nan] = np.float32("nan")
    return out


def store(x: np.ndarray, dtype: str) -> np.ndarray:
    x = np.asarray(x, dtype=np.float32)
    return bf16_round(x) if dtype == "bf16" else x


def momentum_fp32(buf: np.ndarray, g: np.ndarray, mu: float, nesterov: bool, dtype: str):
    """(stored buf', stored x0) following the momentum contract above."""
    buf = np.asarray(buf, dtype=np.float32)
    g = np.asarray(g, dtype=np.float32)
    mu32 = np.float32(mu)
    with np.errstate(over="ignore", invalid="ignore"):
        t = (mu32 * buf).astype(np.float32)
        nb = (t + g).astype(np.float32)
        if nesterov:
            u = (mu32 * nb).astype(np.float32)
            x0 = (g + u).astype(np.float32)
        else:
            x0 = nb
    return store(nb, dtype), store(x0, dtype)


def update_scale(lr: float, rows: int, cols: int) -> np.float32:
    return np.float32(float(np.float32(lr)) * 0.2 * math.sqrt(max(rows, cols)))


def update_fp32(p: np.ndarray, o: np.ndarray, lr: float, wd: float, dtype: str):
    """Stored p' following the update contract above (O given as fp32)."""
    p = np.asarray(p, dtype=np.float32)
    o = np.asarray(o, dtype=np.float32)
    lr32, wd32 = np.float32(lr), np.float32(wd)
    decay = np.float32(np.float32(1.0) - np.float32(lr32 * wd32))
    scale = update_scale(lr, p.shape[0], p.shape[1])
    a = (p * decay).astype(np.float32)
    b = (scale * o).astype(np.float32)
    return store((a - b).astype(np.float32), dtype)


def clip_scale_fp32(g: np.ndarray, coef: float, dtype: str) -> np.ndarray:
    """Stored g * coef: the coefficient rounded to fp32 once, one fp32 product."""
    g = np.asarray(g, dtype=np.float32)
    with np.errstate(invalid="ignore"):  # inf * 0
        return store((g * np.float32(coef)).astype(np.float32), dtype)
