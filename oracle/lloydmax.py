"""Gaussian Lloyd-Max scalar codebooks (oracle; test infrastructure only).

"RoPE-Aware Bit Allocation for KV-Cache Quantization", abstract: Block-GTQ is
built on TurboQuant-MSE (TQ-MSE), an MSE-optimal scalar quantizer applied to
coordinates that are normalised to unit variance. The abstract does not print
the codebook; the reading adopted here is the Lloyd-Max quantizer of a unit
Gaussian with 2^b levels (the MSE-optimal scalar quantizer of that law), for
b = 1..8, with

* D(b)  = its mean squared error per unit variance, D(0) = 1 (a 0-bit
          coordinate is reconstructed as 0);
* frozen centroids = the Lloyd-Max centroids rounded once to fp16 (RNE);
* thresholds = exact midpoints of adjacent frozen centroids, held in fp32
          (the midpoint of two fp16 values is exact in fp32), so that the
          nearest-centroid rule equals "count the thresholds below z", ties
          going to the lower index.

The solver is Lloyd's alternation (midpoint thresholds, conditional-mean
centroids) with the closed-form Gaussian interval mean
    E[X | a < X < b] = (phi(a) - phi(b)) / (Phi(b) - Phi(a)),
started from the compander guess Phi^-1((m + 1/2) / 2^b).
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
from scipy.special import erfc, ndtri

_SQRT2 = math.sqrt(2.0)
_INV_SQRT_2PI = 1.0 / math.sqrt(2.0 * math.pi)
B_MAX = 8
_TABLE_FILE = os.path.join(os.path.dirname(__file__), "lloydmax_tables.json")


def _pdf(x):
    """Standard normal density; 0 at +-inf."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    fin = np.isfinite(x)
    out[fin] = _INV_SQRT_2PI * np.exp(-0.5 * x[fin] * x[fin])
    return out


def _upper_tail(x):
    """Q(x) = P(X > x) = erfc(x / sqrt 2) / 2, accurate in the far tails."""
    return 0.5 * erfc(np.asarray(x, dtype=np.float64) / _SQRT2)


def interval_stats(t):
    """Probability and conditional mean of the cells cut by thresholds ``t``.

    Cells are (-inf, t0], (t0, t1], ..., (t_{L-2}, inf).
    """
    a = np.concatenate([[-np.inf], t])
    b = np.concatenate([t, [np.inf]])
    p = _upper_tail(a) - _upper_tail(b)
    mean = (_pdf(a) - _pdf(b)) / p
    return p, mean


def solve(bits: int, tol: float = 1e-13, max_iter: int = 400_000):
    """Lloyd-Max centroids (fp64, ascending) and distortion for ``bits``.

    Returns (centroids, D, iterations). Iterates until the largest centroid
    move is below ``tol`` or stops improving (fp64 noise floor, ~1e-11 at
    b = 8).
    """
    if bits < 1 or bits > B_MAX:
        raise ValueError("bits must be in 1..8")
    levels = 1 << bits
    c = ndtri((np.arange(levels) + 0.5) / levels)
    best = np.inf
    stall = 0
    it = 0
    for it in range(1, max_iter + 1):
        t = 0.5 * (c[1:] + c[:-1])
        _, c_new = interval_stats(t)
        move = float(np.max(np.abs(c_new - c)))
        c = c_new
        if move < tol:
            break
        if move < best * 0.999:
            best = move
            stall = 0
        else:
            stall += 1
            if stall > 2000 and best < 1e-10:
                break
    c = 0.5 * (c - c[::-1])  # exact symmetry c[m] = -c[L-1-m]
    return c, distortion(c), it


def distortion(c):
    """E[(X - q(X))^2] for X ~ N(0,1) with centroids ``c`` and midpoint cells.

    Per cell (a, b] with centroid c:  (1 + c^2) P - 2 c (phi(a) - phi(b))
    + a phi(a) - b phi(b)  (integrate x^2, x and 1 against phi).
    """
    c = np.asarray(c, dtype=np.float64)
    t = 0.5 * (c[1:] + c[:-1])
    a = np.concatenate([[-np.inf], t])
    b = np.concatenate([t, [np.inf]])
    p = _upper_tail(a) - _upper_tail(b)
    fa, fb = _pdf(a), _pdf(b)
    afa = np.where(np.isfinite(a), a, 0.0) * fa
    bfb = np.where(np.isfinite(b), b, 0.0) * fb
    cell = (1.0 + c * c) * p - 2.0 * c * (fa - fb) + afa - bfb
    return float(np.sum(cell))


def freeze(c):
    """fp16-exact centroids (as fp64) and fp32 midpoint thresholds."""
    c16 = np.asarray(c, dtype=np.float64).astype(np.float16).astype(np.float64)
    thr = ((c16[1:] + c16[:-1]) * 0.5).astype(np.float32)
    # the midpoint of two fp16 numbers is exact in fp32
    assert np.all(thr.astype(np.float64) == (c16[1:] + c16[:-1]) * 0.5)
    return c16, thr


def build_tables():
    """Solve b = 1..8 and return the frozen tables as a JSON-ready dict."""
    out = {"D": [1.0], "centroids": [[0.0]], "centroids_fp64": [[0.0]]}
    for b in range(1, B_MAX + 1):
        c, d, _ = solve(b)
        c16, _ = freeze(c)
        out["D"].append(d)
        out["centroids"].append([float(x) for x in c16])
        out["centroids_fp64"].append([float(x) for x in c])
    return out


_CACHE = None


def tables():
    """Frozen tables: D[0..8], fp16-exact centroids[b], solver centroids[b].

    Read from ``lloydmax_tables.json`` (written by ``oracle/gen_tables.py``,
    which calls only this module); solved on the spot if that file is absent.
    """
    global _CACHE
    if _CACHE is None:
        if os.path.exists(_TABLE_FILE):
            with open(_TABLE_FILE) as f:
                _CACHE = json.load(f)
        else:
            _CACHE = build_tables()
    return _CACHE


def D(bits: int) -> float:
    """Distortion model D(b) of the greedy allocator; D(0) = 1."""
    return float(tables()["D"][bits])


def centroids(bits: int) -> np.ndarray:
    """fp16-exact frozen centroids (fp64 array, ascending), 2^bits entries."""
    return np.asarray(tables()["centroids"][bits], dtype=np.float64)


def thresholds(bits: int) -> np.ndarray:
    """fp32 thresholds (midpoints of the frozen centroids), 2^bits - 1 entries."""
    c16 = centroids(bits)
    return ((c16[1:] + c16[:-1]) * 0.5).astype(np.float32)
