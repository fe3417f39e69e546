"""Greedy marginal-gain bit allocation and the per-head plan (oracle).

Test infrastructure only.

"RoPE-Aware Bit Allocation for KV-Cache Quantization", abstract: high-energy
RoPE blocks are more sensitive to quantization error and should receive more
bits; for each layer and KV head Block-GTQ greedily allocates integer bit
widths by marginal gain, under matched K/V bit budgets (KxVy = x bits per
dimension on keys, y on values). Readings adopted where the abstract is silent:

* Objective: minimise sum_j E_j * D(b_j), with D the Gaussian Lloyd-Max
  distortion per unit variance (``lloydmax.D``), D(0) = 1.
* Greedy: start every block at 0 bits; one step adds 1 bit per dimension to
  the block with the largest gain E_j (D(b_j) - D(b_j + 1)) among blocks below
  b_max = 8; ties go to the lowest block index; J * b_K steps, so the key
  budget (b_K bits per dimension, 2 J b_K bits per token) is met exactly.
  D is convex, so this is optimal for the separable objective.
* Key scale: a_j = sqrt(E_j / (2 sum_l E_l)) (the sum in fp64 in block
  order), the expected RMS of one coordinate of block j after dividing the
  key by its norm; the quantizer
  multiplies by g_j = fp32(1/a_j) (0 when a_j = 0) and reconstruction
  multiplies by a_hat_j = fp32(a_j).
* Plan order: blocks with b_j > 0 sorted by width (descending), then block
  index (ascending). Zero-width blocks are not stored.
* Values use the uniform width b_V on every coordinate.
* Per-width-group key rotation (optional, the alternative reading of "built
  on TQ-MSE" for keys): see ``rot_chunks`` and ``quant.quantize_keys``.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import lloydmax
from .splitmix import k_signs, v_signs

B_MAX = 8
NEAR_TIE_REL = 1e-9


def greedy(E, bits_k: int, b_max: int = B_MAX, D=lloydmax.D):
    """Greedy widths for energies ``E`` (length J) and budget ``bits_k``.

    Returns (widths as int array, near_tie flag). ``near_tie`` is True when a
    step's best and runner-up gains differed by less than 1e-9 relative
    (the decision could flip under a different fp64 rounding of D).
    """
    E = [float(e) for e in E]
    J = len(E)
    if not (0 <= bits_k <= b_max):
        raise ValueError("bits_k out of range")
    b = [0] * J
    near_tie = False
    for _ in range(J * bits_k):
        best_j, best_g, second_g = -1, -np.inf, -np.inf
        for j in range(J):
            if b[j] >= b_max:
                continue
            g = E[j] * (D(b[j]) - D(b[j] + 1))
            if g > best_g:
                second_g = best_g
                best_j, best_g = j, g
            elif g > second_g:
                second_g = g
        if np.isfinite(second_g) and best_g > 0 and (best_g - second_g) <= NEAR_TIE_REL * best_g \
                and best_g != second_g:
            near_tie = True
        b[best_j] += 1
    return np.array(b, dtype=np.int64), near_tie


def objective(E, widths, D=lloydmax.D) -> float:
    return float(sum(float(e) * D(int(w)) for e, w in zip(E, widths)))


def key_scales(E):
    """(g, a_hat) as float32 arrays from energies ``E`` (length J)."""
    E = np.asarray(E, dtype=np.float64)
    tot = 0.0
    for e in E:                 # fp64, block order 0, 1, 2, ...
        tot += float(e)
    g = np.zeros(E.shape, dtype=np.float32)
    ah = np.zeros(E.shape, dtype=np.float32)
    for j, e in enumerate(E):
        a = float(np.sqrt(e / (2.0 * tot))) if tot > 0 else 0.0
        ah[j] = np.float32(a)
        g[j] = np.float32(1.0 / a) if a > 0 else np.float32(0.0)
    return g, ah


def plan_order(widths):
    """Blocks with nonzero width, sorted by (width desc, index asc)."""
    return sorted([j for j in range(len(widths)) if widths[j] > 0],
                  key=lambda j: (-int(widths[j]), j))


@dataclass
class Plan:
    bits_k: int
    bits_v: int
    widths: np.ndarray          # [64] int
    order: list                 # plan rank -> block index
    g: np.ndarray               # [64] float32
    a_hat: np.ndarray           # [64] float32
    signs: np.ndarray           # [128] +-1 (float64)
    energy: np.ndarray = field(default=None)
    near_tie: bool = False
    k_rot: bool = False         # per-width-group key rotation (reading D22)
    k_signs: np.ndarray = field(default=None)  # [128] +-1 by plan position

    @property
    def words_k(self) -> int:
        return 4 * self.bits_k

    @property
    def words_v(self) -> int:
        return 4 * self.bits_v


def rot_chunks(widths, order):
    """Chunks of the per-width-group key rotation, as (first position, size,
    width). Plan position P = 2 r + e is coordinate order[r] + 64 e of rank r.
    A width group is a maximal run of equal-width ranks (2 n positions); it is
    cut into chunks by the binary expansion of 2 n, largest first."""
    out = []
    r = 0
    while r < len(order):
        w = int(widths[order[r]])
        n = 1
        while r + n < len(order) and int(widths[order[r + n]]) == w:
            n += 1
        P, m = 2 * r, 2 * n
        for e in range(7, -1, -1):
            if m & (1 << e):
                out.append((P, 1 << e, w))
                P += 1 << e
        r += n
    return out


def make_plan(E, bits_k: int, bits_v: int, v_seed: int, layer: int, kv_head: int,
              uniform: bool = False, weights=None, rotate_keys: bool = False) -> Plan:
    """Plan of one (layer, KV head) from its block energies ``E[64]``.

    ``uniform=True`` gives every block the width ``bits_k`` (the same key
    bytes as the greedy plan), the uniform-allocation comparator.
    ``weights`` (query-weighted variant): the greedy runs on the products
    E_j * W_j (fp64), i.e. minimises sum_j W_j E_j D(b_j), the expected
    squared logit error when block j's error reaches the logit scaled by the
    query's block energy W_j; the key scales stay those of E.
    """
    E = np.asarray(E, dtype=np.float64)
    if uniform:
        w, tie = np.full(E.shape, bits_k, dtype=np.int64), False
    elif weights is not None:
        w, tie = greedy(E * np.asarray(weights, dtype=np.float64), bits_k)
    else:
        w, tie = greedy(E, bits_k)
    g, ah = key_scales(E)
    s = np.array(v_signs(v_seed, layer, kv_head, 2 * len(E)), dtype=np.float64)
    ks = np.array(k_signs(v_seed, layer, kv_head), dtype=np.float64) if rotate_keys else None
    return Plan(bits_k=bits_k, bits_v=bits_v, widths=w, order=plan_order(w), g=g,
                a_hat=ah, signs=s, energy=E, near_tie=tie, k_rot=rotate_keys, k_signs=ks)
