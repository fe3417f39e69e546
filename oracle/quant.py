"""TQ-MSE style quantizers for keys and values (oracle; test infrastructure).

"RoPE-Aware Bit Allocation for KV-Cache Quantization", abstract: Block-GTQ is a
bit allocator for key-cache quantization built on TurboQuant-MSE; keys get
per-RoPE-block integer widths, values keep the uniform TQ-MSE quantizer at the
matched value budget. TQ-MSE normalises a vector, rotates it so coordinates
are near Gaussian, and applies an MSE-optimal scalar codebook per coordinate.
The related-papers page ("Related papers: Quantization Dominates Rank
Reduction for KV-Cache...", the KV/KQV/QKQV scheme summary) and the KVLinC
summary (Hadamard rotation on values) support a Walsh-Hadamard rotation.

Readings adopted:

Keys (per token, per KV head). No rotation across blocks of different widths
(it would mix the blocks whose widths differ); optionally a rotation inside
each group of equal width (``quantize_keys``). n = fp16 norm of the whole 128-vector; each
coordinate i of block j is scaled to z_i = k_i * (1/n) * g_j and coded with
the width-b_j Lloyd-Max thresholds.

Values. y = H (s . v), H the unnormalised 128-point Sylvester Hadamard matrix,
s the +-1 signs of the plan; n = fp16 norm of v; z_i = y_i * (1/n) (each y_i
has variance |v|^2); coded with the uniform width b_V.

Decision arithmetic (IEEE fp32, no fused multiply-add, fixed order):
* the input is bf16/fp16/fp32; x*x is exact in fp32 for bf16 and fp16 inputs;
* sumsq: with lane l = 0..31 holding coordinates l, l+32, l+64, l+96,
  p_l = ((x_l^2 + x_{l+32}^2) + x_{l+64}^2) + x_{l+96}^2, then for
  m = 16, 8, 4, 2, 1: p_l <- p_l + p_{l xor m}; the sum is p_0;
* n = fp16_RNE(sqrt_RN(sumsq)); if that overflows, n = 65504 and the
  NORM_SAT flag is raised; r = 1/n rounded to nearest;
* keys: z_i = (k_i * r) * g_j; values: z_i = y_i * r;
* code = number of thresholds t with t < z (strict), i.e. ties go low;
* n = 0 gives all codes 0; a token with any non-finite coordinate is stored
  as n = 0, codes 0, and raises NONFINITE;
* FWHT: stages h = 1, 2, 4, ..., 64; for every i with (i & h) == 0 the pair
  (a, b) = (x_i, x_{i+h}) becomes (a + b, a - b), in fp32.
"""
from __future__ import annotations

import numpy as np

from . import lloydmax

FLAG_NONFINITE = 2
FLAG_NORM_SAT = 4
F16_MAX = 65504.0


def sumsq_tree(x32: np.ndarray) -> np.ndarray:
    """Fixed-order fp32 sum of squares over the last axis (length 128)."""
    x32 = np.asarray(x32, dtype=np.float32)
    # an fp32 overflow to inf is the defined result here (the norm then
    # saturates and the token is flagged), so numpy's warning is silenced
    with np.errstate(over="ignore"):
        sq = x32 * x32
        p = ((sq[..., 0:32] + sq[..., 32:64]) + sq[..., 64:96]) + sq[..., 96:128]
        lane = np.arange(32)
        for m in (16, 8, 4, 2, 1):
            p = p + p[..., lane ^ m]
    return p[..., 0]


def fp16_norm(sumsq: np.ndarray):
    """(n as float32 holding an fp16 value, NORM_SAT mask)."""
    s = np.sqrt(np.asarray(sumsq, dtype=np.float32))
    with np.errstate(over="ignore"):
        n16 = s.astype(np.float16)
    sat = np.isinf(n16)
    n16 = np.where(sat, np.float16(F16_MAX), n16)
    return n16.astype(np.float32), sat


def codes_from_z(z: np.ndarray, bits: int) -> np.ndarray:
    """Number of width-``bits`` thresholds strictly below z (NaN -> 0)."""
    thr = lloydmax.thresholds(bits)
    c = np.searchsorted(thr, np.asarray(z, dtype=np.float32), side="left")
    return np.where(np.isnan(z), 0, c).astype(np.int64)


def fwht_f32(x: np.ndarray) -> np.ndarray:
    """Unnormalised Walsh-Hadamard transform along the last axis, fp32 graph.

    Stage h views the last axis as (d / 2h, 2, h): the pair (a, b) of each
    butterfly is (x_i, x_{i+h}) with (i & h) == 0, replaced by (a + b, a - b).
    """
    y = np.array(x, dtype=np.float32, copy=True)
    d = y.shape[-1]
    lead = y.shape[:-1]
    h = 1
    while h < d:
        v = y.reshape(*lead, d // (2 * h), 2, h)
        a = v[..., 0, :]
        b = v[..., 1, :]
        y = np.stack([a + b, a - b], axis=-2).reshape(*lead, d)
        h *= 2
    return y


def _norm_and_recip(x32):
    """Per-token n (fp16 value in float32), r = 1/n, and flags."""
    fin = np.all(np.isfinite(x32), axis=-1)
    x_safe = np.where(fin[..., None], x32, np.float32(0))
    n, sat = fp16_norm(sumsq_tree(x_safe))
    n = np.where(fin, n, np.float32(0))
    with np.errstate(divide="ignore"):
        r = np.float32(1.0) / n
    flags = np.where(~fin, FLAG_NONFINITE, 0) | np.where(sat & fin, FLAG_NORM_SAT, 0)
    return n, r, fin, flags


def rot_scale(size: int) -> np.float32:
    """fp32 factor of a rotation chunk of 2^e positions: 2^-floor(e/2), times
    fp32(sqrt(1/2)) for odd e (an exact power-of-two scaling of one fp32)."""
    e = int(size).bit_length() - 1
    base = np.float32(np.sqrt(0.5)) if e % 2 else np.float32(1.0)
    return np.float32(np.ldexp(base, -(e // 2)))


def quantize_keys(k, plan):
    """Key codes [T, 128] (canonical coords; unused for width-0 blocks), fp16
    norms as float32 [T], per-token flags [T].

    With plan.k_rot (per-width-group rotation): z is formed as without it;
    then per plan position P = 2 r + e (coordinate order[r] + 64 e),
    u_P = s_P z_P; each chunk of ``alloc.rot_chunks`` takes the fp32 FWHT
    graph over its positions and y_P = fp32(h_P * rot_scale(size)); the code
    of position P (width of its group) is stored at coordinate order[r] + 64 e."""
    k32 = np.asarray(k, dtype=np.float32)
    T, d = k32.shape
    half = d // 2
    n, r, fin, flags = _norm_and_recip(k32)
    codes = np.zeros((T, d), dtype=np.int64)
    live = fin & (n > 0)
    if getattr(plan, "k_rot", False):
        from .alloc import rot_chunks
        order = list(plan.order)
        coord = [order[P // 2] + half * (P % 2) for P in range(2 * len(order))]
        with np.errstate(invalid="ignore", over="ignore"):
            u = np.zeros((T, 2 * len(order)), dtype=np.float32)
            for P, i in enumerate(coord):
                z = (k32[:, i] * r) * plan.g[i % half]
                u[:, P] = -z if plan.k_signs[P] < 0 else z
            for P0, sz, w in rot_chunks(plan.widths, order):
                y = fwht_f32(u[:, P0:P0 + sz]) * rot_scale(sz)
                for q in range(sz):
                    codes[:, coord[P0 + q]] = np.where(live, codes_from_z(y[:, q], w), 0)
        return codes, n, flags
    with np.errstate(invalid="ignore", over="ignore"):
        for j in range(half):
            w = int(plan.widths[j])
            if w == 0:
                continue
            for i in (j, j + half):
                z = (k32[:, i] * r) * plan.g[j]
                codes[:, i] = np.where(live, codes_from_z(z, w), 0)
    return codes, n, flags


def quantize_values(v, plan):
    """Value codes [T, 128] (rotated coords), fp16 norms [T], flags [T]."""
    v32 = np.asarray(v, dtype=np.float32)
    n, r, fin, flags = _norm_and_recip(v32)
    sv = np.where(plan.signs[None, :] < 0, -v32, v32).astype(np.float32)
    y = fwht_f32(np.where(fin[:, None], sv, np.float32(0)))
    with np.errstate(invalid="ignore", over="ignore"):
        z = y * r[:, None]
    live = fin & (n > 0)
    codes = np.where(live[:, None], codes_from_z(z, plan.bits_v), 0)
    return codes, n, flags
