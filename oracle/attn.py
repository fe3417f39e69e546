"""Dequantization and exact decode attention in fp64 (oracle; test only).

"RoPE-Aware Bit Allocation for KV-Cache Quantization", abstract: the
packed-cache serving path runs decode attention over the packed K/V cache.
Here that is written as its plain definition on the dequantized cache:

    k_hat_i = n^K * a_hat_j * c_{b_j}[code_i]          (0 for b_j = 0)
    v_hat   = n^V * (1/d) * s . (H c_{b_V}[codes])      (H H = d I)
    o_h     = sum_t softmax_t(q_h . k_hat_t / sqrt d) v_hat_t

over the L cached tokens (no mask: a decode query attends to every cached
token). Query head h reads KV head floor(h / G), G = H_q / H_kv. A sequence
with no cached token gives o = 0.
"""
from __future__ import annotations

import numpy as np

from . import lloydmax


def hadamard(d: int = 128) -> np.ndarray:
    """Sylvester Hadamard matrix, H[i, j] = (-1)^popcount(i & j)."""
    i = np.arange(d)
    x = i[:, None] & i[None, :]
    pc = np.zeros_like(x)
    while np.any(x):
        pc += x & 1
        x >>= 1
    return np.where(pc % 2 == 0, 1.0, -1.0)


def dequant_keys(codes, norms, plan) -> np.ndarray:
    codes = np.asarray(codes)
    T, d = codes.shape
    half = d // 2
    out = np.zeros((T, d), dtype=np.float64)
    n = np.asarray(norms, dtype=np.float64)
    if getattr(plan, "k_rot", False):
        # per chunk: z = s . (H y_hat) / sqrt(size) (the orthonormal inverse)
        from .alloc import rot_chunks
        order = list(plan.order)
        coord = [order[P // 2] + half * (P % 2) for P in range(2 * len(order))]
        for P0, sz, w in rot_chunks(plan.widths, order):
            c = lloydmax.centroids(w)
            yh = np.stack([c[codes[:, coord[P0 + q]]] for q in range(sz)], axis=1)
            zh = (yh @ hadamard(sz)) / np.sqrt(sz) * plan.k_signs[P0:P0 + sz][None, :]
            for q in range(sz):
                i = coord[P0 + q]
                out[:, i] = n * float(plan.a_hat[i % half]) * zh[:, q]
        return out
    for j in range(half):
        w = int(plan.widths[j])
        if w == 0:
            continue
        c = lloydmax.centroids(w)
        for i in (j, j + half):
            out[:, i] = n * float(plan.a_hat[j]) * c[codes[:, i]]
    return out


def dequant_values(codes, norms, plan) -> np.ndarray:
    codes = np.asarray(codes)
    d = codes.shape[1]
    c = lloydmax.centroids(plan.bits_v)
    y = c[codes] * np.asarray(norms, dtype=np.float64)[:, None]
    return (y @ hadamard(d)) * plan.signs[None, :] / d


def attention(q, k_hat, v_hat) -> np.ndarray:
    """softmax(q k_hat^T / sqrt d) v_hat for one KV head; q[Hg, d]."""
    q = np.asarray(q, dtype=np.float64)
    if k_hat.shape[0] == 0:
        return np.zeros_like(q)
    s = q @ k_hat.T / np.sqrt(q.shape[-1])
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    return p @ v_hat


def decode(q, k_hat_heads, v_hat_heads) -> np.ndarray:
    """GQA decode for one sequence: q[Hq, d], per-KV-head dequantized caches."""
    q = np.asarray(q, dtype=np.float64)
    hkv = len(k_hat_heads)
    G = q.shape[0] // hkv
    out = np.zeros_like(q)
    for h in range(hkv):
        out[h * G:(h + 1) * G] = attention(q[h * G:(h + 1) * G], k_hat_heads[h], v_hat_heads[h])
    return out


# Context shards. Softmax over a sequence split into disjoint token ranges is
# the log-sum-exp-weighted mix of the ranges' own softmax outputs; this is the
# plain identity, written out in base 2 (the library keeps base-2 logits).
def range_record(q, k_hat, v_hat):
    """Statistics of one token range for one KV head; q[Hg, d].

    lse2_h = log2 sum_t 2^{s_t}, s_t = q_h . k_hat_t log2(e) / sqrt d, and the
    range's own output o_h = sum_t 2^{s_t - lse2_h} v_hat_t. An empty range
    gives lse2 = -inf and o = 0."""
    q = np.asarray(q, dtype=np.float64)
    if k_hat.shape[0] == 0:
        return np.full(q.shape[0], -np.inf), np.zeros_like(q)
    s = q @ k_hat.T / np.sqrt(q.shape[-1]) * np.log2(np.e)
    m = s.max(axis=1, keepdims=True)
    w = np.exp2(s - m)
    lse2 = m[:, 0] + np.log2(w.sum(axis=1))
    return lse2, np.exp2(s - lse2[:, None]) @ v_hat


def combine_ranges(lse2, o):
    """Output over the union of disjoint ranges from their records.

    lse2[R, Hg], o[R, Hg, d]: o = sum_r 2^{lse2_r - LSE} o_r with
    LSE = log2 sum_r 2^{lse2_r}; ranges with lse2 = -inf add nothing, and if
    every range is empty the output is 0."""
    lse2 = np.asarray(lse2, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    m = lse2.max(axis=0)
    out = np.zeros(o.shape[1:])
    for h in range(lse2.shape[1]):
        if m[h] == -np.inf:
            continue
        w = np.exp2(lse2[:, h] - m[h])
        out[h] = (w[:, None] * o[:, h]).sum(axis=0) / w.sum()
    return out
