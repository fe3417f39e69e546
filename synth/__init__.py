"""Seeded synthetic keys, values and queries for the KV-cache workloads.

This module is the single input source shared by the oracle and the CUDA path.
It holds no step of the quantization method: it only draws the tensors a
RoPE attention layer would hand to the cache (post-RoPE keys, values, and a
post-RoPE decode query) and rounds them to bf16 (fp64 -> fp32 RNE -> bf16
RNE). The RoPE applied here models the upstream attention layer.

Recipe (the workload shapes of Block-GTQ's evaluation: Llama-3.1-8B and
Qwen2.5-3B/7B attention layers, head size 128, 64 RoPE blocks (j, j + 64)):

* base key kappa_t: coordinates of block j drawn N(0, s_j^2), where
  - ``tiny``: s_j = exp(-j / 12);
  - the model-shaped workloads: ln s_j^2 = -j/6 + eps_j, eps_j ~ N(0, 1) per
    (layer, KV head, block) (log-normal, sigma 1, decaying with the block's
    frequency index);
* outliers: every coordinate independently with probability 0.01 is
  multiplied by 8;
* k_t = RoPE(kappa_t, position t); v_t ~ N(0, I); the decode query of each
  query head is RoPE(N(0, I), position L) for a cache of L tokens;
* seeds: numpy SeedSequence([workload id, seed, layer, kv head]) for keys and
  values, ([workload id, seed, layer, 1000 + sequence]) for queries.

``numpy`` draws (host) serve the sizes the oracle handles; ``torch`` draws
(same recipe, same per-block scales, another random stream) serve the
full-size device runs, whose sampled parity checks copy the drawn inputs back.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

D = 128
HALF = 64
OUTLIER_P = 0.01
OUTLIER_X = 8.0


@dataclass(frozen=True)
class Workload:
    name: str
    wid: int
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    context: int
    batch: int
    bits_k: int
    bits_v: int
    rope_base: float
    n_new: int = 0
    contexts: tuple = field(default=())
    block_scale: str = "lognormal"


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 4, 1, 2048, 1, 2, 2, 1e4, block_scale="exp12"),
    "llama8b": Workload("llama8b", 2, 1, 32, 8, 32768, 1, 2, 2, 5e5),
    "qwen3b_128k": Workload("qwen3b_128k", 3, 36, 16, 2, 131072, 1, 3, 3, 1e6),
    "qwen7b_serve": Workload("qwen7b_serve", 4, 28, 28, 4, 32768, 16, 3, 2, 1e6, n_new=16),
    "qwen3b_sweep": Workload("qwen3b_sweep", 5, 36, 16, 2, 131072, 1, 3, 3, 1e6,
                             contexts=(8192, 32768, 131072, 262144, 524288)),
}


# ---------------------------------------------------------------- bf16 helpers
def to_bf16_bits(x) -> np.ndarray:
    """fp64 -> fp32 (RNE) -> bf16 (RNE) as uint16 bit patterns."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    nan = np.isnan(f)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    r = np.where(nan, (u >> 16) | 0x40, r)
    return r.astype(np.uint16)


def bf16_bits_to_f64(b) -> np.ndarray:
    u = np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def _seq(*key) -> np.random.SeedSequence:
    return np.random.SeedSequence([int(k) for k in key])


def block_sigmas(wl: Workload, seed: int, layer: int, kv_head: int) -> np.ndarray:
    """Per-block standard deviations s_j, j = 0..63."""
    j = np.arange(HALF, dtype=np.float64)
    if wl.block_scale == "exp12":
        return np.exp(-j / 12.0)
    eps = np.random.default_rng(_seq(wl.wid, seed, layer, kv_head, 7)).standard_normal(HALF)
    return np.exp(0.5 * (-j / 6.0 + eps))


def _rope(x, pos, base):
    th = np.power(float(base), -2.0 * np.arange(HALF, dtype=np.float64) / D)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * th[None, :]
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[:, :HALF], x[:, HALF:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=1)


def keys_values(wl: Workload, seed: int, layer: int, kv_head: int, n_tokens: int,
                start: int = 0):
    """bf16 bits K[n, 128], V[n, 128] for positions start..start+n-1.

    Drawn for positions 0..start+n-1 and sliced, so a slice is a prefix-
    consistent part of the same sequence.
    """
    total = start + n_tokens
    rng = np.random.default_rng(_seq(wl.wid, seed, layer, kv_head))
    sig = np.concatenate([block_sigmas(wl, seed, layer, kv_head)] * 2)
    kappa = rng.standard_normal((total, D)) * sig[None, :]
    out = rng.random((total, D)) < OUTLIER_P
    kappa = np.where(out, kappa * OUTLIER_X, kappa)
    v = rng.standard_normal((total, D))
    k = _rope(kappa, np.arange(total), wl.rope_base)
    return to_bf16_bits(k[start:]), to_bf16_bits(v[start:])


def keys_pre_rope(wl: Workload, seed: int, layer: int, kv_head: int, n_tokens: int,
                  start: int = 0) -> np.ndarray:
    """bf16 bits of the same keys before RoPE (kappa of keys_values), positions
    start..start+n-1: the input of the fused rotate-and-quantize path."""
    total = start + n_tokens
    rng = np.random.default_rng(_seq(wl.wid, seed, layer, kv_head))
    sig = np.concatenate([block_sigmas(wl, seed, layer, kv_head)] * 2)
    kappa = rng.standard_normal((total, D)) * sig[None, :]
    out = rng.random((total, D)) < OUTLIER_P
    kappa = np.where(out, kappa * OUTLIER_X, kappa)
    return to_bf16_bits(kappa[start:])


def queries(wl: Workload, seed: int, layer: int, seq: int, pos: int) -> np.ndarray:
    """bf16 bits q[n_q_heads, 128] rotated at position ``pos``."""
    rng = np.random.default_rng(_seq(wl.wid, seed, layer, 1000 + seq))
    q = rng.standard_normal((wl.n_q_heads, D))
    return to_bf16_bits(_rope(q, np.full(wl.n_q_heads, pos), wl.rope_base))


def queries_anisotropic(wl: Workload, seed: int, layer: int, kv_head: int, n: int, G: int,
                        start_pos: int) -> np.ndarray:
    """bf16 bits q[n, G, 128] of one KV head's query group at positions
    start_pos..start_pos+n-1, with uneven block energy: coordinates of block j
    scaled by exp(0.75 e_j), e_j ~ N(0, 1) drawn once per (layer, KV head)
    and shared by the group and by every seed (the seed draws the samples). A
    query family for the query-weighted allocation study (the workloads' own
    queries are isotropic)."""
    sc = np.exp(0.75 * np.random.default_rng(_seq(wl.wid, layer, 2000 + kv_head)).standard_normal(HALF))
    sc = np.concatenate([sc, sc])
    rng = np.random.default_rng(_seq(wl.wid, seed, layer, 3000 + kv_head))
    q = rng.standard_normal((n, G, D)) * sc[None, None, :]
    pos = np.repeat(np.arange(start_pos, start_pos + n), G)
    return to_bf16_bits(_rope(q.reshape(n * G, D), pos, wl.rope_base).reshape(n, G, D))


# ---------------------------------------------------------------- torch draws
def _torch_seed(*key) -> int:
    return int(_seq(*key).generate_state(1, np.uint64)[0] & np.uint64((1 << 63) - 1))


def keys_values_torch(wl: Workload, seed: int, layer: int, n_tokens: int, device,
                      start: int = 0):
    """bf16 tensors K, V [n_tokens, n_kv_heads, 128] on ``device``."""
    import torch

    pos = torch.arange(start, start + n_tokens, device=device, dtype=torch.float64)
    th = torch.tensor(np.power(float(wl.rope_base), -2.0 * np.arange(HALF) / D),
                      device=device, dtype=torch.float64)
    ang = pos[:, None] * th[None, :]
    c, s = torch.cos(ang), torch.sin(ang)
    ks, vs = [], []
    for h in range(wl.n_kv_heads):
        g = torch.Generator(device=device)
        g.manual_seed(_torch_seed(wl.wid, seed, layer, h, start))
        sig = np.concatenate([block_sigmas(wl, seed, layer, h)] * 2)
        sig_t = torch.tensor(sig, device=device, dtype=torch.float64)
        kappa = torch.randn((n_tokens, D), generator=g, device=device, dtype=torch.float64) * sig_t
        u = torch.rand((n_tokens, D), generator=g, device=device, dtype=torch.float64)
        kappa = torch.where(u < OUTLIER_P, kappa * OUTLIER_X, kappa)
        v = torch.randn((n_tokens, D), generator=g, device=device, dtype=torch.float64)
        a, b = kappa[:, :HALF], kappa[:, HALF:]
        k = torch.cat([a * c - b * s, a * s + b * c], dim=1)
        ks.append(k.to(torch.float32).to(torch.bfloat16))
        vs.append(v.to(torch.float32).to(torch.bfloat16))
        del kappa, u, v, k, a, b
    return torch.stack(ks, dim=1), torch.stack(vs, dim=1)


def queries_torch(wl: Workload, seed: int, layer: int, batch: int, pos: int, device):
    """bf16 tensor q[batch, n_q_heads, 128] rotated at position ``pos``."""
    import torch

    qs = [torch.from_numpy(queries(wl, seed, layer, b, pos).view(np.int16)) for b in range(batch)]
    return torch.stack(qs).view(torch.bfloat16).to(device)
