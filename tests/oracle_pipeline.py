"""Compose the oracle's steps for one layer (test helper; CPU only)."""
from __future__ import annotations

import numpy as np

import synth
from oracle import alloc, attn, energy, layout, quant


def energies(k_heads):
    """Block energies E[H, 64] of per-head keys (list of float arrays [T, 128])."""
    E, flags = energy.block_energy(np.stack(k_heads, axis=1))
    return E, flags


def layer(k_heads, v_heads, bits_k, bits_v, v_seed, layer_idx, uniform=False, E=None,
          window=None, pack=True, rotate_keys=False):
    """Oracle plans, tile records, dequantized caches for one layer.

    k_heads / v_heads: per KV head float arrays [T, 128] holding bf16 values.
    E: energies to use (default: computed over the first ``window`` tokens).
    pack: also build the tile records (slow at long contexts).
    """
    T = k_heads[0].shape[0]
    if E is None:
        w = T if window is None else window
        E, _ = energies([k[:w] for k in k_heads])
    out = []
    for h, (k, v) in enumerate(zip(k_heads, v_heads)):
        plan = alloc.make_plan(E[h], bits_k, bits_v, v_seed, layer_idx, h, uniform=uniform,
                               rotate_keys=rotate_keys)
        kc, kn, kf = quant.quantize_keys(k, plan)
        vc, vn, vf = quant.quantize_values(v, plan)
        rec = layout.pack(kc, vc, kn, vn, plan, T) if pack else None
        kh = attn.dequant_keys(kc, kn, plan)
        vh = attn.dequant_values(vc, vn, plan)
        out.append(dict(plan=plan, rec=rec, khat=kh, vhat=vh, kflags=kf, vflags=vf,
                        kcodes=kc, vcodes=vc, knorm=kn, vnorm=vn))
    return E, out


def decode(q, heads, length=None):
    """fp64 decode output [n_q, 128] for one sequence from oracle heads."""
    kh = [h["khat"] if length is None else h["khat"][:length] for h in heads]
    vh = [h["vhat"] if length is None else h["vhat"][:length] for h in heads]
    return attn.decode(q, kh, vh)


def rel_err(o, ref):
    """Per (sequence, head): max |o - ref| / max |ref|; returns the max over all."""
    o = np.asarray(o, dtype=np.float64).reshape(-1, 128)
    ref = np.asarray(ref, dtype=np.float64).reshape(-1, 128)
    den = np.abs(ref).max(axis=1)
    num = np.abs(o - ref).max(axis=1)
    zero = den == 0
    if np.any(zero):
        assert np.all(num[zero] == 0)
    return float(np.max(np.where(zero, 0.0, num / np.where(zero, 1.0, den))))


def bf16_heads(kb, vb):
    """bf16 bit arrays [T, H, 128] -> per-head float lists."""
    k = synth.bf16_bits_to_f64(kb)
    v = synth.bf16_bits_to_f64(vb)
    return [k[:, h] for h in range(k.shape[1])], [v[:, h] for h in range(v.shape[1])]
