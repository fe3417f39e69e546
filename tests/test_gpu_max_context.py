"""GPU parity at the largest context of the sweep: one 512K-token layer of the
Qwen-3B shape (2 KV heads, G = 8, K3V3), bulk prefill then a fused step.

Sampled tile records bit-exact against the oracle's packing; decode outputs
against the fp64 oracle, evaluated range by range (64K tokens at a time) and
combined with the oracle's log-sum-exp combine, so the host memory stays
bounded; the fused append + decode step at 512K + 1 tokens the same way.
"""
import numpy as np
import pytest
import torch

import oracle_pipeline as op
import synth
from bit_kv_cache_19_b200 import kvq
from bit_kv_cache_19_b200.runtime import PackedLayer
from oracle import alloc, attn, layout, quant

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 2e-3
CHUNK = 65536


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(DEV)


def _oracle_decode_chunked(q, kh, vh, plans, n_kv, G):
    """fp64 decode over all tokens from per-range records (oracle combine)."""
    out = np.zeros((n_kv * G, 128))
    for h in range(n_kv):
        lses, outs = [], []
        for a in range(0, kh[h].shape[0], CHUNK):
            b = min(a + CHUNK, kh[h].shape[0])
            kc, kn, _ = quant.quantize_keys(kh[h][a:b], plans[h])
            vc, vn, _ = quant.quantize_values(vh[h][a:b], plans[h])
            lse, o = attn.range_record(q[h * G:(h + 1) * G], attn.dequant_keys(kc, kn, plans[h]),
                                       attn.dequant_values(vc, vn, plans[h]))
            lses.append(lse)
            outs.append(o)
        out[h * G:(h + 1) * G] = attn.combine_ranges(np.stack(lses), np.stack(outs))
    return out


def test_512k_layer_prefill_and_fused_step():
    wl = synth.WORKLOADS["qwen3b_sweep"]
    T = 524288
    n_kv, G = wl.n_kv_heads, wl.n_q_heads // wl.n_kv_heads
    cfg = kvq.make_cfg(n_kv, wl.bits_k, wl.bits_v, v_seed=512)
    k, v = synth.keys_values_torch(wl, 0, 4, T + 1, DEV)
    L = PackedLayer(cfg, 1, T + 32, layer=4)
    L.alloc_bits(k[:T])
    L.append(k[None, :T].contiguous(), v[None, :T].contiguous())
    torch.cuda.synchronize()
    assert int(L.lens.item()) == T and L.flags() == 0
    kf = k.float().cpu().numpy().astype(np.float64)
    vf = v.float().cpu().numpy().astype(np.float64)
    del k
    kh = [kf[:, h] for h in range(n_kv)]
    vh = [vf[:, h] for h in range(n_kv)]
    E, _ = op.energies([x[:T] for x in kh])
    assert np.array_equal(L.energy, E)
    plans = [alloc.make_plan(E[h], wl.bits_k, wl.bits_v, 512, 4, h) for h in range(n_kv)]
    rng = np.random.default_rng(2)
    n_tiles = T // 32
    tiles = np.unique(np.concatenate([rng.integers(0, n_tiles, 23), [0, n_tiles - 1]]))
    nw = 128 * (wl.bits_k + wl.bits_v)
    for h in range(n_kv):
        got = L.head_records(0, h, n_tiles)
        for t in tiles:
            sl = slice(32 * t, 32 * t + 32)
            kc, kn, _ = quant.quantize_keys(kh[h][sl], plans[h])
            vc, vn, _ = quant.quantize_values(vh[h][sl], plans[h])
            ref = layout.pack(kc, vc, kn, vn, plans[h], 32)
            assert np.array_equal(got[t, :nw], ref[0, :nw]), (h, t)
            assert np.array_equal(got[t, nw:], ref[0, nw:]), (h, t)
    # decode over the 512K tokens
    qb = synth.queries(wl, 0, 4, 0, T)
    out = L.decode(dev_bf16(qb)[None], max_len=T + 32).cpu().numpy()[0]
    q = synth.bf16_bits_to_f64(qb)
    assert op.rel_err(out, _oracle_decode_chunked(q, [x[:T] for x in kh], [x[:T] for x in vh],
                                                  plans, n_kv, G)) <= TOL
    # fused step: append token T and decode over T + 1 tokens
    qb2 = synth.queries(wl, 0, 4, 0, T + 1)
    knew = torch.from_numpy(kf[None, T:T + 1].astype(np.float32)).to(DEV).to(torch.bfloat16)
    out2 = L.append_decode(knew, v[None, T:T + 1].contiguous(), dev_bf16(qb2)[None],
                           max_len=T + 32, step_flags=kvq.STEP_EARLY).cpu().numpy()[0]
    assert int(L.lens.item()) == T + 1 and L.flags() == 0
    ref2 = _oracle_decode_chunked(synth.bf16_bits_to_f64(qb2), kh, vh, plans, n_kv, G)
    assert op.rel_err(out2, ref2) <= TOL
