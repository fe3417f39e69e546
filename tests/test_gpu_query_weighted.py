"""GPU: query-weighted allocation variant through the C ABI.

kvq_block_energy of calibration queries equals the oracle's exact integer
block energy bit for bit; PackedLayer.alloc_bits_query_weighted builds the
oracle's weighted plans; a cache quantized under such a plan decodes within
the usual tolerance of the fp64 oracle.
"""
import numpy as np
import pytest
import torch

import oracle_pipeline as op
import synth
from bit_kv_cache_19_b200 import kvq
from bit_kv_cache_19_b200.runtime import PackedLayer
from oracle import alloc, attn, energy, quant

pytestmark = pytest.mark.gpu
DEV = "cuda"


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(DEV)


def test_query_weighted_plans_and_decode():
    wl = synth.WORKLOADS["llama8b"]
    T, n_kv = 4096, wl.n_kv_heads
    G = wl.n_q_heads // n_kv
    kv = [synth.keys_values(wl, 0, 2, h, T) for h in range(n_kv)]
    kb = np.stack([x[0] for x in kv], 1)
    vb = np.stack([x[1] for x in kv], 1)
    qc = np.concatenate([synth.queries_anisotropic(wl, 0, 2, h, 300, G, T) for h in range(n_kv)],
                        axis=1)                                   # [300, n_q, 128]
    cfg = kvq.make_cfg(n_kv, wl.bits_k, wl.bits_v, v_seed=2)
    L = PackedLayer(cfg, 1, T, layer=2)
    plans = L.alloc_bits_query_weighted(dev_bf16(kb), dev_bf16(qc))
    kh, vh = op.bf16_heads(kb, vb)
    E, _ = op.energies(kh)
    assert np.array_equal(L.energy, E)
    Eq_gpu = kvq.block_energy(dev_bf16(qc))
    Eq, _ = energy.block_energy(synth.bf16_bits_to_f64(qc))
    assert np.array_equal(Eq_gpu, Eq)
    W, _ = energy.query_weights(synth.bf16_bits_to_f64(qc), n_kv)
    for h in range(n_kv):
        ref = alloc.make_plan(E[h], wl.bits_k, wl.bits_v, 2, 2, h, weights=W[h])
        assert np.array_equal(plans[h]["width"].astype(int), ref.widths)
        assert np.array_equal(plans[h]["g"], ref.g)
    L.append(dev_bf16(kb)[None], dev_bf16(vb)[None])
    q = synth.queries_anisotropic(wl, 1, 2, 0, 1, wl.n_q_heads, T)[0]
    out = L.decode(dev_bf16(q)[None], max_len=T).cpu().numpy()[0]
    assert L.flags() == 0
    heads = []
    for h in range(n_kv):
        plan = alloc.make_plan(E[h], wl.bits_k, wl.bits_v, 2, 2, h, weights=W[h])
        kc, kn, _ = quant.quantize_keys(kh[h], plan)
        vc, vn, _ = quant.quantize_values(vh[h], plan)
        heads.append(dict(khat=attn.dequant_keys(kc, kn, plan),
                          vhat=attn.dequant_values(vc, vn, plan)))
    assert op.rel_err(out, op.decode(synth.bf16_bits_to_f64(q), heads)) <= 2e-3
