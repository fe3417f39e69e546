"""One decode workspace shared by calls of different shapes (GPU).

kvq.h promises that a zero-filled workspace sized for the largest
batch x n_kv_heads serves any sequence of kvq_decode_attn calls on one stream,
whatever their max_len or query-head count: the per-(sequence, KV head)
counter and bucket blocks sit at fixed distances from the end and the split
records never reach them. Each call is checked against the fp64 oracle.
"""
import numpy as np
import pytest
import torch

import oracle_pipeline as op
import synth
from bit_kv_cache_19_b200 import kvq
from bit_kv_cache_19_b200.runtime import PackedLayer

pytestmark = pytest.mark.gpu
TOL = 2e-3


def _bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _layer(rng, n_kv, batch, T, cap, bits_k=3, bits_v=3, v_seed=5):
    cfg = kvq.make_cfg(n_kv, bits_k, bits_v, v_seed=v_seed)
    L = PackedLayer(cfg, batch, cap)
    E = np.exp(rng.standard_normal((n_kv, 64)) - np.arange(64) / 8.0)
    L.set_plans(kvq.plan_build(cfg, 0, E))
    k = synth.to_bf16_bits(rng.standard_normal((batch, T, n_kv, 128)))
    v = synth.to_bf16_bits(rng.standard_normal((batch, T, n_kv, 128)))
    L.append(_bf16_dev(k), _bf16_dev(v))
    heads = []
    for b in range(batch):
        kh, vh = op.bf16_heads(k[b], v[b])
        heads.append(op.layer(kh, vh, bits_k, bits_v, v_seed, 0, E=E, pack=False)[1])
    return cfg, L, heads


def test_shared_workspace_across_shapes():
    rng = np.random.default_rng(31)
    layers = [_layer(rng, 2, 4, 1200, 1280), _layer(rng, 2, 1, 300, 320),
              _layer(rng, 2, 2, 2000, 2048, bits_k=2, bits_v=4)]
    # sized for the largest batch x n_kv (8 pairs); max_len / n_q do not matter
    ws = torch.zeros(kvq.decode_workspace_bytes(layers[0][0], 4, 8, 64), dtype=torch.uint8,
                     device="cuda")
    for it, (li, G) in enumerate([(0, 8), (1, 4), (2, 16), (0, 2), (1, 8), (2, 8), (0, 8)]):
        cfg, L, heads = layers[li]
        qb = synth.to_bf16_bits(rng.standard_normal((L.batch, 2 * G, 128)))
        out = L.decode(_bf16_dev(qb), ws=ws).cpu().numpy()
        q = synth.bf16_bits_to_f64(qb)
        ref = np.stack([op.decode(q[b], heads[b]) for b in range(L.batch)])
        assert op.rel_err(out, ref) <= TOL, (it, li, G)
        assert L.flags() == 0

