"""Deterministic decode mode (GPU): with kvq_set_decode_deterministic(1) the
split records are merged in split order, so repeated decodes of the same
inputs give identical bits (the default sums splits by L2 atomics in arrival
order and agrees only to fp32 rounding); the outputs stay within 2e-3 of the
fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle_pipeline as op
import synth
from bit_kv_cache_19_b200 import kvq
from bit_kv_cache_19_b200.runtime import PackedLayer
from test_gpu_parity import dev_bf16

pytestmark = pytest.mark.gpu
TOL = 2e-3


def test_deterministic_decode_repeats_bit_for_bit():
    rng = np.random.default_rng(29)
    n_kv, batch, T, G = 2, 2, 20000, 8
    cfg = kvq.make_cfg(n_kv, 3, 3, v_seed=2)
    L = PackedLayer(cfg, batch, T)
    E = np.exp(rng.standard_normal((n_kv, 64)) - np.arange(64) / 8.0)
    L.set_plans(kvq.plan_build(cfg, 0, E))
    kb = synth.to_bf16_bits(rng.standard_normal((batch, T, n_kv, 128)))
    vb = synth.to_bf16_bits(rng.standard_normal((batch, T, n_kv, 128)))
    L.append(dev_bf16(kb), dev_bf16(vb))
    qb = synth.to_bf16_bits(rng.standard_normal((batch, n_kv * G, 128)))
    q = dev_bf16(qb)
    ws = L.workspace(n_kv * G, T)
    try:
        assert kvq.lib().kvq_set_decode_deterministic(1) == kvq.OK
        outs = [L.decode(q, ws=ws).cpu().numpy() for _ in range(4)]
    finally:
        kvq.lib().kvq_set_decode_deterministic(0)
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])
    assert L.flags() == 0
    for s in range(batch):
        kh, vh = op.bf16_heads(kb[s], vb[s])
        heads = op.layer(kh, vh, 3, 3, 2, 0, E=E, pack=False)[1]
        ref = op.decode(synth.bf16_bits_to_f64(qb[s]), heads)
        assert op.rel_err(outs[0][s], ref) <= TOL
    # the default mode after it, on the same workspace, still agrees to rounding
    o = L.decode(q, ws=ws).cpu().numpy()
    assert op.rel_err(o, outs[0]) <= 1e-5 and L.flags() == 0


def test_deterministic_fused_step_repeats():
    # the fused append + decode step in deterministic mode: two layers fed
    # the same inputs end with the same records and the same outputs
    rng = np.random.default_rng(30)
    n_kv, T, G = 2, 9000, 8
    cfg = kvq.make_cfg(n_kv, 3, 2, v_seed=4)
    E = np.exp(rng.standard_normal((n_kv, 64)))
    kb = synth.to_bf16_bits(rng.standard_normal((1, T, n_kv, 128)))
    vb = synth.to_bf16_bits(rng.standard_normal((1, T, n_kv, 128)))
    kn = dev_bf16(synth.to_bf16_bits(rng.standard_normal((1, 3, n_kv, 128))))
    vn = dev_bf16(synth.to_bf16_bits(rng.standard_normal((1, 3, n_kv, 128))))
    q = dev_bf16(synth.to_bf16_bits(rng.standard_normal((1, n_kv * G, 128))))
    outs, layers = [], []
    try:
        kvq.lib().kvq_set_decode_deterministic(1)
        for _ in range(2):
            L = PackedLayer(cfg, 1, T + 64)
            L.set_plans(kvq.plan_build(cfg, 0, E))
            L.append(dev_bf16(kb), dev_bf16(vb))
            outs.append(L.append_decode(kn, vn, q).cpu().numpy())
            layers.append(L)
    finally:
        kvq.lib().kvq_set_decode_deterministic(0)
    assert np.array_equal(outs[0], outs[1])
    assert torch.equal(layers[0].caches[0], layers[1].caches[0])
    assert all(L.flags() == 0 and int(L.lens.item()) == T + 3 for L in layers)
