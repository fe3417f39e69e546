"""A bounded wait that runs out (GPU): the decode kernel's timeout path.

Every wait of the kernels on a barrier or a copy gives up after a limit and
sets KVQ_FLAG_TIMEOUT instead of trapping or spinning. The test hook
kvq_debug_decode_stall makes each warp first wait a few microseconds on a
barrier nothing arrives on: the call must return, the status must carry
TIMEOUT, and the next normal call on the same workspace must be right
against the oracle (the timed-out launch still completed its split
reduction and left the workspace's counters and buckets at zero).
"""
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


def test_wait_that_runs_out_flags_timeout_and_leaves_workspace_usable():
    rng = np.random.default_rng(17)
    n_kv, batch, T, G = 2, 2, 3000, 8
    cfg = kvq.make_cfg(n_kv, 3, 3, v_seed=3)
    L = PackedLayer(cfg, batch, T)
    E = np.exp(rng.standard_normal((n_kv, 64)) - np.arange(64) / 8.0)
    L.set_plans(kvq.plan_build(cfg, 0, E))
    kb = synth.to_bf16_bits(rng.standard_normal((batch, T, n_kv, 128)))
    vb = synth.to_bf16_bits(rng.standard_normal((batch, T, n_kv, 128)))
    L.append(dev_bf16(kb), dev_bf16(vb))
    ws = L.workspace(n_kv * G, T)
    qb = synth.to_bf16_bits(rng.standard_normal((batch, n_kv * G, 128)))
    q = dev_bf16(qb)
    torch.cuda.synchronize()
    assert L.flags() == 0
    try:
        assert kvq.lib().kvq_debug_decode_stall(20000) == kvq.OK  # ~10 us at 2 GHz
        L.decode(q, ws=ws)
        L.decode(q, ws=ws)
        torch.cuda.synchronize()
    finally:
        assert kvq.lib().kvq_debug_decode_stall(0) == kvq.OK
    assert L.flags() & kvq.FLAG_TIMEOUT
    L.status.zero_()
    out = L.decode(q, ws=ws).cpu().numpy()
    assert L.flags() == 0
    for s in range(batch):
        kh, vh = op.bf16_heads(kb[s], vb[s])
        heads = op.layer(kh, vh, 3, 3, 3, 0, E=E, pack=False)[1]
        ref = op.decode(synth.bf16_bits_to_f64(qb[s]), heads)
        assert op.rel_err(out[s], ref) <= TOL
    assert kvq.lib().kvq_debug_decode_stall(-1) == kvq.ERR_ARG
