"""GPU: context-sharded decode (kvq_decode_attn_partial + kvq_combine_partials)
through the C ABI against the oracle.

A sequence's cache is split by token ranges into separate caches (as one per
GPU would hold them); each range is decoded into records and the stacked
records are combined. Checked: the combined output against the fp64 oracle
over all tokens (max relative error 2e-3 per head, as for kvq_decode_attn)
and against the single-cache GPU decode; each range alone (a combine of its
record) against the oracle's attention over the range; the record's
log-sum-exp m + log2 l against the oracle's; empty ranges.
"""
import numpy as np
import pytest
import torch

import oracle_pipeline as op
import synth
from bit_kv_cache_19_b200 import kvq
from bit_kv_cache_19_b200.runtime import PackedLayer
from oracle import attn

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 2e-3


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(DEV)


def _shard_layers(cfg, plans, kb, vb, cuts):
    """One PackedLayer (batch of one) per token range [a, b) of kb / vb."""
    shards = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        L = PackedLayer(cfg, 1, max(b - a, 1))
        L.set_plans(plans)
        if b > a:
            L.append(dev_bf16(kb[a:b])[None], dev_bf16(vb[a:b])[None])
        shards.append(L)
    return shards


def _check(cfg, E, kb, vb, qb, cuts, layer_idx, v_seed):
    T = kb.shape[0]
    n_kv, G = cfg.n_kv_heads, qb.shape[0] // cfg.n_kv_heads
    plans = kvq.plan_build(cfg, layer_idx, E)
    kh, vh = op.bf16_heads(kb, vb)
    _, heads = op.layer(kh, vh, cfg.bits_k, cfg.bits_v, v_seed, layer_idx, E=E, pack=False)
    q = synth.bf16_bits_to_f64(qb)
    qd = dev_bf16(qb)[None]

    shards = _shard_layers(cfg, plans, kb, vb, cuts)
    recs = torch.stack([L.decode_partial(qd) for L in shards])
    out = shards[0].combine(recs).cpu().numpy()[0]
    torch.cuda.synchronize()
    assert all(L.flags() == 0 for L in shards)
    assert op.rel_err(out, op.decode(q, heads)) <= TOL

    full = PackedLayer(cfg, 1, T)
    full.set_plans(plans)
    full.append(dev_bf16(kb)[None], dev_bf16(vb)[None])
    ref_gpu = full.decode(qd).cpu().numpy()[0]
    # P' = p n^V enters the value MMA in fp16 (relative rounding <= 2^-11 per
    # weight) and p depends on each split's running max, so two partitions of
    # the same context agree to about that, not to fp32 rounding
    assert op.rel_err(out, ref_gpu) <= 1e-3

    r_host = recs.cpu().numpy()[:, 0]
    for i, (a, b) in enumerate(zip(cuts[:-1], cuts[1:])):
        one = shards[0].combine(recs[i:i + 1].contiguous()).cpu().numpy()[0]
        if b == a:
            assert np.all(r_host[i, :, 0] == -np.inf) and np.all(r_host[i, :, 1] == 0)
            assert np.all(one == 0)
            continue
        for h in range(n_kv):
            sl = slice(h * G, (h + 1) * G)
            lse, o = attn.range_record(q[sl], heads[h]["khat"][a:b], heads[h]["vhat"][a:b])
            assert op.rel_err(one[sl], o) <= TOL, (a, b, h)
            got_lse = r_host[i, sl, 0] + np.log2(r_host[i, sl, 1])
            assert np.max(np.abs(got_lse - lse)) <= 1e-3, (a, b, h)


@pytest.mark.parametrize("bits_k,bits_v,G,cuts", [
    (3, 3, 8, [0, 1000, 1000, 2017, 3000]),   # an empty range, ragged ends
    (2, 2, 4, [0, 1, 33, 3000]),              # one-token and partial-tile ranges
    (4, 2, 7, [0, 1500, 3000]),
    (3, 3, 16, [0, 700, 1800, 1800, 3000]),  # two query groups per CTA (G = 16)
])
def test_shards_combine_to_whole_context(bits_k, bits_v, G, cuts):
    rng = np.random.default_rng(bits_k * 10 + G)
    n_kv, T = 2, cuts[-1]
    cfg = kvq.make_cfg(n_kv, bits_k, bits_v, v_seed=21)
    E = np.exp(1.5 * rng.standard_normal((n_kv, 64)) - np.arange(64) / 8.0)
    sig = np.sqrt(np.concatenate([E, E], axis=1) / 2)
    kb = synth.to_bf16_bits(rng.standard_normal((T, n_kv, 128)) * sig[None])
    vb = synth.to_bf16_bits(rng.standard_normal((T, n_kv, 128)))
    qb = synth.to_bf16_bits(rng.standard_normal((n_kv * G, 128)) * 2.0)
    _check(cfg, E, kb, vb, qb, cuts, 4, 21)


def test_qwen3b_layer_two_shards():
    """A 64K-token slice of the Qwen-3B-shaped workload (2 KV heads, G = 8,
    K3V3) split over two shards of 32K."""
    wl = synth.WORKLOADS["qwen3b_128k"]
    T = 65536
    kv = [synth.keys_values(wl, 0, 7, h, T) for h in range(wl.n_kv_heads)]
    kb = np.stack([x[0] for x in kv], 1)
    vb = np.stack([x[1] for x in kv], 1)
    kh, _ = op.bf16_heads(kb, vb)
    E, _ = op.energies(kh)
    cfg = kvq.make_cfg(wl.n_kv_heads, wl.bits_k, wl.bits_v, v_seed=3)
    qb = synth.queries(wl, 0, 7, 0, T)
    _check(cfg, E, kb, vb, qb, [0, T // 2, T], 7, 3)
