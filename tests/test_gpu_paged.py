"""GPU: paged caches (block table over a page pool) through the C ABI.

Pages are handed out in a shuffled order, so the sequences' pages interleave
in the pool. Checked: every tile record, gathered through the block table,
bit-exact against the oracle's packing; decode outputs against the fp64
oracle (max relative error 2e-3 per head) and against the contiguous-cache
decode of the same tokens; the fused append + decode step; refused page ids
(flagged, nothing written, no fault).
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle_pipeline as op
import synth
from bit_kv_cache_19_b200 import kvq
from bit_kv_cache_19_b200.runtime import PackedLayer, PagedLayer

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 2e-3


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(DEV)


def _row_pages(P, s):
    """kvq_pages of sequence s alone (its block-table row)."""
    return kvq.Pages(P.pool.data_ptr(), P.table.data_ptr() + 4 * s * P.table.shape[1],
                     P.n_pages, P.page_tiles, P.table.shape[1])


def _random_kv(rng, n_kv, T, E):
    sig = np.sqrt(np.concatenate([E, E], axis=1) / 2)
    kb = synth.to_bf16_bits(rng.standard_normal((T, n_kv, 128)) * sig[None])
    vb = synth.to_bf16_bits(rng.standard_normal((T, n_kv, 128)))
    return kb, vb


@pytest.mark.parametrize("bits_k,bits_v,G,page_tiles", [
    (3, 3, 8, 1), (2, 2, 4, 4), (4, 2, 7, 2), (8, 5, 16, 8)])
def test_paged_equals_contiguous_and_oracle(bits_k, bits_v, G, page_tiles):
    rng = np.random.default_rng(bits_k * 1000 + page_tiles)
    n_kv, lens = 2, [300, 33, 1000, 0]
    cfg = kvq.make_cfg(n_kv, bits_k, bits_v, v_seed=8)
    E = np.exp(1.5 * rng.standard_normal((n_kv, 64)) - np.arange(64) / 8.0)
    plans = kvq.plan_build(cfg, 2, E)
    span = 32 * page_tiles
    max_pages = -(-max(lens) // span) + 1
    n_pages = sum(-(-T // span) for T in lens) + 3
    P = PagedLayer(cfg, len(lens), n_pages, page_tiles, max_pages)
    P.set_plans(plans)
    C = PackedLayer(cfg, len(lens), max(lens) + 64)
    C.set_plans(plans)
    order = list(rng.permutation(n_pages))
    data = []
    for s, T in enumerate(lens):
        P.reserve(s, T, order=order)
    for s, T in enumerate(lens):
        kb, vb = _random_kv(rng, n_kv, T, E)
        data.append((kb, vb))
        cut = sorted({0, T // 3, T // 3 + 1, T})
        for a, b in zip(cut[:-1], cut[1:]):
            if b <= a:
                continue
            k, v = dev_bf16(kb[a:b])[None], dev_bf16(vb[a:b])[None]
            kvq.paged_quantize_append(cfg, P.plan_ptrs[s:s + 1], k, v, _row_pages(P, s),
                                      P.lens[s:s + 1], P.status)
            kvq.quantize_append(cfg, C.plan_ptrs[s:s + 1], k, v, C.cache_ptrs[s:s + 1],
                                C.lens[s:s + 1], C.cap, C.status)
    torch.cuda.synchronize()
    assert P.lens.cpu().tolist() == lens and P.flags() == 0 and C.flags() == 0
    refs = []
    for s, T in enumerate(lens):
        if T == 0:
            refs.append(None)
            continue
        kh, vh = op.bf16_heads(*data[s])
        heads = op.layer(kh, vh, bits_k, bits_v, 8, 2, E=E)[1]
        refs.append(heads)
        nt = -(-T // 32)
        for h in range(n_kv):
            got = P.head_records(s, h, nt)
            nw = 128 * (bits_k + bits_v)
            assert np.array_equal(got[:, :nw], heads[h]["rec"][:, :nw]), (s, h)
            assert np.array_equal(got, C.head_records(s, h, nt)), (s, h)
    qb = synth.to_bf16_bits(rng.standard_normal((len(lens), n_kv * G, 128)))
    q = dev_bf16(qb)
    out = P.decode(q, max_len=P.cap).cpu().numpy()
    out_c = C.decode(q, max_len=P.cap).cpu().numpy()
    assert P.flags() == 0
    for s, T in enumerate(lens):
        if T == 0:
            assert np.all(out[s] == 0)
            continue
        assert op.rel_err(out[s], op.decode(synth.bf16_bits_to_f64(qb[s]), refs[s])) <= TOL
        assert op.rel_err(out[s], out_c[s]) <= 1e-5


@pytest.mark.parametrize("flags", [0, kvq.STEP_EARLY])
def test_paged_fused_step(flags):
    """Prefill 1000 tokens per sequence, then 3 fused steps appending 16 tokens
    each (crossing page boundaries with 1-tile pages) and decoding."""
    rng = np.random.default_rng(11 + flags)
    n_kv, G, B, T0, n_new = 2, 8, 2, 1000, 16
    cfg = kvq.make_cfg(n_kv, 3, 3, v_seed=4)
    E = np.exp(rng.standard_normal((n_kv, 64)) - np.arange(64) / 10.0)
    plans = kvq.plan_build(cfg, 0, E)
    P = PagedLayer(cfg, B, 80, 1, 40)
    P.set_plans(plans)
    total = T0 + 3 * n_new
    order = list(rng.permutation(80))
    kvs = [_random_kv(rng, n_kv, total, E) for _ in range(B)]
    for s in range(B):
        P.reserve(s, total, order=order)
    kb = np.stack([x[0] for x in kvs])
    vb = np.stack([x[1] for x in kvs])
    P.append(dev_bf16(kb[:, :T0]), dev_bf16(vb[:, :T0]))
    ws = P.workspace(n_kv * G, P.cap)
    for step in range(3):
        a, b = T0 + step * n_new, T0 + (step + 1) * n_new
        qb = synth.to_bf16_bits(rng.standard_normal((B, n_kv * G, 128)))
        out = P.append_decode(dev_bf16(kb[:, a:b]), dev_bf16(vb[:, a:b]), dev_bf16(qb), ws=ws,
                              step_flags=flags).cpu().numpy()
        assert P.lens.cpu().tolist() == [b] * B and P.flags() == 0
        for s in range(B):
            kh, vh = op.bf16_heads(kvs[s][0][:b], kvs[s][1][:b])
            heads = op.layer(kh, vh, 3, 3, 4, 0, E=E, pack=step == 2)[1]
            assert op.rel_err(out[s], op.decode(synth.bf16_bits_to_f64(qb[s]), heads)) <= TOL
            if step == 2:
                nt = -(-b // 32)
                for h in range(n_kv):
                    assert np.array_equal(P.head_records(s, h, nt)[:, :768],
                                          heads[h]["rec"][:, :768])


def test_refused_pages_are_flagged():
    rng = np.random.default_rng(2)
    n_kv = 1
    cfg = kvq.make_cfg(n_kv, 3, 3, v_seed=1)
    E = np.exp(rng.standard_normal((n_kv, 64)))
    P = PagedLayer(cfg, 1, 4, 1, 8)
    P.set_plans(kvq.plan_build(cfg, 0, E))
    P.reserve(0, 64)                      # pages for tiles 0 and 1 only
    kb, vb = _random_kv(rng, n_kv, 100, E)
    before = P.pool.clone()
    # tile 2 has no page (-1): the whole append of tokens 0..99 per tile
    P.append(dev_bf16(kb)[None], dev_bf16(vb)[None])
    torch.cuda.synchronize()
    assert P.flags() & kvq.FLAG_BAD_PAGE
    tb = kvq.tile_bytes(cfg)
    # tiles 0 and 1 were written into their pages; pages 2 and 3 untouched
    assert torch.equal(P.pool[2 * tb:], before[2 * tb:])
    # decode reaching the missing page: flagged, no fault
    P.status.zero_()
    q = dev_bf16(synth.to_bf16_bits(rng.standard_normal((1, 4, 128))))
    P.decode(q, max_len=P.cap)
    torch.cuda.synchronize()
    assert P.flags() & kvq.FLAG_BAD_PAGE
    # a page id outside the pool
    P.table_host[0, 2] = 4
    P.table.copy_(torch.from_numpy(P.table_host))
    P.status.zero_()
    P.decode(q, max_len=P.cap)
    torch.cuda.synchronize()
    assert P.flags() & kvq.FLAG_BAD_PAGE


def test_paged_qwen3b_64k():
    """A 64K-token, 2-KV-head layer of the Qwen-3B-shaped workload (G = 8,
    K3V3) in 16-tile pages handed out in shuffled order."""
    wl = synth.WORKLOADS["qwen3b_128k"]
    T, page_tiles = 65536, 16
    kv = [synth.keys_values(wl, 0, 3, h, T) for h in range(wl.n_kv_heads)]
    kb = np.stack([x[0] for x in kv], 1)
    vb = np.stack([x[1] for x in kv], 1)
    kh, vh = op.bf16_heads(kb, vb)
    E, _ = op.energies(kh)
    cfg = kvq.make_cfg(wl.n_kv_heads, wl.bits_k, wl.bits_v, v_seed=6)
    n_pages = T // (32 * page_tiles)
    P = PagedLayer(cfg, 1, n_pages, page_tiles, n_pages)
    P.set_plans(kvq.plan_build(cfg, 3, E))
    P.reserve(0, T, order=list(np.random.default_rng(0).permutation(n_pages)))
    P.append(dev_bf16(kb)[None], dev_bf16(vb)[None])
    qb = synth.queries(wl, 0, 3, 0, T)
    out = P.decode(dev_bf16(qb)[None], max_len=T).cpu().numpy()[0]
    assert P.flags() == 0
    _, heads = op.layer(kh, vh, wl.bits_k, wl.bits_v, 6, 3, E=E, pack=False)
    assert op.rel_err(out, op.decode(synth.bf16_bits_to_f64(qb), heads)) <= TOL


def test_paged_context_shards_combine():
    """A sequence split into a paged shard and a contiguous shard: the combine
    of the paged partial records and the contiguous ones equals the decode of
    one cache holding every token."""
    rng = np.random.default_rng(21)
    n_kv, G, T, cut = 2, 8, 900, 420
    cfg = kvq.make_cfg(n_kv, 3, 3, v_seed=9)
    E = np.exp(rng.standard_normal((n_kv, 64)) - np.arange(64) / 9.0)
    plans = kvq.plan_build(cfg, 1, E)
    kb, vb = _random_kv(rng, n_kv, T, E)
    P = PagedLayer(cfg, 1, 20, 2, 10)
    P.set_plans(plans)
    P.reserve(0, cut, order=list(rng.permutation(20)))
    P.append(dev_bf16(kb[:cut])[None], dev_bf16(vb[:cut])[None])
    C = PackedLayer(cfg, 1, T - cut)
    C.set_plans(plans)
    C.append(dev_bf16(kb[cut:])[None], dev_bf16(vb[cut:])[None])
    F = PackedLayer(cfg, 1, T)
    F.set_plans(plans)
    F.append(dev_bf16(kb)[None], dev_bf16(vb)[None])
    qb = synth.to_bf16_bits(rng.standard_normal((1, n_kv * G, 128)))
    q = dev_bf16(qb)
    recs = torch.stack([P.decode_partial(q), C.decode_partial(q, max_len=T)])
    out = P.combine(recs).cpu().numpy()
    ref = F.decode(q).cpu().numpy()
    assert P.flags() == 0 and C.flags() == 0
    assert op.rel_err(out, ref) <= 1e-3
    kh, vh = op.bf16_heads(kb, vb)
    heads = op.layer(kh, vh, 3, 3, 9, 1, E=E, pack=False)[1]
    assert op.rel_err(out[0], op.decode(synth.bf16_bits_to_f64(qb[0]), heads)) <= TOL
