"""GPU parity of the per-width-group key rotation (KVQ_ALLOC_ROTATE_KEYS)
through the C ABI: packed words and norms bit-exact against the oracle (bulk
append in several calls, the fused append of the serving step), decode
outputs within max relative error 2e-3 of the fp64 oracle, which decodes with
the exact orthonormal inverse rotation while the kernel rotates the query.
"""
import numpy as np
import pytest
import torch

import oracle_pipeline as op
import synth
from bit_kv_cache_19_b200 import kvq
from bit_kv_cache_19_b200.runtime import PackedLayer
from oracle import alloc, layout, quant

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 2e-3
ROT = kvq.ALLOC_ROTATE_KEYS


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(DEV)


def check_records(got, ref, n_tokens, bits_k, bits_v):
    nw = 128 * (bits_k + bits_v)
    assert np.array_equal(got[:, :nw], ref[:, :nw]), "packed code words differ"
    gn = got[:, nw:].view(np.uint16).reshape(-1, 2, 32)
    rn = ref[:, nw:].view(np.uint16).reshape(-1, 2, 32)
    valid = np.arange(gn.shape[0] * 32).reshape(-1, 32) < n_tokens
    for part in range(2):
        assert np.array_equal(gn[:, part][valid], rn[:, part][valid]), "norms differ"


def _random_kv(rng, n_kv, T, E, outliers=True):
    sig = np.sqrt(np.concatenate([E, E], axis=1) / 2)
    k = rng.standard_normal((T, n_kv, 128)) * sig[None]
    if outliers:
        k = np.where(rng.random(k.shape) < 0.01, 8.0 * k, k)
    return synth.to_bf16_bits(k), synth.to_bf16_bits(rng.standard_normal((T, n_kv, 128)))


@pytest.mark.parametrize("bits_k,bits_v,G,uniform", [
    (1, 1, 1, False), (2, 2, 4, False), (3, 3, 8, False), (3, 2, 7, True), (4, 4, 12, False),
    (5, 6, 16, False), (8, 8, 3, False), (2, 5, 8, True), (7, 3, 8, False)])
def test_rotated_plans_ragged(bits_k, bits_v, G, uniform):
    rng = np.random.default_rng(bits_k * 100 + bits_v * 10 + G)
    n_kv, lens, cap = 2, [300, 33, 1, 0, 64], 320
    mode = (kvq.ALLOC_UNIFORM if uniform else kvq.ALLOC_GREEDY) | ROT
    cfg = kvq.make_cfg(n_kv, bits_k, bits_v, v_seed=5, alloc_mode=mode)
    L = PackedLayer(cfg, len(lens), cap)
    E = np.exp(1.5 * rng.standard_normal((n_kv, 64)) - np.arange(64) / 8.0)
    L.set_plans(kvq.plan_build(cfg, 3, E))
    refs = []
    for s, T in enumerate(lens):
        if T == 0:
            refs.append(None)
            continue
        kb, vb = _random_kv(rng, n_kv, T, E)
        cut = sorted({0, T // 3, T // 3 + 1, T})
        for a, b in zip(cut[:-1], cut[1:]):
            kvq.quantize_append(cfg, L.plan_ptrs[s:s + 1], dev_bf16(kb[a:b])[None],
                                dev_bf16(vb[a:b])[None], L.cache_ptrs[s:s + 1],
                                L.lens[s:s + 1], cap, L.status)
        kh, vh = op.bf16_heads(kb, vb)
        refs.append(op.layer(kh, vh, bits_k, bits_v, 5, 3, E=E, uniform=uniform,
                             rotate_keys=True)[1])
    torch.cuda.synchronize()
    assert L.lens.cpu().tolist() == lens and L.flags() == 0
    for s, T in enumerate(lens):
        if T == 0:
            continue
        for h in range(n_kv):
            check_records(L.head_records(s, h, (T + 31) // 32), refs[s][h]["rec"], T, bits_k,
                          bits_v)
    qb = synth.to_bf16_bits(rng.standard_normal((len(lens), n_kv * G, 128)))
    out = L.decode(dev_bf16(qb), max_len=cap).cpu().numpy()
    for s, T in enumerate(lens):
        if T == 0:
            assert np.all(out[s] == 0)
            continue
        assert op.rel_err(out[s], op.decode(synth.bf16_bits_to_f64(qb[s]), refs[s])) <= TOL


@pytest.mark.parametrize("n_new,flags", [(1, 0), (16, kvq.STEP_EARLY), (40, 0)])
def test_rotated_fused_append_decode(n_new, flags):
    rng = np.random.default_rng(300 + n_new)
    n_kv, G, cap = 2, 8, 384
    starts = [300, 31, 0]
    cfg = kvq.make_cfg(n_kv, 3, 3, v_seed=6, alloc_mode=ROT)
    L = PackedLayer(cfg, len(starts), cap)
    E = np.exp(1.2 * rng.standard_normal((n_kv, 64)) - np.arange(64) / 8.0)
    L.set_plans(kvq.plan_build(cfg, 2, E))
    data = []
    for s, T0 in enumerate(starts):
        kb, vb = _random_kv(rng, n_kv, T0 + n_new, E)
        data.append((kb, vb))
        if T0:
            kvq.quantize_append(cfg, L.plan_ptrs[s:s + 1], dev_bf16(kb[:T0])[None],
                                dev_bf16(vb[:T0])[None], L.cache_ptrs[s:s + 1],
                                L.lens[s:s + 1], cap, L.status)
    knew = torch.stack([dev_bf16(kb[T0:T0 + n_new]) for (kb, _), T0 in zip(data, starts)])
    vnew = torch.stack([dev_bf16(vb[T0:T0 + n_new]) for (_, vb), T0 in zip(data, starts)])
    qb = synth.to_bf16_bits(rng.standard_normal((len(starts), n_kv * G, 128)))
    out = L.append_decode(knew, vnew, dev_bf16(qb), step_flags=flags).cpu().numpy()
    torch.cuda.synchronize()
    assert L.flags() == 0
    for s, T0 in enumerate(starts):
        T = T0 + n_new
        kb, vb = data[s]
        kh, vh = op.bf16_heads(kb[:T], vb[:T])
        _, heads = op.layer(kh, vh, 3, 3, 6, 2, E=E, rotate_keys=True)
        for h in range(n_kv):
            check_records(L.head_records(s, h, (T + 31) // 32), heads[h]["rec"], T, 3, 3)
        assert op.rel_err(out[s], op.decode(synth.bf16_bits_to_f64(qb[s]), heads)) <= TOL


def test_rotated_full_size_qwen3b_layer():
    """A full 128K-token Qwen-3B-shaped layer (2 KV heads, G = 8, K3V3) with
    rotated keys, in the bench's launch configuration: plans from the GPU
    energies, 48 sampled tiles per head bit-exact, decode against the oracle."""
    wl = synth.WORKLOADS["qwen3b_128k"]
    T = wl.context
    cfg = kvq.make_cfg(wl.n_kv_heads, wl.bits_k, wl.bits_v, v_seed=99, alloc_mode=ROT)
    k, v = synth.keys_values_torch(wl, 0, 9, T, DEV)
    L = PackedLayer(cfg, 1, T, layer=9)
    L.alloc_bits(k)
    L.append(k[None], v[None])
    torch.cuda.synchronize()
    assert L.flags() == 0
    kf = k.float().cpu().numpy().astype(np.float64)
    vf = v.float().cpu().numpy().astype(np.float64)
    kh = [kf[:, h] for h in range(wl.n_kv_heads)]
    vh = [vf[:, h] for h in range(wl.n_kv_heads)]
    E, _ = op.energies(kh)
    rng = np.random.default_rng(1)
    n_tiles = T // 32
    tiles = np.unique(np.concatenate([rng.integers(0, n_tiles, 47), [n_tiles - 1]]))
    for h in range(wl.n_kv_heads):
        plan = alloc.make_plan(E[h], wl.bits_k, wl.bits_v, 99, 9, h, rotate_keys=True)
        got = L.head_records(0, h, n_tiles)
        for t in tiles:
            sl = slice(32 * t, 32 * t + 32)
            kc, kn, _ = quant.quantize_keys(kh[h][sl], plan)
            vc, vn, _ = quant.quantize_values(vh[h][sl], plan)
            check_records(got[t:t + 1], layout.pack(kc, vc, kn, vn, plan, 32), 32, wl.bits_k,
                          wl.bits_v)
    qb = synth.queries(wl, 0, 9, 0, T)
    out = L.decode(dev_bf16(qb)[None], max_len=T).cpu().numpy()[0]
    _, heads = op.layer(kh, vh, wl.bits_k, wl.bits_v, 99, 9, E=E, pack=False, rotate_keys=True)
    assert op.rel_err(out, op.decode(synth.bf16_bits_to_f64(qb), heads)) <= TOL


def test_rotated_edge_tokens_and_paged_cache():
    """Rotated plans with a non-finite key, a non-finite value, a zero key and
    a key whose norm saturates fp16: codes and norms bit-exact against the
    oracle; the same tokens in a paged cache (shuffled 1-tile pages) give the
    same records and the same decode output."""
    from bit_kv_cache_19_b200.runtime import PagedLayer
    rng = np.random.default_rng(8)
    n_kv, T = 1, 90
    cfg = kvq.make_cfg(n_kv, 3, 3, v_seed=2, alloc_mode=ROT)
    E = np.exp(rng.standard_normal((n_kv, 64)))
    kb, vb = _random_kv(rng, n_kv, T, E)
    k = synth.bf16_bits_to_f64(kb)
    v = synth.bf16_bits_to_f64(vb)
    k[5, 0, 17] = np.nan
    v[9, 0, 3] = np.inf
    k[11, 0, :] = 0.0
    k[12, 0, :] = 3e38
    kb, vb = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
    plans = kvq.plan_build(cfg, 0, E)
    L = PackedLayer(cfg, 1, 96)
    L.set_plans(plans)
    L.append(dev_bf16(kb)[None], dev_bf16(vb)[None])
    P = PagedLayer(cfg, 1, 5, 1, 3)
    P.set_plans(plans)
    P.reserve(0, T, order=[4, 1, 3])
    P.append(dev_bf16(kb)[None], dev_bf16(vb)[None])
    torch.cuda.synchronize()
    fl = L.flags()
    assert fl & kvq.FLAG_NONFINITE and fl & kvq.FLAG_NORM_SAT and P.flags() == fl
    kh, vh = op.bf16_heads(kb, vb)
    _, heads = op.layer(kh, vh, 3, 3, 2, 0, E=E, rotate_keys=True)
    check_records(L.head_records(0, 0, 3), heads[0]["rec"], T, 3, 3)
    assert np.array_equal(P.head_records(0, 0, 3), L.head_records(0, 0, 3))
    qb = synth.to_bf16_bits(rng.standard_normal((1, 8, 128)))
    out = L.decode(dev_bf16(qb), max_len=96).cpu().numpy()
    out_p = P.decode(dev_bf16(qb), max_len=96).cpu().numpy()
    assert op.rel_err(out[0], op.decode(synth.bf16_bits_to_f64(qb[0]), heads)) <= TOL
    assert op.rel_err(out_p[0], out[0]) <= 1e-5
