"""GPU parity: libkvq (through its C ABI) against the CPU oracle.

Codes, packed words, norms and plans are compared bit for bit; decode outputs
within max relative error 2e-3 per (sequence, query head):
max_i |o_i - o*_i| / max_i |o*_i|, o* the fp64 oracle on its own dequantized
cache built from the same bf16 inputs.
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


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(DEV)


def host_f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def check_plan(p, ref):
    assert p["magic"] == kvq.PLAN_MAGIC
    assert np.array_equal(p["width"].astype(int), ref.widths)
    assert list(p["order"][:p["n_ranks"]]) == ref.order
    assert np.array_equal(p["g"], ref.g) and np.array_equal(p["a_hat"], ref.a_hat)


def check_records(got, ref, n_tokens, bits_k, bits_v):
    nw = 128 * (bits_k + bits_v)
    assert np.array_equal(got[:, :nw], ref[:, :nw]), "packed code words differ"
    gn = got[:, nw:].view(np.uint16).reshape(-1, 2, 32)
    rn = ref[:, nw:].view(np.uint16).reshape(-1, 2, 32)
    pos = np.arange(gn.shape[0] * 32).reshape(-1, 32)
    valid = pos < n_tokens
    for part in range(2):
        assert np.array_equal(gn[:, part][valid], rn[:, part][valid]), "norms differ"


def test_tiny_end_to_end():
    wl = synth.WORKLOADS["tiny"]
    T = wl.context
    kb, vb = synth.keys_values(wl, 0, 0, 0, T)
    kb, vb = kb[:, None, :], vb[:, None, :]
    kh, vh = op.bf16_heads(kb, vb)
    E, heads = op.layer(kh, vh, wl.bits_k, wl.bits_v, v_seed=11, layer_idx=0)
    cfg = kvq.make_cfg(1, wl.bits_k, wl.bits_v, v_seed=11)
    L = PackedLayer(cfg, 1, T + 64)
    k, v = dev_bf16(kb), dev_bf16(vb)
    plans = L.alloc_bits(k)
    assert np.array_equal(L.energy, E), "energies are exact integers: must match bit for bit"
    check_plan(plans[0], heads[0]["plan"])
    for a, b in [(0, 1000), (1000, 1001), (1001, 1048), (1048, T)]:
        L.append(k[a:b][None], v[a:b][None])
    torch.cuda.synchronize()
    assert int(L.lens.item()) == T and L.flags() == 0
    check_records(L.head_records(0, 0, T // 32), heads[0]["rec"], T, wl.bits_k, wl.bits_v)
    qb = synth.queries(wl, 0, 0, 0, T)
    out = L.decode(dev_bf16(qb)[None]).cpu().numpy()[0]
    ref = op.decode(synth.bf16_bits_to_f64(qb), heads)
    assert op.rel_err(out, ref) <= TOL


def _random_layer(rng, n_kv, T, scale_E):
    E = np.exp(scale_E * rng.standard_normal((n_kv, 64)) - np.arange(64) / 8.0)
    sig = np.sqrt(np.concatenate([E, E], axis=1) / 2)  # [n_kv, 128]
    k = rng.standard_normal((T, n_kv, 128)) * sig[None]
    v = rng.standard_normal((T, n_kv, 128))
    return E, synth.to_bf16_bits(k), synth.to_bf16_bits(v)


@pytest.mark.parametrize("bits_k,bits_v,G", [
    (1, 1, 1), (2, 2, 4), (3, 2, 7), (3, 3, 8), (4, 4, 12), (5, 6, 16), (8, 8, 3),
    (2, 5, 8), (6, 3, 2), (7, 7, 8), (3, 8, 5), (8, 1, 16)])
def test_random_plans_ragged(bits_k, bits_v, G):
    """Random energies and widths over every width 1..8, ragged lengths
    (300, 33, 1, 0, 64) in one batch, appends cut so tiles are filled in
    several calls (read-modify-write of partly filled tiles)."""
    rng = np.random.default_rng(bits_k * 100 + bits_v * 10 + G)
    n_kv, lens, cap = 2, [300, 33, 1, 0, 64], 320
    cfg = kvq.make_cfg(n_kv, bits_k, bits_v, v_seed=5)
    L = PackedLayer(cfg, len(lens), cap)
    E, _, _ = _random_layer(rng, n_kv, 1, 1.5)
    L.set_plans(kvq.plan_build(cfg, 3, E))
    refs = []
    for s, T in enumerate(lens):
        if T == 0:
            refs.append(None)
            continue
        _, kb, vb = _random_layer(rng, n_kv, T, 1.5)
        cut = sorted({0, T // 3, T // 3 + 1, T})
        for a, b in zip(cut[:-1], cut[1:]):
            kvq.quantize_append(cfg, L.plan_ptrs[s:s + 1], dev_bf16(kb[a:b])[None],
                                dev_bf16(vb[a:b])[None], L.cache_ptrs[s:s + 1],
                                L.lens[s:s + 1], cap, L.status)
        kh, vh = op.bf16_heads(kb, vb)
        refs.append(op.layer(kh, vh, bits_k, bits_v, 5, 3, E=E)[1])
    torch.cuda.synchronize()
    assert L.lens.cpu().tolist() == lens and L.flags() == 0
    for s, T in enumerate(lens):
        if T == 0:
            continue
        nt = (T + 31) // 32
        for h in range(n_kv):
            check_records(L.head_records(s, h, nt), refs[s][h]["rec"], T, bits_k, bits_v)
    qb = synth.to_bf16_bits(rng.standard_normal((len(lens), n_kv * G, 128)))
    out = L.decode(dev_bf16(qb), max_len=cap).cpu().numpy()
    for s, T in enumerate(lens):
        if T == 0:
            assert np.all(out[s] == 0)
            continue
        q = synth.bf16_bits_to_f64(qb[s])
        assert op.rel_err(out[s], op.decode(q, refs[s])) <= TOL, (s, T)


def test_edge_flags():
    rng = np.random.default_rng(7)
    cfg = kvq.make_cfg(1, 3, 3, v_seed=2)
    E, kb, vb = _random_layer(rng, 1, 70, 1.0)
    k = synth.bf16_bits_to_f64(kb)
    v = synth.bf16_bits_to_f64(vb)
    k[5, 0, 17] = np.nan            # non-finite key token
    v[9, 0, 3] = np.inf             # non-finite value token
    k[11, 0, :] = 3e38              # sumsq overflows fp32 -> saturated norm
    kb, vb = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
    L = PackedLayer(cfg, 1, 96)
    L.set_plans(kvq.plan_build(cfg, 0, E))
    L.append(dev_bf16(kb)[None], dev_bf16(vb)[None])
    torch.cuda.synchronize()
    fl = L.flags()
    assert fl & kvq.FLAG_NONFINITE and fl & kvq.FLAG_NORM_SAT and not fl & kvq.FLAG_CAPACITY
    kh, vh = op.bf16_heads(kb, vb)
    _, heads = op.layer(kh, vh, 3, 3, 2, 0, E=E)
    check_records(L.head_records(0, 0, 3), heads[0]["rec"], 70, 3, 3)
    # capacity: 70 + 30 > 96 -> skipped, length unchanged, cache unchanged
    before = L.caches[0].clone()
    L.status.zero_()
    L.append(dev_bf16(kb[:30])[None], dev_bf16(vb[:30])[None])
    torch.cuda.synchronize()
    assert L.flags() & kvq.FLAG_CAPACITY and int(L.lens.item()) == 70
    assert torch.equal(before, L.caches[0])
    # decode with max_len below the length: clamped and flagged
    L.status.zero_()
    qb = synth.to_bf16_bits(rng.standard_normal((1, 8, 128)))
    out = L.decode(dev_bf16(qb), max_len=40).cpu().numpy()[0]
    assert L.flags() & kvq.FLAG_CAPACITY
    ref = op.decode(synth.bf16_bits_to_f64(qb[0]), heads, length=40)
    assert op.rel_err(out, ref) <= TOL
    # a plan record with a bad magic is refused on the device
    bad = kvq.plan_build(cfg, 0, E)
    bad["magic"] = 0
    L.set_plans(bad, check=False)  # the device check is under test
    L.status.zero_()
    L.decode(dev_bf16(qb), max_len=96)
    torch.cuda.synchronize()
    assert L.flags() & kvq.FLAG_BAD_PLAN


def test_fp32_and_fp16_inputs():
    rng = np.random.default_rng(3)
    cfg = kvq.make_cfg(2, 3, 2, v_seed=9)
    E, kb, vb = _random_layer(rng, 2, 100, 1.0)
    kh, vh = op.bf16_heads(kb, vb)
    _, heads = op.layer(kh, vh, 3, 2, 9, 1, E=E)
    for dt in (torch.float32, torch.float16):
        L = PackedLayer(cfg, 1, 128)
        L.set_plans(kvq.plan_build(cfg, 1, E))
        k = torch.from_numpy(np.stack(kh, 1)).to(DEV, dt)
        v = torch.from_numpy(np.stack(vh, 1)).to(DEV, dt)
        L.append(k[None], v[None])
        torch.cuda.synchronize()
        for h in range(2):
            if dt == torch.float32:  # bf16 values are exact in fp32: identical codes
                check_records(L.head_records(0, h, 4), heads[h]["rec"], 100, 3, 2)
        q = torch.from_numpy(rng.standard_normal((1, 8, 128))).to(DEV, dt)
        out = L.decode(q).cpu().numpy()[0]
        if dt == torch.float32:
            assert op.rel_err(out, op.decode(host_f64(q[0]), heads)) <= TOL


@pytest.mark.parametrize("name,layer_idx", [("llama8b", 0), ("qwen3b_128k", 17)])
def test_full_size_layer(name, layer_idx):
    """One layer at full size, in the bench's launch configuration: bulk
    prefill append, then decode with max_len = context. Energies and plans
    exact; 48 sampled tiles per head bit-exact; decode output against the
    full oracle pipeline of the layer."""
    wl = synth.WORKLOADS[name]
    T = wl.context
    cfg = kvq.make_cfg(wl.n_kv_heads, wl.bits_k, wl.bits_v, v_seed=1234)
    k, v = synth.keys_values_torch(wl, 0, layer_idx, T, DEV)
    L = PackedLayer(cfg, 1, T, layer=layer_idx)
    L.alloc_bits(k)
    L.append(k[None], v[None])
    torch.cuda.synchronize()
    assert int(L.lens.item()) == T and L.flags() == 0
    kf, vf = host_f64(k), host_f64(v)
    kh = [kf[:, h] for h in range(wl.n_kv_heads)]
    vh = [vf[:, h] for h in range(wl.n_kv_heads)]
    E, _ = op.energies(kh)
    assert np.array_equal(L.energy, E)
    rng = np.random.default_rng(0)
    n_tiles = T // 32
    tiles = np.unique(np.concatenate([rng.integers(0, n_tiles, 47), [n_tiles - 1]]))
    for h in range(wl.n_kv_heads):
        plan = alloc.make_plan(E[h], wl.bits_k, wl.bits_v, 1234, layer_idx, h)
        check_plan(L.plans_host[h], plan)
        got = L.head_records(0, h, n_tiles)
        for t in tiles:
            sl = slice(32 * t, 32 * t + 32)
            kc, kn, _ = quant.quantize_keys(kh[h][sl], plan)
            vc, vn, _ = quant.quantize_values(vh[h][sl], plan)
            ref = layout.pack(kc, vc, kn, vn, plan, 32)
            check_records(got[t:t + 1], ref, 32, wl.bits_k, wl.bits_v)
    qb = synth.queries(wl, 0, layer_idx, 0, T)
    out = L.decode(dev_bf16(qb)[None], max_len=T).cpu().numpy()[0]
    _, heads = op.layer(kh, vh, wl.bits_k, wl.bits_v, 1234, layer_idx, E=E, pack=False)
    assert op.rel_err(out, op.decode(synth.bf16_bits_to_f64(qb), heads)) <= TOL


def test_serving_step_append_then_decode():
    """16 sequences x (32K - 16) cached tokens, append 16 per sequence, decode
    (7B-Qwen-shaped serving step, K3V2, G = 7); sequences 0 and 9 checked in
    full against the oracle, all appended tiles bit-exact."""
    wl = synth.WORKLOADS["qwen7b_serve"]
    T0, n_new, B = wl.context - wl.n_new, wl.n_new, wl.batch
    cfg = kvq.make_cfg(wl.n_kv_heads, wl.bits_k, wl.bits_v, v_seed=77)
    L = PackedLayer(cfg, B, wl.context, layer=3)
    ks, vs = [], []
    for s in range(B):
        k, v = synth.keys_values_torch(wl, s, 3, wl.context, DEV)
        ks.append(k)
        vs.append(v)
    L.alloc_bits(ks[0][:T0])
    kall, vall = torch.stack(ks), torch.stack(vs)
    L.append(kall[:, :T0].contiguous(), vall[:, :T0].contiguous())
    L.append(kall[:, T0:].contiguous(), vall[:, T0:].contiguous())
    torch.cuda.synchronize()
    assert L.lens.cpu().tolist() == [wl.context] * B and L.flags() == 0
    E = L.energy
    q = torch.stack([dev_bf16(synth.queries(wl, s, 3, 0, wl.context)) for s in range(B)])
    out = L.decode(q, max_len=wl.context).cpu().numpy()
    for s in (0, 9):
        kf, vf = host_f64(ks[s]), host_f64(vs[s])
        kh = [kf[:, h] for h in range(wl.n_kv_heads)]
        vh = [vf[:, h] for h in range(wl.n_kv_heads)]
        _, heads = op.layer(kh, vh, wl.bits_k, wl.bits_v, 77, 3, E=E, pack=False)
        nt = wl.context // 32
        for h in range(wl.n_kv_heads):
            got = L.head_records(s, h, nt)
            tail = slice(wl.context - 64, wl.context)
            plan = heads[h]["plan"]
            ref = layout.pack(heads[h]["kcodes"][tail], heads[h]["vcodes"][tail],
                              heads[h]["knorm"][tail], heads[h]["vnorm"][tail], plan, 64)
            check_records(got[-2:], ref, 64, wl.bits_k, wl.bits_v)
        assert op.rel_err(out[s], op.decode(host_f64(q[s]), heads)) <= TOL


@pytest.mark.parametrize("n_new,bits,flags", [(1, (3, 3), 0), (1, (3, 3), 1), (16, (3, 2), 1),
                                              (40, (2, 2), 0), (5, (6, 1), 1)])
def test_fused_append_decode(n_new, bits, flags):
    """kvq_append_decode (append n_new tokens and decode in one launch) against
    the oracle: packed words and norms bit-exact, new lengths, outputs; one
    sequence starts empty, one is refused for capacity (len unchanged, decoded
    over its old tokens)."""
    bk, bv = bits
    rng = np.random.default_rng(100 + n_new)
    n_kv, G, cap = 2, 8, 384
    starts = [300, 31, 0, cap - n_new + 1]   # the last one overflows
    cfg = kvq.make_cfg(n_kv, bk, bv, v_seed=6)
    L = PackedLayer(cfg, len(starts), cap)
    E, _, _ = _random_layer(rng, n_kv, 1, 1.2)
    L.set_plans(kvq.plan_build(cfg, 2, E))
    data = []
    for s, T0 in enumerate(starts):
        _, kb, vb = _random_layer(rng, n_kv, T0 + n_new, 1.2)
        data.append((kb, vb))
        if T0:
            kvq.quantize_append(cfg, L.plan_ptrs[s:s + 1], dev_bf16(kb[:T0])[None],
                                dev_bf16(vb[:T0])[None], L.cache_ptrs[s:s + 1],
                                L.lens[s:s + 1], cap, L.status)
    torch.cuda.synchronize()
    assert L.flags() == 0
    knew = torch.stack([dev_bf16(kb[T0:T0 + n_new]) for (kb, _), T0 in zip(data, starts)])
    vnew = torch.stack([dev_bf16(vb[T0:T0 + n_new]) for (_, vb), T0 in zip(data, starts)])
    qb = synth.to_bf16_bits(rng.standard_normal((len(starts), n_kv * G, 128)))
    ws = L.workspace(n_kv * G, cap)
    out = L.append_decode(knew, vnew, dev_bf16(qb), ws=ws, step_flags=flags).cpu().numpy()
    torch.cuda.synchronize()
    assert L.flags() == kvq.FLAG_CAPACITY
    expect_len = [T0 + n_new for T0 in starts[:-1]] + [starts[-1]]
    assert L.lens.cpu().tolist() == expect_len
    for s, T in enumerate(expect_len):
        kb, vb = data[s]
        kh, vh = op.bf16_heads(kb[:T], vb[:T])
        _, heads = op.layer(kh, vh, bk, bv, 6, 2, E=E)
        for h in range(n_kv):
            check_records(L.head_records(s, h, (T + 31) // 32), heads[h]["rec"], T, bk, bv)
        q = synth.bf16_bits_to_f64(qb[s])
        assert op.rel_err(out[s], op.decode(q, heads)) <= TOL, s
    # the counters are back at zero: a second fused step on the same workspace
    L.status.zero_()
    k2 = torch.zeros((len(starts), 1, n_kv, 128), dtype=torch.bfloat16, device=DEV)
    L.append_decode(k2, k2, dev_bf16(qb), ws=ws, step_flags=flags)
    torch.cuda.synchronize()
    assert L.lens.cpu().tolist()[:-1] == [x + 1 for x in expect_len[:-1]]


def test_early_prefetch_layer_loop_matches_plain():
    """A loop of fused steps over layers that share one workspace, launched
    with STEP_EARLY (each layer's caches streamed before the previous layer's
    kernel has ended), gives the same lengths and packed caches bit for bit,
    and the same outputs to fp32 rounding, as the same loop without it."""
    rng = np.random.default_rng(77)
    n_kv, G, cap, n_layers, n_steps = 2, 8, 704, 3, 4
    starts = [300, 31, 640]
    cfg = kvq.make_cfg(n_kv, 3, 2, v_seed=12)
    sets = []
    for _ in range(2):
        layers = [PackedLayer(cfg, len(starts), cap, layer=li) for li in range(n_layers)]
        sets.append((layers, layers[0].workspace(n_kv * G, cap)))
    for li in range(n_layers):
        E, _, _ = _random_layer(rng, n_kv, 1, 1.2)
        plans = kvq.plan_build(cfg, li, E)
        for s, T0 in enumerate(starts):
            _, kb, vb = _random_layer(rng, n_kv, T0, 1.2)
            for layers, _ in sets:
                L = layers[li]
                L.set_plans(plans)
                kvq.quantize_append(cfg, L.plan_ptrs[s:s + 1], dev_bf16(kb)[None],
                                    dev_bf16(vb)[None], L.cache_ptrs[s:s + 1],
                                    L.lens[s:s + 1], cap, L.status)
    torch.cuda.synchronize()
    shape = (len(starts), 1, n_kv, 128)
    for step in range(n_steps):
        ks = [dev_bf16(synth.to_bf16_bits(rng.standard_normal(shape))) for _ in range(n_layers)]
        vs = [dev_bf16(synth.to_bf16_bits(rng.standard_normal(shape))) for _ in range(n_layers)]
        qs = [dev_bf16(synth.to_bf16_bits(rng.standard_normal((len(starts), n_kv * G, 128))))
              for _ in range(n_layers)]
        outs = []
        for (layers, ws), flags in zip(sets, (0, kvq.STEP_EARLY)):
            o = [layers[li].append_decode(ks[li], vs[li], qs[li], ws=ws, step_flags=flags)
                 for li in range(n_layers)]
            outs.append(o)
        torch.cuda.synchronize()
        for li in range(n_layers):
            # the split sums run through L2 atomics in arrival order: equal
            # to fp32 rounding (the packed caches below are bit-exact)
            a_, b_ = outs[0][li].double(), outs[1][li].double()
            den = a_.abs().amax(dim=-1).clamp_min(1e-30)
            assert float(((a_ - b_).abs().amax(dim=-1) / den).max()) <= 1e-5, (step, li)
            assert bool(torch.isfinite(outs[1][li]).all())
    for li in range(n_layers):
        a, b = sets[0][0][li], sets[1][0][li]
        assert a.lens.cpu().tolist() == [T0 + n_steps for T0 in starts]
        assert torch.equal(a.lens, b.lens)
        for s in range(len(starts)):
            assert torch.equal(a.caches[s], b.caches[s]), (li, s)
        assert a.flags() == 0 and b.flags() == 0


@pytest.mark.parametrize("bits", [(3, 3), (5, 2), (2, 7)])
def test_chunked_appends_mixed_lengths(bits):
    """Appends of 1, 5, 37, 64, 3 and 30 tokens to five sequences that start
    at different lengths (fresh tiles, partly filled tiles, tile boundaries,
    fields that straddle words): every record bit-exact against the oracle's
    pack of the whole sequence, lengths and flags as expected."""
    bk, bv = bits
    rng = np.random.default_rng(500 + 10 * bk + bv)
    n_kv = 2
    starts = [0, 7, 31, 32, 100]
    chunks = [1, 5, 37, 64, 3, 30]
    total = sum(chunks)
    cap = max(starts) + total + 32
    cfg = kvq.make_cfg(n_kv, bk, bv, v_seed=21)
    L = PackedLayer(cfg, len(starts), cap, layer=4)
    E, _, _ = _random_layer(rng, n_kv, 1, 1.2)
    L.set_plans(kvq.plan_build(cfg, 4, E))
    data = []
    for s, T0 in enumerate(starts):
        _, kb, vb = _random_layer(rng, n_kv, T0 + total, 1.2)
        data.append((kb, vb))
        if T0:
            kvq.quantize_append(cfg, L.plan_ptrs[s:s + 1], dev_bf16(kb[:T0])[None],
                                dev_bf16(vb[:T0])[None], L.cache_ptrs[s:s + 1],
                                L.lens[s:s + 1], cap, L.status)
    off = 0
    for n in chunks:
        k = torch.stack([dev_bf16(kb[T0 + off:T0 + off + n]) for (kb, _), T0 in zip(data, starts)])
        v = torch.stack([dev_bf16(vb[T0 + off:T0 + off + n]) for (_, vb), T0 in zip(data, starts)])
        L.append(k, v)
        off += n
    torch.cuda.synchronize()
    assert L.flags() == 0
    assert L.lens.cpu().tolist() == [T0 + total for T0 in starts]
    for s, T0 in enumerate(starts):
        T = T0 + total
        kb, vb = data[s]
        kh, vh = op.bf16_heads(kb[:T], vb[:T])
        _, heads = op.layer(kh, vh, bk, bv, 21, 4, E=E)
        for h in range(n_kv):
            check_records(L.head_records(s, h, (T + 31) // 32), heads[h]["rec"], T, bk, bv)


def test_split_maxima_outside_bucket_range_take_the_record_merge():
    """Queries large enough that split maxima leave the exponent-bucket range
    [-256, 256) (base-2 logits): the last split merges all split records
    instead; the output still matches the oracle, and the next call on the
    same workspace (buckets and flags cleared) is right again."""
    rng = np.random.default_rng(31)
    n_kv, G, T = 2, 8, 3000
    cfg = kvq.make_cfg(n_kv, 3, 3, v_seed=4)
    L = PackedLayer(cfg, 1, 3072)
    E, kb, vb = _random_layer(rng, n_kv, T, 1.0)
    L.set_plans(kvq.plan_build(cfg, 0, E))
    L.append(dev_bf16(kb)[None], dev_bf16(vb)[None])
    kh, vh = op.bf16_heads(kb, vb)
    _, heads = op.layer(kh, vh, 3, 3, 4, 0, E=E, pack=False)
    ws = L.workspace(n_kv * G, 3072)
    for scale in (400.0, 1.0, -400.0, 1.0):
        qb = synth.to_bf16_bits(rng.standard_normal((1, n_kv * G, 128)) * scale)
        out = L.decode(dev_bf16(qb), ws=ws).cpu().numpy()[0]
        ref = op.decode(synth.bf16_bits_to_f64(qb[0]), heads)
        assert np.isfinite(out).all(), scale
        assert op.rel_err(out, ref) <= TOL, scale
    assert L.flags() == 0


@pytest.mark.parametrize("rot", [0, kvq.ALLOC_ROTATE_KEYS])
def test_degenerate_plans_zero_and_single_block_energy(rot):
    """Plans from degenerate energies (all zero: every key scale 0, so every
    dequantized key is 0 and attention is uniform; one nonzero block) with
    and without key rotation: records bit-exact, outputs against the oracle."""
    rng = np.random.default_rng(12)
    n_kv, G, T = 2, 8, 200
    E = np.zeros((n_kv, 64))
    E[1, 9] = 2.5
    cfg = kvq.make_cfg(n_kv, 3, 2, v_seed=3, alloc_mode=rot)
    L = PackedLayer(cfg, 1, 256)
    L.set_plans(kvq.plan_build(cfg, 1, E))
    kb = synth.to_bf16_bits(rng.standard_normal((T, n_kv, 128)))
    vb = synth.to_bf16_bits(rng.standard_normal((T, n_kv, 128)))
    L.append(dev_bf16(kb)[None], dev_bf16(vb)[None])
    qb = synth.to_bf16_bits(rng.standard_normal((1, n_kv * G, 128)))
    out = L.decode(dev_bf16(qb), max_len=256).cpu().numpy()[0]
    torch.cuda.synchronize()
    assert L.flags() == 0
    kh, vh = op.bf16_heads(kb, vb)
    _, heads = op.layer(kh, vh, 3, 2, 3, 1, E=E, rotate_keys=bool(rot))
    for h in range(n_kv):
        check_records(L.head_records(0, h, (T + 31) // 32), heads[h]["rec"], T, 3, 2)
    ref = op.decode(synth.bf16_bits_to_f64(qb[0]), heads)
    assert op.rel_err(out, ref) <= TOL
    # head 0 has all-zero scales: its keys dequantize to 0, attention is the mean of V
    assert np.allclose(ref[:G], heads[0]["vhat"].mean(axis=0)[None], rtol=0, atol=1e-12)
