"""GPU parity of the recent-token window (kvq_window_append,
kvq_decode_attn_window) against the oracle's window reading.

After any sequence of appends, the packed cache must hold exactly the oracle
records of the tokens that left the window (bit for bit), the ring must hold
the window tokens exactly (token t in slot t mod R), and decode must be the
fp64 attention over the dequantized packed tokens and the exact window tokens
within 2e-3.
"""
import numpy as np
import pytest
import torch

import oracle_pipeline as op
import synth
from bit_kv_cache_19_b200 import kvq
from bit_kv_cache_19_b200.runtime import PackedLayer
from oracle import window
from test_gpu_parity import check_records, dev_bf16

pytestmark = pytest.mark.gpu
TOL = 2e-3
V_SEED = 6


def _inputs(rng, batch, T, n_kv):
    k = synth.to_bf16_bits(rng.standard_normal((batch, T, n_kv, 128)))
    v = synth.to_bf16_bits(rng.standard_normal((batch, T, n_kv, 128)))
    return k, v


def _check_state(L, kb, vb, T, E, bits_k, bits_v, R, rng, G):
    n_kv = L.cfg.n_kv_heads
    sp = window.split_point(T, R)
    assert L.lens.cpu().tolist() == [sp] * L.batch
    assert L.wlens.cpu().tolist() == [min(R, T) if R else 0] * L.batch
    assert L.flags() == 0
    qb = synth.to_bf16_bits(rng.standard_normal((L.batch, n_kv * G, 128)))
    out = L.decode_window(dev_bf16(qb)).cpu().numpy()
    for s in range(L.batch):
        kh, vh = op.bf16_heads(kb[s, :T], vb[s, :T])
        heads = op.layer([x[:sp] for x in kh], [x[:sp] for x in vh], bits_k, bits_v, V_SEED, 0,
                         E=E, pack=sp > 0)[1] if sp else None
        if sp:
            for h in range(n_kv):
                check_records(L.head_records(s, h, (sp + 31) // 32), heads[h]["rec"], sp,
                              bits_k, bits_v)
        if R:
            wk, wv = L.window_rows(s)
            for t, slot in window.ring_slots(T, R):
                assert np.array_equal(wk[slot], synth.bf16_bits_to_f64(kb[s, t])), (t, slot)
                assert np.array_equal(wv[slot], synth.bf16_bits_to_f64(vb[s, t])), (t, slot)
        empty = [np.zeros((0, 128))] * n_kv
        ref = window.decode(synth.bf16_bits_to_f64(qb[s]),
                            [x["khat"] for x in heads] if sp else empty,
                            [x["vhat"] for x in heads] if sp else empty,
                            [x[sp:] for x in kh], [x[sp:] for x in vh])
        assert op.rel_err(out[s], ref) <= TOL, (s, T, sp)


# R = 260: 17 window record parts of 16 tokens, with evictions; R = 700: 32
# parts of 32 tokens (two staged sub-chunks each) over a window that holds
# every token, so most parts are empty
@pytest.mark.parametrize("R,bits_k,bits_v,G", [(48, 3, 2, 4), (32, 2, 3, 8), (100, 4, 4, 16),
                                               (1, 3, 3, 7), (260, 3, 3, 8), (700, 2, 2, 5)])
def test_window_appends_and_decode(R, bits_k, bits_v, G):
    rng = np.random.default_rng(R * 7 + bits_k)
    n_kv, batch = 2, 2
    steps = [300, 1, 5, 17, 1, 64, 2, 40]
    T = sum(steps)
    cfg = kvq.make_cfg(n_kv, bits_k, bits_v, v_seed=V_SEED)
    L = PackedLayer(cfg, batch, T + 32, window=R)
    E = np.exp(rng.standard_normal((n_kv, 64)) - np.arange(64) / 8.0)
    L.set_plans(kvq.plan_build(cfg, 0, E))
    kb, vb = _inputs(rng, batch, T, n_kv)
    t = 0
    for i, n in enumerate(steps):
        L.append_window(dev_bf16(kb[:, t:t + n]), dev_bf16(vb[:, t:t + n]))
        t += n
        torch.cuda.synchronize()
        if i in (0, 1, 3, len(steps) - 1):
            _check_state(L, kb, vb, t, E, bits_k, bits_v, R, rng, G)


def test_window_holds_everything_short_sequences():
    # fewer tokens than the window: nothing is quantized, decode is exact attention
    rng = np.random.default_rng(5)
    n_kv, batch, R = 2, 3, 128
    cfg = kvq.make_cfg(n_kv, 3, 3, v_seed=V_SEED)
    L = PackedLayer(cfg, batch, 256, window=R)
    E = np.exp(rng.standard_normal((n_kv, 64)))
    L.set_plans(kvq.plan_build(cfg, 0, E))
    kb, vb = _inputs(rng, batch, 90, n_kv)
    L.append_window(dev_bf16(kb[:, :60]), dev_bf16(vb[:, :60]))
    L.append_window(dev_bf16(kb[:, 60:]), dev_bf16(vb[:, 60:]))
    torch.cuda.synchronize()
    _check_state(L, kb, vb, 90, E, 3, 3, R, rng, 8)


def test_no_window_is_the_plain_append_and_decode():
    rng = np.random.default_rng(6)
    n_kv, batch, T = 2, 2, 200
    cfg = kvq.make_cfg(n_kv, 3, 2, v_seed=V_SEED)
    E = np.exp(rng.standard_normal((n_kv, 64)))
    La = PackedLayer(cfg, batch, 256, window=0)
    Lb = PackedLayer(cfg, batch, 256)
    for L in (La, Lb):
        L.set_plans(kvq.plan_build(cfg, 0, E))
    kb, vb = _inputs(rng, batch, T, n_kv)
    La.append_window(dev_bf16(kb), dev_bf16(vb))
    Lb.append(dev_bf16(kb), dev_bf16(vb))
    torch.cuda.synchronize()
    for s in range(batch):
        assert torch.equal(La.caches[s], Lb.caches[s])
    assert La.lens.cpu().tolist() == [T, T]
    _check_state(La, kb, vb, T, E, 3, 2, 0, rng, 4)
    q = dev_bf16(synth.to_bf16_bits(rng.standard_normal((batch, n_kv * 4, 128))))
    a = La.decode_window(q).cpu().numpy()
    b = Lb.decode(q).cpu().numpy()
    assert op.rel_err(a, b) <= 1e-5


def test_window_evictions_past_capacity_flag_and_leave_state():
    rng = np.random.default_rng(8)
    n_kv, R, cap = 1, 16, 64
    cfg = kvq.make_cfg(n_kv, 2, 2, v_seed=V_SEED)
    L = PackedLayer(cfg, 1, cap, window=R)
    L.set_plans(kvq.plan_build(cfg, 0, np.exp(rng.standard_normal((n_kv, 64)))))
    kb, vb = _inputs(rng, 1, 120, n_kv)
    L.append_window(dev_bf16(kb[:, :70]), dev_bf16(vb[:, :70]))  # 54 packed, 16 in the window
    torch.cuda.synchronize()
    assert L.lens.item() == 54 and L.wlens.item() == 16 and L.flags() == 0
    L.append_window(dev_bf16(kb[:, 70:]), dev_bf16(vb[:, 70:]))  # would pack 104 > 64
    torch.cuda.synchronize()
    assert L.flags() & kvq.FLAG_CAPACITY
    assert L.lens.item() == 54 and L.wlens.item() == 16


@pytest.mark.parametrize("dtype", ["fp16", "fp32"])
def test_window_with_rotated_keys_and_other_input_types(dtype):
    # plans with the width-group key rotation; fp16 / fp32 appends: the ring
    # holds the values exactly and evicted tokens are quantized like any other
    rng = np.random.default_rng(11 if dtype == "fp16" else 12)
    n_kv, batch, R = 2, 2, 40
    steps = [150, 3, 30, 1, 50]
    T = sum(steps)
    cfg = kvq.make_cfg(n_kv, 3, 3, v_seed=V_SEED, alloc_mode=kvq.ALLOC_GREEDY | kvq.ALLOC_ROTATE_KEYS)
    L = PackedLayer(cfg, batch, T + 32, window=R)
    E = np.exp(rng.standard_normal((n_kv, 64)) - np.arange(64) / 8.0)
    L.set_plans(kvq.plan_build(cfg, 0, E))
    # inputs exactly representable in bf16 (the oracle's input type) and in
    # the append's type: bf16 values away from fp16's subnormal range are
    # exact in fp16 (fewer mantissa bits, a wider exponent than needed)
    kb, vb = _inputs(rng, batch, T, n_kv)
    kf, vf = synth.bf16_bits_to_f64(kb), synth.bf16_bits_to_f64(vb)
    kf[np.abs(kf) < 2.0 ** -14] = 0.0
    vf[np.abs(vf) < 2.0 ** -14] = 0.0
    kb, vb = synth.to_bf16_bits(kf), synth.to_bf16_bits(vf)
    tdt = torch.float16 if dtype == "fp16" else torch.float32
    kd = torch.from_numpy(kf).to(tdt).cuda()
    vd = torch.from_numpy(vf).to(tdt).cuda()
    assert np.array_equal(kd.double().cpu().numpy(), kf)
    assert np.array_equal(vd.double().cpu().numpy(), vf)
    t = 0
    for n in steps:
        L.append_window(kd[:, t:t + n].contiguous(), vd[:, t:t + n].contiguous())
        t += n
    torch.cuda.synchronize()
    sp = window.split_point(T, R)
    assert L.lens.cpu().tolist() == [sp] * batch and L.flags() == 0
    qb = synth.to_bf16_bits(rng.standard_normal((batch, n_kv * 8, 128)))
    out = L.decode_window(dev_bf16(qb)).cpu().numpy()
    for s_ in range(batch):
        kh, vh = op.bf16_heads(kb[s_], vb[s_])
        heads = op.layer([x[:sp] for x in kh], [x[:sp] for x in vh], 3, 3, V_SEED, 0, E=E,
                         rotate_keys=True)[1]
        for h in range(n_kv):
            check_records(L.head_records(s_, h, (sp + 31) // 32), heads[h]["rec"], sp, 3, 3)
        ref = window.decode(synth.bf16_bits_to_f64(qb[s_]), [x["khat"] for x in heads],
                            [x["vhat"] for x in heads], [x[sp:] for x in kh],
                            [x[sp:] for x in vh])
        assert op.rel_err(out[s_], ref) <= TOL


def _oracle_out(L, kb, vb, T, E, bits_k, bits_v, R, qb, s):
    """fp64 oracle output of sequence s after T tokens (packed ones
    dequantized, window ones exact) for queries qb (bf16 bits)."""
    n_kv = L.cfg.n_kv_heads
    sp = window.split_point(T, R)
    kh, vh = op.bf16_heads(kb[s, :T], vb[s, :T])
    heads = op.layer([x[:sp] for x in kh], [x[:sp] for x in vh], bits_k, bits_v, V_SEED, 0,
                     E=E, pack=False)[1] if sp else None
    empty = [np.zeros((0, 128))] * n_kv
    return window.decode(synth.bf16_bits_to_f64(qb), [x["khat"] for x in heads] if sp else empty,
                         [x["vhat"] for x in heads] if sp else empty, [x[sp:] for x in kh],
                         [x[sp:] for x in vh])


# one-token window steps in one launch (kvq_append_decode_window) against the
# two calls (kvq_window_append + kvq_decode_attn_window) and the oracle: full
# windows (an eviction every step), windows still filling (T0 < R), R = 1,
# a 16-head query group (two MMA n-tiles) and a window of 17 tokens
@pytest.mark.parametrize("R,T0,bits_k,bits_v,G", [(48, 300, 3, 3, 8), (64, 20, 3, 2, 4),
                                                  (1, 100, 2, 2, 8), (100, 130, 4, 3, 16),
                                                  (17, 64, 3, 3, 7)])
def test_fused_window_steps(R, T0, bits_k, bits_v, G):
    _fused_steps(R, T0, bits_k, bits_v, G, [1] * 40)


# steps of several tokens in one launch: the tokens leaving the window span
# tiles and, for the smaller caches, the boundary between two splits (so two
# CTAs each append some of them and write the new tokens that take their
# slots); step sizes up to min(R, 64)
@pytest.mark.parametrize("R,T0,bits_k,bits_v,G,steps", [
    (48, 300, 3, 3, 8, [5, 17, 32, 1, 48, 7, 3]),
    (100, 230, 3, 2, 4, [64, 1, 33, 9, 64]),
    (20, 40, 2, 2, 16, [20, 3, 19, 1, 7]),
    (300, 100, 3, 3, 8, [64, 64, 50, 64, 2, 64])])
def test_fused_window_steps_of_several_tokens(R, T0, bits_k, bits_v, G, steps):
    _fused_steps(R, T0, bits_k, bits_v, G, steps)


def _fused_steps(R, T0, bits_k, bits_v, G, steps):
    rng = np.random.default_rng(R * 13 + T0 + len(steps))
    n_kv, batch = 2, 2
    S = len(steps)
    T = T0 + sum(steps)
    cfg = kvq.make_cfg(n_kv, bits_k, bits_v, v_seed=V_SEED)
    E = np.exp(rng.standard_normal((n_kv, 64)) - np.arange(64) / 8.0)
    plans = kvq.plan_build(cfg, 0, E)
    Lf = PackedLayer(cfg, batch, T + 32, window=R)  # fused steps
    Lu = PackedLayer(cfg, batch, T + 32, window=R)  # the two calls
    for L in (Lf, Lu):
        L.set_plans(plans)
    kb, vb = _inputs(rng, batch, T, n_kv)
    for L in (Lf, Lu):
        L.append_window(dev_bf16(kb[:, :T0]), dev_bf16(vb[:, :T0]))
    nb = kvq.window_decode_workspace_bytes(cfg, batch, n_kv * G, T + 32)
    wsf = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    wsu = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    qbs = synth.to_bf16_bits(rng.standard_normal((S, batch, n_kv * G, 128)))
    t = T0
    for i, n in enumerate(steps):
        k1, v1, q = dev_bf16(kb[:, t:t + n]), dev_bf16(vb[:, t:t + n]), dev_bf16(qbs[i])
        out_f = Lf.append_decode_window(k1, v1, q, ws=wsf).cpu().numpy()
        Lu.append_window(k1, v1)
        out_u = Lu.decode_window(q, ws=wsu).cpu().numpy()
        t += n
        torch.cuda.synchronize()
        assert Lf.flags() == 0 and Lu.flags() == 0, i
        assert op.rel_err(out_f, out_u) <= 1e-5, i
        if i in (0, 1, S // 2, S - 1):
            for s in range(batch):
                ref = _oracle_out(Lf, kb, vb, t, E, bits_k, bits_v, R, qbs[i][s], s)
                assert op.rel_err(out_f[s], ref) <= TOL, (i, s)
    # the same packed caches, rings and lengths as the two calls
    assert torch.equal(Lf.lens, Lu.lens) and torch.equal(Lf.wlens, Lu.wlens)
    for s in range(batch):
        assert torch.equal(Lf.caches[s], Lu.caches[s])
        assert torch.equal(Lf.wins[s], Lu.wins[s])
    _check_state(Lf, kb, vb, T, E, bits_k, bits_v, R, rng, G)


def test_fused_window_step_capacity_leaves_sequence():
    # an eviction that does not fit the capacity: CAPACITY, nothing moves
    rng = np.random.default_rng(31)
    n_kv, R, cap = 1, 8, 32
    cfg = kvq.make_cfg(n_kv, 2, 2, v_seed=V_SEED)
    L = PackedLayer(cfg, 1, cap, window=R)
    L.set_plans(kvq.plan_build(cfg, 0, np.exp(rng.standard_normal((n_kv, 64)))))
    kb, vb = _inputs(rng, 1, 41, n_kv)
    L.append_window(dev_bf16(kb[:, :40]), dev_bf16(vb[:, :40]))  # 32 packed (full), 8 in the ring
    torch.cuda.synchronize()
    assert L.lens.item() == 32 and L.wlens.item() == 8 and L.flags() == 0
    ring = L.wins[0].clone()
    q = dev_bf16(synth.to_bf16_bits(rng.standard_normal((1, 4, 128))))
    L.append_decode_window(dev_bf16(kb[:, 40:41]), dev_bf16(vb[:, 40:41]), q)
    torch.cuda.synchronize()
    assert L.flags() & kvq.FLAG_CAPACITY
    assert L.lens.item() == 32 and L.wlens.item() == 8
    assert torch.equal(ring, L.wins[0])


def test_window_step_of_several_tokens_is_the_two_calls():
    # n_new > 1: kvq_append_decode_window runs kvq_window_append and
    # kvq_decode_attn_window, so its state equals theirs and its output agrees
    rng = np.random.default_rng(41)
    n_kv, batch, R, G = 2, 2, 24, 8
    cfg = kvq.make_cfg(n_kv, 3, 3, v_seed=V_SEED)
    plans = kvq.plan_build(cfg, 0, np.exp(rng.standard_normal((n_kv, 64))))
    La, Lb = PackedLayer(cfg, batch, 256, window=R), PackedLayer(cfg, batch, 256, window=R)
    for L in (La, Lb):
        L.set_plans(plans)
    kb, vb = _inputs(rng, batch, 120, n_kv)
    t = 0
    for n in (50, 5, 17, 3):
        k, v = dev_bf16(kb[:, t:t + n]), dev_bf16(vb[:, t:t + n])
        q = dev_bf16(synth.to_bf16_bits(rng.standard_normal((batch, n_kv * G, 128))))
        oa = La.append_decode_window(k, v, q).cpu().numpy()
        Lb.append_window(k, v)
        ob = Lb.decode_window(q).cpu().numpy()
        t += n
        torch.cuda.synchronize()
        assert La.flags() == 0 and op.rel_err(oa, ob) <= 1e-5
    assert torch.equal(La.lens, Lb.lens) and torch.equal(La.wlens, Lb.wlens)
    for s in range(batch):
        assert torch.equal(La.caches[s], Lb.caches[s]) and torch.equal(La.wins[s], Lb.wins[s])
