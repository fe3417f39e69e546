"""Pins of the oracle tile layout and exact attention (CPU)."""
import json
import os

import numpy as np
import pytest
from scipy.special import softmax

from oracle import alloc, attn, layout
from oracle.splitmix import v_signs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _plan(widths, bits_k, bits_v):
    w = np.asarray(widths)
    g, ah = alloc.key_scales(np.ones(64))
    return alloc.Plan(bits_k=bits_k, bits_v=bits_v, widths=w, order=alloc.plan_order(w),
                      g=g, a_hat=ah, signs=np.array(v_signs(1, 0, 0), dtype=np.float64))


def _random_plan(rng, bits_k, bits_v):
    # random widths in 0..8 with sum 64 bits_k
    w = np.zeros(64, dtype=int)
    left = 64 * bits_k
    while left:
        j = rng.integers(64)
        if w[j] < 8:
            w[j] += 1
            left -= 1
    return _plan(w, bits_k, bits_v)


def test_slot_orders_are_permutations():
    assert sorted(layout.slot_k(np.arange(32)).tolist()) == list(range(32))
    assert sorted(layout.slot_v(np.arange(32)).tolist()) == list(range(32))
    # fragment contiguity: slots 4g..4g+3 hold tokens g, g+8, g+16, g+24
    for g in range(8):
        assert [layout.slot_k(g + 8 * i) for i in range(4)] == [4 * g + i for i in range(4)]
    # slots 8c..8c+7 hold tokens 2c + 8i + e
    for c in range(4):
        assert [layout.slot_v(2 * c + 8 * i + e) for i in range(4) for e in range(2)] == \
            list(range(8 * c, 8 * c + 8))


@pytest.mark.parametrize("bits", [(1, 1), (2, 2), (3, 2), (3, 3), (8, 8), (5, 1)])
def test_round_trip_and_sizes(bits):
    rng = np.random.default_rng(sum(bits))
    plan = _random_plan(rng, *bits)
    L = 100
    kc = np.zeros((L, 128), dtype=np.int64)
    for j in range(64):
        w = plan.widths[j]
        kc[:, j] = rng.integers(0, 1 << w, L)
        kc[:, j + 64] = rng.integers(0, 1 << w, L)
    vc = rng.integers(0, 1 << plan.bits_v, (L, 128))
    kn = rng.standard_normal(L).astype(np.float16).astype(np.float32)
    vn = rng.standard_normal(L).astype(np.float16).astype(np.float32)
    rec = layout.pack(kc, vc, kn, vn, plan, L)
    assert rec.shape == (4, layout.tile_words(*bits))
    # code bits per token = 128 (b_K + b_V) exactly; norms 2 x 2 bytes
    assert layout.tile_bytes(*bits) == 32 * (16 * (bits[0] + bits[1]) + 4)
    kc2, vc2, kn2, vn2 = layout.unpack(rec, plan, L)
    assert np.array_equal(kc2, kc) and np.array_equal(vc2, vc)
    assert np.array_equal(kn2, kn) and np.array_equal(vn2, vn)
    # positions 100..127 hold no token: their code bits are zero
    kc3, vc3, _, _ = layout.unpack(rec, plan, 128)
    assert kc3[L:].max() == 0 and vc3[L:].max() == 0


def test_golden_hand_worked_tile():
    with open(os.path.join(GOLDEN, "layout_hand_tile.json")) as f:
        g = json.load(f)
    w = np.zeros(64, dtype=int)
    for j in g["blocks_width8"]:
        w[j] = 8
    plan = _plan(w, g["bits_k"], g["bits_v"])
    L = g["length"]
    kc = np.zeros((L, 128), dtype=np.int64)
    vc = np.zeros((L, 128), dtype=np.int64)
    kn = np.zeros(L, dtype=np.float32)
    vn = np.zeros(L, dtype=np.float32)
    for t, i, c in g["k_codes"]:
        kc[t, i] = c
    for t, p, c in g["v_codes"]:
        vc[t, p] = c
    for t, x in g["k_norm"]:
        kn[t] = x
    for t, x in g["v_norm"]:
        vn[t] = x
    rec = layout.pack(kc, vc, kn, vn, plan, L)[0]
    expect = np.zeros(layout.tile_words(g["bits_k"], g["bits_v"]), dtype=np.uint32)
    for idx, val in g["nonzero_words"]:
        expect[idx] = int(val, 16)
    assert np.array_equal(rec, expect)


def test_attention_bypass_equals_textbook():
    rng = np.random.default_rng(0)
    q = rng.standard_normal((4, 128))
    k = rng.standard_normal((300, 128))
    v = rng.standard_normal((300, 128))
    o = attn.attention(q, k, v)
    ref = np.array([softmax(q[h] @ k.T / np.sqrt(128)) @ v for h in range(4)])
    assert np.allclose(o, ref, rtol=1e-12, atol=1e-13)
    # a second formula: log-sum-exp with explicit loops on one head
    s = [float(np.dot(q[1], k[t])) / np.sqrt(128) for t in range(300)]
    m = max(s)
    w = [np.exp(x - m) for x in s]
    o1 = sum(wi * v[t] for t, wi in enumerate(w)) / sum(w)
    assert np.allclose(o[1], o1, rtol=1e-11)


def test_attention_special_cases():
    rng = np.random.default_rng(1)
    q = rng.standard_normal((2, 128))
    v = rng.standard_normal((1, 128))
    assert np.allclose(attn.attention(q, rng.standard_normal((1, 128)), v), np.repeat(v, 2, 0))
    k = np.repeat(rng.standard_normal((1, 128)), 50, 0)
    v = rng.standard_normal((50, 128))
    assert np.allclose(attn.attention(q, k, v), np.repeat(v.mean(0, keepdims=True), 2, 0))
    assert np.array_equal(attn.attention(q, np.zeros((0, 128)), np.zeros((0, 128))), np.zeros_like(q))


def test_gqa_mapping():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((6, 128))
    ks = [rng.standard_normal((20, 128)) for _ in range(2)]
    vs = [rng.standard_normal((20, 128)) for _ in range(2)]
    o = attn.decode(q, ks, vs)
    assert np.allclose(o[4], attn.attention(q[4:5], ks[1], vs[1])[0])
    assert np.allclose(o[2], attn.attention(q[2:3], ks[0], vs[0])[0])


def test_range_records_combine_to_attention_over_all_tokens():
    """Context shards: the combine of the ranges' records equals softmax
    attention over every token (pinned to the textbook form above), for cut
    points that leave empty and one-token ranges."""
    from scipy.special import logsumexp
    rng = np.random.default_rng(5)
    T, Hg = 300, 4
    q = rng.standard_normal((Hg, 128)) * 2.0
    k = rng.standard_normal((T, 128))
    v = rng.standard_normal((T, 128))
    full = attn.attention(q, k, v)
    for cuts in ([0, 0, 150, 300, 300], [0, 1, 2, 299, 300], [0, 77, 133, 134, 300]):
        recs = [attn.range_record(q, k[a:b], v[a:b]) for a, b in zip(cuts[:-1], cuts[1:])]
        lse = np.stack([r[0] for r in recs])
        o = np.stack([r[1] for r in recs])
        assert np.max(np.abs(attn.combine_ranges(lse, o) - full)) < 1e-12
        for (a, b), l in zip(zip(cuts[:-1], cuts[1:]), lse):
            if b > a:  # log2 sum 2^s from the library's natural-log logsumexp
                s = q @ k[a:b].T / np.sqrt(128.0)
                assert np.allclose(l, logsumexp(s, axis=1) / np.log(2.0), rtol=0, atol=1e-12)
            else:
                assert np.all(l == -np.inf)
    # one token: lse2 is its own base-2 logit and the output its value
    l1, o1 = attn.range_record(q, k[:1], v[:1])
    assert np.allclose(l1, (q @ k[0]) / np.sqrt(128.0) * np.log2(np.e), rtol=0, atol=1e-12)
    assert np.allclose(o1, np.broadcast_to(v[0], o1.shape), rtol=0, atol=1e-12)
    # every range empty: output 0
    le, oe = attn.range_record(q, k[:0], v[:0])
    assert np.all(attn.combine_ranges(np.stack([le, le]), np.stack([oe, oe])) == 0.0)
