"""Pins of the oracle's recent-token window (CPU).

The window reading: the R most recent tokens stay exact, older ones are
quantized in order as they leave, decode attends over both. Pinned against
a step-by-step simulation of appends and evictions, the plain attention
definition at the two ends (no window, everything in the window) and the
range-combine identity.
"""
import numpy as np
import pytest
from scipy.special import softmax

from oracle import alloc, attn, quant, window


def _plan(rng):
    E = np.exp(rng.standard_normal(64) - np.arange(64) / 8.0)
    return alloc.make_plan(E, 3, 2, v_seed=4, layer=0, kv_head=0)


def _simulate(appends, R):
    """Evict oldest-first whenever the window would hold more than R tokens."""
    packed, win, t = [], [], 0
    for n in appends:
        win.extend(range(t, t + n))
        t += n
        while len(win) > R:
            packed.append(win.pop(0))
    return packed, win


@pytest.mark.parametrize("R", [0, 1, 5, 32, 100])
def test_split_point_matches_a_simulation_of_appends(R):
    rng = np.random.default_rng(R)
    for _ in range(50):
        appends = rng.integers(0, 40, size=rng.integers(1, 12)).tolist()
        packed, win = _simulate(appends, R)
        T = sum(appends)
        sp = window.split_point(T, R)
        assert packed == list(range(sp))
        assert win == list(range(sp, T))
        if R:
            slots = [s for _, s in window.ring_slots(T, R)]
            assert len(set(slots)) == len(slots)  # a token per slot
            assert all(s == t % R for t, s in window.ring_slots(T, R))


def test_no_window_is_the_packed_decode():
    rng = np.random.default_rng(1)
    plan = _plan(rng)
    k, v = rng.standard_normal((300, 128)), rng.standard_normal((300, 128))
    q = rng.standard_normal((4, 128))
    kc, kn, _ = quant.quantize_keys(k, plan)
    vc, vn, _ = quant.quantize_values(v, plan)
    kh, vh = attn.dequant_keys(kc, kn, plan), attn.dequant_values(vc, vn, plan)
    empty = np.zeros((0, 128))
    got = window.decode(q, [kh], [vh], [empty], [empty])
    assert np.array_equal(got, attn.decode(q, [kh], [vh]))


def test_all_in_window_is_exact_attention():
    rng = np.random.default_rng(2)
    k, v = rng.standard_normal((70, 128)), rng.standard_normal((70, 128))
    q = rng.standard_normal((8, 128))
    empty = np.zeros((0, 128))
    got = window.decode(q, [empty, empty], [empty, empty], [k[:35], k[35:]], [v[:35], v[35:]])
    # textbook attention, per query head, KV head floor(h / 4)
    for h in range(8):
        kk, vv = (k[:35], v[:35]) if h < 4 else (k[35:], v[35:])
        p = softmax(kk @ q[h] / np.sqrt(128.0))
        np.testing.assert_allclose(got[h], p @ vv, rtol=1e-12, atol=1e-13)


def test_mixed_equals_combined_ranges():
    rng = np.random.default_rng(3)
    plan = _plan(rng)
    T, R = 400, 48
    k, v = rng.standard_normal((T, 128)), rng.standard_normal((T, 128))
    q = rng.standard_normal((4, 128))
    sp = window.split_point(T, R)
    kc, kn, _ = quant.quantize_keys(k[:sp], plan)
    vc, vn, _ = quant.quantize_values(v[:sp], plan)
    kh, vh = attn.dequant_keys(kc, kn, plan), attn.dequant_values(vc, vn, plan)
    got = window.decode(q, [kh], [vh], [k[sp:]], [v[sp:]])
    r1 = attn.range_record(q, kh, vh)
    r2 = attn.range_record(q, k[sp:], v[sp:])
    ref = attn.combine_ranges(np.stack([r1[0], r2[0]]), np.stack([r1[1], r2[1]]))
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)
    # the window tokens really are exact: a window token equal to a packed
    # token's dequantized key/value would be indistinguishable, so check
    # that quantizing them instead changes the output
    kc2, kn2, _ = quant.quantize_keys(k, plan)
    vc2, vn2, _ = quant.quantize_values(v, plan)
    allq = attn.decode(q, [attn.dequant_keys(kc2, kn2, plan)],
                       [attn.dequant_values(vc2, vn2, plan)])
    assert np.max(np.abs(allq - got)) > 1e-6
