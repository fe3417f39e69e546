"""Pins of the oracle's greedy allocation, plan and sign generator (CPU)."""
import itertools

import numpy as np
import pytest

from oracle import alloc, lloydmax
from oracle.splitmix import splitmix64, v_signs


_COMBOS = np.array(list(itertools.product(range(9), repeat=4)))
_DTAB = np.array([lloydmax.D(b) for b in range(9)])


def _brute(E, bits):
    """Exhaustive optimum over all widths in 0..8 with sum 4 * bits."""
    c = _COMBOS[_COMBOS.sum(axis=1) == 4 * bits]
    f = (_DTAB[c] * np.asarray(E)[None, :]).sum(axis=1)
    best = f.min()
    near = np.abs(f - best) <= 1e-15 * best
    return best, tuple(c[np.argmin(f)]), int(near.sum())


def test_greedy_equals_brute_force_d8():
    # head size 8 = 4 RoPE blocks; every budget 1..8 b/dim; 120 seeds
    rng = np.random.default_rng(0)
    for seed in range(120):
        E = np.exp(rng.standard_normal(4) * 2.0)
        for bits in range(1, 9):
            w, _ = alloc.greedy(E, bits)
            assert w.sum() == 4 * bits
            best, arg, n_best = _brute(E, bits)
            f = alloc.objective(E, w)
            assert abs(f - best) <= 1e-12 * best
            if n_best == 1:
                assert tuple(w) == arg


def test_equal_energy_gives_uniform_and_tie_rule():
    for bits in range(0, 9):
        w, tie = alloc.greedy(np.ones(64), bits)
        assert np.all(w == bits) and not tie
    # one odd step: ties go to the lowest block index
    w, _ = alloc.greedy(np.ones(4), 1)
    assert w.tolist() == [1, 1, 1, 1]
    w, _ = alloc.greedy([1.0, 1.0, 1.0, 1.0], 0)
    assert w.tolist() == [0, 0, 0, 0]


def test_greedy_nested_and_energy_ordered():
    rng = np.random.default_rng(1)
    E = np.exp(rng.standard_normal(64))
    prev = np.zeros(64, dtype=int)
    for bits in range(1, 9):
        w, _ = alloc.greedy(E, bits)
        assert np.all(w >= prev)
        prev = w
        # more energy never gets fewer bits
        o = np.argsort(-E)
        assert np.all(np.diff(w[o]) <= 0)


def test_greedy_first_steps_by_hand():
    # two blocks, budget 1 b/dim = 2 steps; gains E_j (D(b) - D(b+1)) with
    # D(0)-D(1) = 2/pi = 0.6366, D(1)-D(2) = 0.2459
    D = lloydmax.D
    g0, g1 = D(0) - D(1), D(1) - D(2)
    # E = (1, 4): 4 g0 = 2.55 > 4 g1 = 0.98 > g0 = 0.64 -> block 1 twice
    assert 4 * g1 > g0
    assert alloc.greedy([1.0, 4.0], 1)[0].tolist() == [0, 2]
    # E = (1, 2): 2 g0 = 1.27 > g0 = 0.64 > 2 g1 = 0.49 -> one bit each
    assert g0 > 2 * g1
    assert alloc.greedy([1.0, 2.0], 1)[0].tolist() == [1, 1]


def test_key_scales():
    rng = np.random.default_rng(2)
    E = np.exp(rng.standard_normal(64))
    g, ah = alloc.key_scales(E)
    assert abs(2 * np.sum(ah.astype(np.float64) ** 2) - 1) < 1e-6
    assert np.allclose(g.astype(np.float64) * ah.astype(np.float64), 1, rtol=1e-6)
    E[5] = 0
    g, ah = alloc.key_scales(E)
    assert g[5] == 0 and ah[5] == 0


def test_plan_order():
    w = np.array([2, 0, 3, 2, 3] + [0] * 59)
    assert alloc.plan_order(w) == [2, 4, 0, 3]


def test_splitmix64_known_answers():
    # SplitMix64 reference implementation, seed 0: first three outputs
    assert splitmix64(0, 0) == 0xE220A8397B1DCDAF
    assert splitmix64(0, 1) == 0x6E789E6AA1B965F4
    assert splitmix64(0, 2) == 0x06C45D188009454F


def test_v_signs():
    s = v_signs(12345, 3, 1)
    assert len(s) == 128 and set(s) <= {-1, 1}
    assert s == v_signs(12345, 3, 1)
    assert s != v_signs(12345, 3, 0) and s != v_signs(12345, 2, 1)
    assert 40 < sum(1 for x in s if x > 0) < 88


def test_query_weighted_greedy():
    """Query-weighted variant: the widths minimise sum_j W_j E_j D(b_j)
    (exhaustive search at 4 blocks), constant weights change nothing, and the
    key scales stay those of E."""
    rng = np.random.default_rng(3)
    for seed in range(60):
        E = np.exp(rng.standard_normal(4) * 2.0)
        W = np.exp(rng.standard_normal(4) * 1.5)
        for bits in (1, 2, 3, 5):
            J = 4
            w = alloc.greedy(E * W, bits)[0]
            best, arg, n_best = _brute(E * W, bits)
            f = float((_DTAB[w] * E * W).sum())
            assert f <= best * (1 + 1e-12)
            if n_best == 1:
                assert tuple(w) == arg
            assert int(w.sum()) == J * bits
    E = np.exp(rng.standard_normal(64))
    W = np.exp(rng.standard_normal(64))
    base = alloc.make_plan(E, 3, 3, 1, 0, 0)
    for c in (1.0, 2.0, 0.125):           # powers of two: E * c is exact
        p = alloc.make_plan(E, 3, 3, 1, 0, 0, weights=np.full(64, c))
        assert np.array_equal(p.widths, base.widths)
    pw = alloc.make_plan(E, 3, 3, 1, 0, 0, weights=W)
    assert np.array_equal(pw.g, base.g) and np.array_equal(pw.a_hat, base.a_hat)
    assert int(pw.widths.sum()) == 64 * 3 and not np.array_equal(pw.widths, base.widths)


def test_query_weights_group_mean():
    """W[h] is the mean block energy of KV head h's query group: identical
    query heads give their own energy; two heads give the average."""
    from oracle import energy
    rng = np.random.default_rng(4)
    q = rng.standard_normal((50, 4, 128))
    q[:, 1] = q[:, 0]
    W, _ = energy.query_weights(q, 2)
    Eq, _ = energy.block_energy(q)
    assert np.array_equal(W[0], Eq[0])          # (a + a) / 2 = a exactly
    assert np.allclose(W[1], (Eq[2] + Eq[3]) / 2, rtol=1e-15, atol=0)
    # and each block energy is the textbook mean of the block's squared length
    ref = (q[:, 2, :64] ** 2 + q[:, 2, 64:] ** 2).mean(axis=0)
    assert np.allclose(Eq[2], ref, rtol=1e-9, atol=0)
