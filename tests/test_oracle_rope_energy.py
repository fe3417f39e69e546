"""Pins of the oracle's RoPE block identity and block energy (CPU)."""
from fractions import Fraction

import numpy as np
import pytest

from oracle import energy, rope


@pytest.mark.parametrize("base", [1e4, 5e5, 1e6])
def test_rope_block_identity(base):
    rng = np.random.default_rng(1)
    for _ in range(20):
        q, k = rng.standard_normal(128), rng.standard_normal(128)
        m, n = rng.integers(0, 200000, 2)
        lhs = rope.rotate(q, m, base) @ rope.rotate(k, n, base)
        terms = rope.block_terms(q, k, m, n, base)
        assert terms.shape == (64,)
        assert abs(lhs - terms.sum()) < 1e-9 * (1 + abs(lhs))


def test_rope_textbook_two_by_two():
    # block j rotated by pos * base^(-2j/d), independently of other blocks
    x = np.zeros(128)
    x[5], x[69] = 1.0, 0.0
    y = rope.rotate(x, 3, 1e4)
    a = 3 * 1e4 ** (-2 * 5 / 128)
    assert np.allclose([y[5], y[69]], [np.cos(a), np.sin(a)], atol=1e-15)
    assert np.count_nonzero(np.abs(y) > 1e-18) == 2


def test_rope_orthogonal_and_energy_invariant():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((50, 128))
    y = rope.rotate(x, np.arange(50), 5e5)
    bx = x[:, :64] ** 2 + x[:, 64:] ** 2
    by = y[:, :64] ** 2 + y[:, 64:] ** 2
    assert np.allclose(bx, by, rtol=1e-12, atol=1e-15)


def test_energy_exact_integer_brute_force():
    # tiny input: S_j equals the exact rational sum of floor(k^2 2^32)
    rng = np.random.default_rng(3)
    k = np.float32(rng.standard_normal((5, 2, 128)) * 0.3).astype(np.float64)
    S, fl = energy.block_energy_int(k)
    assert fl == 0
    for h in range(2):
        for j in (0, 17, 63):
            ref = 0
            for t in range(5):
                for i in (j, j + 64):
                    ref += int(Fraction(k[t, h, i]) ** 2 * 2 ** 32 // 1)
            assert S[h][j] == ref


def test_energy_order_independent_and_close_to_fp64():
    rng = np.random.default_rng(4)
    k = np.float32(rng.standard_normal((777, 3, 128))).astype(np.float64)
    S1, _ = energy.block_energy_int(k)
    S2, _ = energy.block_energy_int(k[rng.permutation(777)])
    assert S1 == S2
    E, _ = energy.block_energy(k)
    ref = (k[:, :, :64] ** 2 + k[:, :, 64:] ** 2).mean(axis=0)
    # the 2^-32 grid truncates at most 2^-32 per term
    assert np.all(np.abs(E - ref) <= 2 * 2.0 ** -32 + 1e-15 * ref)


def test_energy_rope_invariant():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((400, 1, 128))
    y = rope.rotate(x[:, 0], np.arange(400), 1e4)[:, None, :]
    Ex, _ = energy.block_energy(x)
    Ey, _ = energy.block_energy(y)
    assert np.allclose(Ex, Ey, rtol=1e-7)


def test_energy_flags_and_saturation():
    k = np.zeros((2, 1, 128))
    k[0, 0, 3] = np.nan
    k[1, 0, 4] = 2.0 ** 20          # k^2 2^32 = 2^72 saturates
    S, fl = energy.block_energy_int(k)
    assert fl == energy.FLAG_NONFINITE
    assert S[0][3] == 0
    assert S[0][4] == 2 ** 64 - 1


# ---- the fp32 recipe of the fused rotate-and-quantize path
@pytest.mark.parametrize("base", [1e4, 1e6])
def test_rope_f32_close_to_fp64_and_blockwise(base):
    rng = np.random.default_rng(9)
    x = np.float32(rng.standard_normal((300, 128)) * 3).astype(np.float64)
    pos = rng.integers(0, 600000, 300)
    y32 = rope.rotate_f32(x, pos, base)
    y64 = rope.rotate(x, pos, base)
    assert y32.dtype == np.float32
    # two fp32 products and one sum, each rounded, plus fp32 cos/sin: a few
    # units of 2^-24 of the block magnitude
    mag = np.sqrt(x[:, :64] ** 2 + x[:, 64:] ** 2)
    err = np.maximum(np.abs(y32[:, :64] - y64[:, :64]), np.abs(y32[:, 64:] - y64[:, 64:]))
    assert np.all(err <= 4 * 2.0 ** -24 * mag + 1e-30)
    # block j only mixes coordinates j and j + 64
    e = np.zeros(128)
    e[7] = 1.0
    z = rope.rotate_f32(e, 12345, base)
    a = 12345 * float(base) ** (-2 * 7 / 128)
    assert z[7] == np.float32(np.cos(a)) and z[71] == np.float32(np.sin(a))
    assert np.count_nonzero(z) == 2


def test_rope_f32_identity_at_position_zero():
    rng = np.random.default_rng(10)
    x = np.float32(rng.standard_normal((20, 128)))
    assert np.array_equal(rope.rotate_f32(x, np.zeros(20), 5e5), x)
