"""Pins of the oracle's Gaussian Lloyd-Max codebooks (CPU)."""
import math

import numpy as np
import pytest
from scipy.integrate import quad
from scipy.stats import norm

from oracle import lloydmax


# Published Lloyd-Max distortions of the unit Gaussian at 1, 2 and 3 bits,
# quoted to 4 significant digits.
@pytest.mark.parametrize("b,pin", [(1, 0.3634), (2, 0.1175), (3, 0.03454)])
def test_distortion_pins(b, pin):
    d = lloydmax.D(b)
    # within one unit of the last quoted digit: 0.3634 and 0.1175 are the
    # rounded values, 0.03454 the truncated one (D(3) = 0.0345478)
    assert abs(d - pin) < 10 ** (math.floor(math.log10(pin)) - 3)


def test_one_bit_closed_form():
    # 1-bit Lloyd-Max of N(0,1): centroids +-E|X| = +-sqrt(2/pi), D = 1 - 2/pi
    c = np.array(lloydmax.tables()["centroids_fp64"][1])
    assert np.allclose(c, [-math.sqrt(2 / math.pi), math.sqrt(2 / math.pi)], atol=1e-13)
    assert abs(lloydmax.D(1) - (1 - 2 / math.pi)) < 1e-13


def test_d0_and_monotone_convex():
    D = [lloydmax.D(b) for b in range(9)]
    assert D[0] == 1.0
    dd = np.diff(D)
    assert np.all(dd < 0)                 # more bits, less distortion
    assert np.all(np.diff(-dd) < 0)       # gains shrink: convex, greedy is optimal


def test_high_rate_trend():
    # Panter-Dite: D(b) 4^b -> sqrt(3) pi / 2 for a unit Gaussian
    lim = math.sqrt(3) * math.pi / 2
    r = [lloydmax.D(b) * 4 ** b for b in range(4, 9)]
    assert all(x < lim for x in r)
    assert abs(r[-1] - lim) / lim < 0.02
    assert np.all(np.diff(r) > 0)


@pytest.mark.parametrize("b", range(1, 9))
def test_fixed_point_conditions(b):
    c = np.array(lloydmax.tables()["centroids_fp64"][b])
    assert np.allclose(c, -c[::-1], atol=0)                     # symmetric
    t = 0.5 * (c[1:] + c[:-1])
    _, mean = lloydmax.interval_stats(t)
    assert np.max(np.abs(mean - c)) < 1e-9                       # centroid condition
    assert np.all(np.diff(c) > 0)


@pytest.mark.parametrize("b", [2, 3, 4])
def test_distortion_by_quadrature(b):
    # an independent numerical integral of (x - q(x))^2 phi(x)
    c = np.array(lloydmax.tables()["centroids_fp64"][b])
    t = 0.5 * (c[1:] + c[:-1])
    edges = np.concatenate([[-np.inf], t, [np.inf]])
    tot = sum(quad(lambda x, ci=ci: (x - ci) ** 2 * norm.pdf(x), edges[i], edges[i + 1],
                   epsabs=1e-15, epsrel=1e-13)[0] for i, ci in enumerate(c))
    assert abs(tot - lloydmax.D(b)) < 1e-12


def test_literature_values():
    # Max (1960) tables, 4 digits: 2-bit levels +-0.4528, +-1.510; 16-level D ~ 0.009497
    c2 = np.array(lloydmax.tables()["centroids_fp64"][2])
    assert np.allclose(np.abs(c2), [1.510, 0.4528, 0.4528, 1.510], atol=6e-4)
    assert abs(lloydmax.D(4) - 0.009497) / 0.009497 < 1e-3


@pytest.mark.parametrize("b", range(1, 9))
def test_frozen_tables(b):
    c = np.array(lloydmax.tables()["centroids_fp64"][b])
    c16 = lloydmax.centroids(b)
    # fp16-exact, and the RNE rounding of the solver's centroids
    assert np.array_equal(c16.astype(np.float16).astype(np.float64), c16)
    assert np.array_equal(c.astype(np.float16).astype(np.float64), c16)
    assert len(np.unique(c16)) == 1 << b
    # every centroid is far (vs solver accuracy) from an fp16 rounding boundary
    up = np.nextafter(c16.astype(np.float16), np.float16(np.inf)).astype(np.float64)
    dn = np.nextafter(c16.astype(np.float16), np.float16(-np.inf)).astype(np.float64)
    margin = np.minimum(0.5 * (up - c16) - (c - c16), (c - c16) - 0.5 * (dn - c16))
    assert np.min(margin) > 1e-8
    thr = lloydmax.thresholds(b)
    assert thr.dtype == np.float32
    assert np.array_equal(thr.astype(np.float64), 0.5 * (c16[1:] + c16[:-1]))


def test_tables_file_matches_solver():
    # the committed tables are what the solver writes (b <= 4: fast to re-solve)
    for b in range(1, 5):
        c, d, _ = lloydmax.solve(b)
        assert abs(d - lloydmax.D(b)) < 1e-14
        assert np.array_equal(lloydmax.freeze(c)[0], lloydmax.centroids(b))
