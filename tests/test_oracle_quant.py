"""Pins of the oracle quantizers: fp32 decision recipe, FWHT, MSE (CPU)."""
import math

import numpy as np
import pytest

from oracle import alloc, attn, lloydmax, quant


def _plan(widths, bits_k, bits_v, E=None):
    E = np.ones(64) if E is None else np.asarray(E, dtype=np.float64)
    g, ah = alloc.key_scales(E)
    w = np.asarray(widths)
    from oracle.splitmix import v_signs
    return alloc.Plan(bits_k=bits_k, bits_v=bits_v, widths=w, order=alloc.plan_order(w),
                      g=g, a_hat=ah, signs=np.array(v_signs(7, 0, 0), dtype=np.float64), energy=E)


def test_sumsq_tree_exact_on_integers():
    rng = np.random.default_rng(0)
    x = rng.integers(-50, 50, (20, 128)).astype(np.float32)
    assert np.array_equal(quant.sumsq_tree(x), (x.astype(np.int64) ** 2).sum(1).astype(np.float32))


def test_sumsq_tree_order_matters_and_is_fixed():
    # values where fp32 rounding depends on order: the tree gives one result,
    # within the fp32 error bound of the exact sum
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((1000, 128)) * np.exp(rng.standard_normal((1000, 128)) * 3)).astype(np.float32)
    s = quant.sumsq_tree(x).astype(np.float64)
    ex = np.array([math.fsum(r) for r in x.astype(np.float64) ** 2])
    assert np.all(np.abs(s - ex) <= 8 * 2.0 ** -24 * ex)


def test_fwht_is_hadamard():
    H = attn.hadamard(128)
    assert np.array_equal(H @ H, 128 * np.eye(128))
    e = np.eye(128, dtype=np.float32)
    assert np.array_equal(quant.fwht_f32(e), H.T.astype(np.float32))
    rng = np.random.default_rng(2)
    xi = rng.integers(-9, 9, (5, 128)).astype(np.float32)
    assert np.array_equal(quant.fwht_f32(quant.fwht_f32(xi)), 128 * xi)
    x = rng.standard_normal((5, 128)).astype(np.float32)
    y = quant.fwht_f32(x).astype(np.float64)
    assert np.allclose((y ** 2).sum(1), 128 * (x.astype(np.float64) ** 2).sum(1), rtol=1e-5)


@pytest.mark.parametrize("b", range(1, 9))
def test_codes_threshold_rule(b):
    c16 = lloydmax.centroids(b).astype(np.float32)
    # each frozen centroid codes to its own index
    assert np.array_equal(quant.codes_from_z(c16, b), np.arange(1 << b))
    t = lloydmax.thresholds(b)
    # exactly on a threshold: the lower index (strict "<")
    assert np.array_equal(quant.codes_from_z(t, b), np.arange((1 << b) - 1))
    up = np.nextafter(t, np.float32(np.inf))
    assert np.array_equal(quant.codes_from_z(up, b), np.arange(1, 1 << b))
    assert quant.codes_from_z(np.float32(np.nan), b) == 0
    assert quant.codes_from_z(np.float32(-np.inf), b) == 0
    assert quant.codes_from_z(np.float32(np.inf), b) == (1 << b) - 1


def test_norm_is_fp16_of_fp32_sqrt():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((64, 128)).astype(np.float32)
    n, sat = quant.fp16_norm(quant.sumsq_tree(x))
    ref = np.sqrt(quant.sumsq_tree(x)).astype(np.float16).astype(np.float32)
    assert np.array_equal(n, ref) and not sat.any()
    n, sat = quant.fp16_norm(np.float32([70000.0 ** 2, 65519.0 ** 2]))
    assert n.tolist() == [65504.0, 65504.0] and sat.tolist() == [True, False]


def test_key_decision_recipe_by_hand():
    # one token, every block 2 bits: z_i = fp32(fp32(k_i r) g_j)
    plan = _plan([2] * 64, 2, 2)
    rng = np.random.default_rng(4)
    k = rng.standard_normal(128).astype(np.float32)
    codes, n, fl = quant.quantize_keys(k[None, :], plan)
    sq = np.float32(0)
    nn = np.sqrt(quant.sumsq_tree(k[None, :])[0]).astype(np.float16).astype(np.float32)
    assert n[0] == nn and fl[0] == 0
    r = np.float32(1) / nn
    thr = lloydmax.thresholds(2)
    for i in range(128):
        z = np.float32(np.float32(k[i] * r) * plan.g[i % 64])
        assert codes[0, i] == int(np.sum(thr < z))
    del sq


def test_edge_tokens():
    plan = _plan([2] * 64, 2, 2)
    k = np.zeros((3, 128), dtype=np.float32)
    k[1, 7] = np.nan
    k[2, :] = 1e30  # sumsq overflows fp32
    codes, n, fl = quant.quantize_keys(k, plan)
    assert codes[0].max() == 0 and n[0] == 0 and fl[0] == 0
    assert codes[1].max() == 0 and n[1] == 0 and fl[1] == quant.FLAG_NONFINITE
    assert n[2] == 65504 and fl[2] == quant.FLAG_NORM_SAT
    vc, vn, vf = quant.quantize_values(k, plan)
    assert vc[0].max() == 0 and vc[1].max() == 0 and vf[1] == quant.FLAG_NONFINITE


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_value_mse_matches_lloydmax(b):
    # isotropic Gaussian values: the rotated, normalised coordinates are close
    # to N(0,1), so the relative MSE is close to D(b)
    plan = _plan([b] * 64, b, b)
    rng = np.random.default_rng(10 + b)
    v = rng.standard_normal((4000, 128))
    vb = v.astype(np.float32)
    codes, n, _ = quant.quantize_values(vb, plan)
    vh = attn.dequant_values(codes, n, plan)
    rel = np.sum((vh - vb) ** 2) / np.sum(vb.astype(np.float64) ** 2)
    assert abs(rel - lloydmax.D(b)) / lloydmax.D(b) < 0.03


@pytest.mark.parametrize("b", [1, 2, 3])
def test_key_mse_matches_lloydmax(b):
    plan = _plan([b] * 64, b, b)
    rng = np.random.default_rng(20 + b)
    k = rng.standard_normal((4000, 128)).astype(np.float32)
    codes, n, _ = quant.quantize_keys(k, plan)
    kh = attn.dequant_keys(codes, n, plan)
    rel = np.sum((kh - k) ** 2) / np.sum(k.astype(np.float64) ** 2)
    assert abs(rel - lloydmax.D(b)) / lloydmax.D(b) < 0.03


def _sphere_distortion(b, d=128):
    """E[(x - q_b(x))^2] for x = sqrt(d) u_1, u uniform on the unit sphere of
    R^d (the coordinate a token's normalised vector presents to the
    quantizer), q_b the frozen centroids and thresholds of width b. The
    coordinate's density is C (1 - x^2 / d)^((d - 3) / 2) on [-sqrt(d),
    sqrt(d)] with C = Gamma(d/2) / (Gamma((d-1)/2) sqrt(pi d)); integrated
    cell by cell by quadrature."""
    from scipy import integrate, special

    logc = special.gammaln(d / 2) - special.gammaln((d - 1) / 2) - 0.5 * np.log(np.pi * d)

    def dens(x):
        return np.exp(logc + (d - 3) / 2 * np.log1p(-x * x / d))

    c = lloydmax.centroids(b)
    edges = np.concatenate([[-np.sqrt(d)], lloydmax.thresholds(b).astype(np.float64),
                            [np.sqrt(d)]])
    return sum(integrate.quad(lambda x: (x - c[k]) ** 2 * dens(x), edges[k], edges[k + 1],
                              limit=200, epsabs=1e-15, epsrel=1e-12)[0] for k in range(len(c)))


@pytest.mark.parametrize("b", range(1, 9))
def test_mse_matches_sphere_quadrature_every_width(b):
    # keys and values of isotropic Gaussian tokens: after the norm (and, for
    # values, the rotation) each coordinate is sqrt(128) times a coordinate of
    # a uniform unit vector, so the relative MSE is the quantizer's exact
    # distortion under that density (a little below the Gaussian D(b)); 4000
    # tokens give about 0.5 % of sampling spread
    plan = _plan([b] * 64, b, b)
    ds = _sphere_distortion(b)
    rng = np.random.default_rng(300 + b)
    k = rng.standard_normal((4000, 128)).astype(np.float32)
    codes, n, _ = quant.quantize_keys(k, plan)
    kh = attn.dequant_keys(codes, n, plan)
    rel_k = np.sum((kh - k) ** 2) / np.sum(k.astype(np.float64) ** 2)
    v = rng.standard_normal((4000, 128)).astype(np.float32)
    codes, n, _ = quant.quantize_values(v, plan)
    vh = attn.dequant_values(codes, n, plan)
    rel_v = np.sum((vh - v) ** 2) / np.sum(v.astype(np.float64) ** 2)
    assert abs(rel_k - ds) / ds < 0.02, (rel_k, ds)
    assert abs(rel_v - ds) / ds < 0.02, (rel_v, ds)
    assert ds < lloydmax.D(b)  # lighter tails than the Gaussian


def test_key_block_widths_respected():
    w = np.zeros(64, dtype=int)
    w[[0, 1, 2]] = [8, 3, 1]
    plan = _plan(w, 1, 1)
    rng = np.random.default_rng(5)
    k = rng.standard_normal((500, 128)).astype(np.float32)
    codes, _, _ = quant.quantize_keys(k, plan)
    for j, wj in enumerate(w):
        for i in (j, j + 64):
            assert codes[:, i].max() <= (1 << wj) - 1 if wj else codes[:, i].max() == 0
    assert codes[:, 0].max() > 200
