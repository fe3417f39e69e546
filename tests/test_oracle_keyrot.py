"""Pins of the oracle's per-width-group key rotation (CPU).

Reading: keys keep the per-block widths and scales; inside each group of
blocks of one width the scaled coordinates are rotated by randomised
Walsh-Hadamard chunks (binary expansion of the group's size) before the
width's Lloyd-Max codes, and decoding applies the inverse rotation. Pinned
against an independent matrix formulation, the orthogonality of the
transform, the textbook distortion of a Gaussian source, the SplitMix64
stream, and its effect on an outlier.
"""
import numpy as np
import pytest
from scipy.linalg import hadamard

from oracle import alloc, attn, lloydmax, quant
from oracle.splitmix import k_signs, splitmix64


def _plan(rng, bits, rotate=True, uniform=False):
    E = np.exp(1.5 * rng.standard_normal(64) - np.arange(64) / 8.0)
    return alloc.make_plan(E, bits, 2, 7, 3, 1, uniform=uniform, rotate_keys=rotate)


def test_chunks_partition_each_width_group():
    rng = np.random.default_rng(0)
    for bits in range(1, 9):
        p = _plan(rng, bits)
        ch = alloc.rot_chunks(p.widths, p.order)
        covered = []
        for P0, sz, w in ch:
            assert sz & (sz - 1) == 0 and 1 <= sz <= 128
            covered += list(range(P0, P0 + sz))
            # every position of a chunk belongs to a rank of width w
            assert all(p.widths[p.order[P // 2]] == w for P in range(P0, P0 + sz))
        assert covered == list(range(2 * len(p.order)))
        # within a group: sizes strictly decreasing (binary expansion, largest first)
        by_w = {}
        for P0, sz, w in ch:
            by_w.setdefault(w, []).append(sz)
        for w, sizes in by_w.items():
            n = sum(1 for j in p.order if p.widths[j] == w)
            assert sum(sizes) == 2 * n and sizes == sorted(sizes, reverse=True)
            assert len(set(sizes)) == len(sizes)


def test_rot_scale_and_signs():
    for e in range(8):
        c = float(quant.rot_scale(1 << e))
        assert abs(c * c * (1 << e) - 1.0) < 2 ** -22
        if e % 2 == 0:
            assert c == 2.0 ** (-e // 2)
    assert np.float32(np.sqrt(0.5)) == np.float32(0.70710678118654752)
    key = splitmix64(7, (3 << 32) + 1)
    ref = [-1 if splitmix64(key, 128 + P) >> 63 else 1 for P in range(128)]
    assert k_signs(7, 3, 1) == ref
    assert _plan(np.random.default_rng(1), 3).k_signs.tolist() == ref


@pytest.mark.parametrize("bits", [1, 2, 3, 5, 8])
def test_codes_equal_matrix_formulation(bits):
    """y = c H diag(s) z per chunk with scipy's Hadamard in fp64: the codes
    agree with the oracle's fp32 butterflies except within 1e-5 of a
    threshold."""
    rng = np.random.default_rng(bits)
    p = _plan(rng, bits)
    k = rng.standard_normal((200, 128)) * np.sqrt(np.concatenate([p.energy, p.energy]))[None] \
        + (rng.random((200, 128)) < 0.01) * 20.0
    codes, n, _ = quant.quantize_keys(k, p)
    k32 = k.astype(np.float32)
    r = (np.float32(1.0) / n).astype(np.float64)
    order = list(p.order)
    coord = [order[P // 2] + 64 * (P % 2) for P in range(2 * len(order))]
    checked = 0
    for P0, sz, w in alloc.rot_chunks(p.widths, order):
        idx = [coord[P0 + q] for q in range(sz)]
        z = k32[:, idx].astype(np.float64) * r[:, None] * p.g[[i % 64 for i in idx]].astype(np.float64)
        y = (z * p.k_signs[P0:P0 + sz][None]) @ hadamard(sz).T / np.sqrt(sz)
        thr = lloydmax.thresholds(w).astype(np.float64)
        ref = np.searchsorted(thr, y, side="left")
        near = np.min(np.abs(y[..., None] - thr[None, None, :]), axis=-1) < 1e-5 * (1 + np.abs(y))
        got = codes[:, idx]
        assert np.all((got == ref) | near)
        checked += np.sum(~near)
    assert checked > 1000


def test_inverse_and_gaussian_distortion():
    """A uniform plan (one group of 128 positions, one 128-point chunk) on an
    isotropic Gaussian: the rotated coordinates are again N(0, 1), so the
    relative error is the textbook Lloyd-Max D(b) (within sampling error);
    a wrong inverse (sign, transpose, scale) would not be."""
    rng = np.random.default_rng(5)
    E = np.ones(64)
    for b in (2, 3, 4):
        p = alloc.make_plan(E, b, 2, 1, 0, 0, uniform=True, rotate_keys=True)
        assert alloc.rot_chunks(p.widths, p.order) == [(0, 128, b)]
        k = rng.standard_normal((4000, 128))
        codes, n, _ = quant.quantize_keys(k, p)
        kh = attn.dequant_keys(codes, n, p)
        rel = np.sum((k - kh) ** 2) / np.sum(k ** 2)
        assert abs(rel / lloydmax.D(b) - 1.0) < 0.05, (b, rel, lloydmax.D(b))


def test_rotation_spreads_an_outlier():
    """One coordinate 30x the others: without rotation its block's codebook
    clips it; with rotation its energy is spread over the chunk and the key
    error drops."""
    rng = np.random.default_rng(6)
    E = np.ones(64)
    k = rng.standard_normal((500, 128))
    k[:, 5] *= 30.0
    errs = []
    for rot in (False, True):
        p = alloc.make_plan(E, 3, 2, 1, 0, 0, uniform=True, rotate_keys=rot)
        codes, n, _ = quant.quantize_keys(k, p)
        errs.append(np.sum((k - attn.dequant_keys(codes, n, p)) ** 2))
    assert errs[1] < 0.5 * errs[0]


def test_no_rotation_flag_is_the_plain_quantizer():
    rng = np.random.default_rng(7)
    p0 = _plan(rng, 3, rotate=False)
    p1 = alloc.make_plan(p0.energy, 3, 2, 7, 3, 1, rotate_keys=False)
    k = rng.standard_normal((50, 128))
    assert np.array_equal(quant.quantize_keys(k, p0)[0], quant.quantize_keys(k, p1)[0])
    assert p1.k_signs is None and not p1.k_rot
