"""Host-side checks of libkvq on the CPU: exports, codebooks, plans, errors."""
import ctypes
import os
import re

import numpy as np
import pytest

from bit_kv_cache_19_b200 import kvq
from oracle import alloc, lloydmax

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "kvq.h")).read()
    return sorted(set(re.findall(r"KVQ_API\s+[\w\s\*]+?\b(kvq_\w+)\s*\(", src)))


def test_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 12
    L = kvq.lib()
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(kvq.EXPORTS)


@pytest.mark.parametrize("b", range(1, 9))
def test_library_codebook_equals_oracle(b):
    c, t, d = kvq.codebook(b)
    assert np.array_equal(c.astype(np.float64), lloydmax.centroids(b))
    assert np.array_equal(t, lloydmax.thresholds(b))
    assert abs(d - lloydmax.D(b)) <= 1e-10 * lloydmax.D(b)


def _energies(rng, n, kind):
    j = np.arange(64)
    if kind == "decay":
        return np.exp(-j / 6.0 + rng.standard_normal((n, 64)))
    if kind == "flat":
        return np.ones((n, 64))
    if kind == "zeros":
        E = np.exp(rng.standard_normal((n, 64)))
        E[:, ::3] = 0.0
        return E
    return np.exp(3 * rng.standard_normal((n, 64)))


@pytest.mark.parametrize("kind", ["decay", "flat", "zeros", "wild"])
@pytest.mark.parametrize("bits", [(1, 1), (2, 2), (3, 2), (3, 3), (4, 8), (8, 1)])
def test_plan_build_equals_oracle(kind, bits):
    rng = np.random.default_rng(hash((kind, bits)) % 2 ** 32)
    E = _energies(rng, 3, kind)
    bk, bv = bits
    for mode in (kvq.ALLOC_GREEDY, kvq.ALLOC_UNIFORM):
        cfg = kvq.make_cfg(3, bk, bv, v_seed=987654321, alloc_mode=mode)
        got = kvq.plan_build(cfg, 5, E)
        for h in range(3):
            ref = alloc.make_plan(E[h], bk, bv, 987654321, 5, h, uniform=mode == kvq.ALLOC_UNIFORM)
            assert not ref.near_tie or mode == kvq.ALLOC_UNIFORM or kind == "flat"
            p = got[h]
            assert p["magic"] == kvq.PLAN_MAGIC and p["layer"] == 5 and p["kv_head"] == h
            assert np.array_equal(p["width"].astype(int), ref.widths)
            assert p["n_ranks"] == len(ref.order)
            assert list(p["order"][:p["n_ranks"]]) == ref.order
            assert np.array_equal(p["g"], ref.g) and np.array_equal(p["a_hat"], ref.a_hat)
            signs = np.array([-1.0 if (p["v_sign"][i >> 5] >> (i & 31)) & 1 else 1.0
                              for i in range(128)])
            assert np.array_equal(signs, ref.signs)
            # segment offsets and the half-step schedule are consistent
            off = 0
            for r in range(p["n_ranks"]):
                assert p["seg_off"][r] == off
                off += 2 * int(p["width"][p["order"][r]])
            assert off == 128 * bk == p["seg_off"][p["n_ranks"]]
            covered = []
            for hs in range(p["n_half"]):
                r0, n, w = p["hs_rank0"][hs], p["hs_count"][hs], p["hs_width"][hs]
                assert 1 <= n <= 4
                assert all(p["width"][p["order"][r]] == w for r in range(r0, r0 + n))
                covered += list(range(r0, r0 + n))
            assert covered == list(range(p["n_ranks"]))
            assert p["n_half"] <= 24
            # classes: maximal runs of one width over the half steps
            hs = 0
            for ci in range(p["n_class"]):
                w, h0, n = p["cls_w"][ci], p["cls_hs0"][ci], p["cls_nhs"][ci]
                assert h0 == hs and n >= 1
                assert all(p["hs_width"][x] == w for x in range(h0, h0 + n))
                assert p["cls_last"][ci] == p["hs_count"][h0 + n - 1]
                assert p["cls_seg0"][ci] == p["seg_off"][p["hs_rank0"][h0]]
                hs += n
            assert hs == p["n_half"]
            assert len(set(p["cls_w"][:p["n_class"]])) == p["n_class"]


@pytest.mark.parametrize("bits", [(2, 2), (3, 3), (4, 2)])
def test_plan_build_weighted_equals_oracle(bits):
    """Query-weighted plans: the library averages the query heads' energies
    over each group and runs the greedy on E * W; widths, order and scales
    equal the oracle's (group mean in increasing head order, fp64)."""
    from oracle import energy
    rng = np.random.default_rng(sum(bits))
    bk, bv = bits
    n_kv, G = 2, 4
    q = rng.standard_normal((64, n_kv * G, 128)) * np.exp(rng.standard_normal(128))[None, None]
    Eq, _ = energy.block_energy(q)
    W, _ = energy.query_weights(q, n_kv)
    E = np.exp(1.5 * rng.standard_normal((n_kv, 64)) - np.arange(64) / 8.0)
    cfg = kvq.make_cfg(n_kv, bk, bv, v_seed=3)
    got = kvq.plan_build_weighted(cfg, 1, E, Eq)
    plain = kvq.plan_build(cfg, 1, E)
    for h in range(n_kv):
        ref = alloc.make_plan(E[h], bk, bv, 3, 1, h, weights=W[h])
        assert not ref.near_tie
        assert np.array_equal(got[h]["width"].astype(int), ref.widths)
        assert list(got[h]["order"][:got[h]["n_ranks"]]) == ref.order
        assert np.array_equal(got[h]["g"], ref.g) and np.array_equal(got[h]["a_hat"], ref.a_hat)
        assert np.array_equal(got[h]["g"], plain[h]["g"])
    L = kvq.lib()
    assert L.kvq_plan_build_weighted(ctypes.byref(cfg), 0, E.ctypes.data, Eq.ctypes.data, 7,
                                     got.ctypes.data) == kvq.ERR_ARG
    bad = Eq.copy()
    bad[0, 0] = -1.0
    assert L.kvq_plan_build_weighted(ctypes.byref(cfg), 0, E.ctypes.data, bad.ctypes.data, 8,
                                     got.ctypes.data) == kvq.ERR_ARG
    assert kvq.lib().kvq_energy_workspace_bytes(16) >= 16 * 64 * 16


@pytest.mark.parametrize("bits", [(1, 1), (3, 3), (8, 2)])
def test_plan_build_rotate_keys_equals_oracle(bits):
    """KVQ_ALLOC_ROTATE_KEYS: same widths, order and scales as without it;
    k_rot set and the key signs of the oracle's SplitMix64 positions."""
    from oracle.splitmix import k_signs
    rng = np.random.default_rng(bits[0] * 9 + bits[1])
    E = np.exp(1.5 * rng.standard_normal((2, 64)) - np.arange(64) / 8.0)
    bk, bv = bits
    for mode in (kvq.ALLOC_GREEDY, kvq.ALLOC_UNIFORM):
        cfg0 = kvq.make_cfg(2, bk, bv, v_seed=55, alloc_mode=mode)
        cfg1 = kvq.make_cfg(2, bk, bv, v_seed=55, alloc_mode=mode | kvq.ALLOC_ROTATE_KEYS)
        p0 = kvq.plan_build(cfg0, 4, E)
        p1 = kvq.plan_build(cfg1, 4, E)
        for h in range(2):
            ref = alloc.make_plan(E[h], bk, bv, 55, 4, h, uniform=mode == kvq.ALLOC_UNIFORM,
                                  rotate_keys=True)
            assert p0[h]["k_rot"] == 0 and p1[h]["k_rot"] == 1
            assert np.array_equal(p1[h]["width"], p0[h]["width"])
            assert np.array_equal(p1[h]["g"], p0[h]["g"])
            sg = [-1 if (p1[h]["k_sign"][P >> 5] >> (P & 31)) & 1 else 1 for P in range(128)]
            assert sg == k_signs(55, 4, h) == ref.k_signs.tolist()
    bad = kvq.make_cfg(2, 3, 3, alloc_mode=0x200)
    assert kvq.lib().kvq_plan_build(ctypes.byref(bad), 0, E.ctypes.data, 1,
                                    np.zeros(1, kvq.PLAN_DTYPE).ctypes.data) == kvq.ERR_ARG


def test_sizes():
    cfg = kvq.make_cfg(2, 3, 3)
    assert kvq.tile_bytes(cfg) == 3200 == 32 * 100
    assert kvq.cache_bytes(cfg, 131072) == 4096 * 2 * 3200
    assert kvq.cache_bytes(cfg, 33) == 2 * 2 * 3200
    assert kvq.alloc_workspace_bytes(cfg) >= 2 * 64 * 16
    assert kvq.decode_workspace_bytes(cfg, 1, 16, 131072) > 0
    # decode workspace: sized by batch x n_kv only (records bounded by one
    # wave; per-pair counter/bucket blocks at fixed distances from the end)
    w = kvq.decode_workspace_bytes(cfg, 4, 16, 1 << 10)
    assert w == kvq.decode_workspace_bytes(cfg, 4, 4, 1 << 20)
    assert w == kvq.decode_workspace_bytes(kvq.make_cfg(cfg.n_kv_heads, 1, 8), 4, 8, 77)
    assert kvq.decode_workspace_bytes(cfg, 8, 16, 1 << 10) - w == 4 * cfg.n_kv_heads * 135296
    assert kvq.lib().kvq_plan_bytes() == 1024


def test_window_sizes_and_argument_errors_without_gpu():
    L = kvq.lib()
    cfg = kvq.make_cfg(2, 3, 2)
    assert kvq.window_bytes(cfg, 48) == 2 * 48 * 2 * 128 * 4
    assert kvq.window_bytes(cfg, 0) == 0 and kvq.window_bytes(cfg, -1) == 0
    d = kvq.decode_workspace_bytes(cfg, 3, 8, 1000)
    # the packed tokens' records and up to 32 window record parts
    assert kvq.window_decode_workspace_bytes(cfg, 3, 8, 1000) == d + (33 * 3 * 8 * 528 + 255) // 256 * 256
    p = ctypes.c_void_p(256)
    # negative R, a null length array, a window call without its ring
    assert L.kvq_window_append(ctypes.byref(cfg), p, p, p, 0, 1, p, p, 100, p, p, -1, 1, p,
                               None) == kvq.ERR_ARG
    assert L.kvq_window_append(ctypes.byref(cfg), p, p, p, 0, 1, p, p, 100, p, None, 8, 1, p,
                               None) == kvq.ERR_ARG
    assert L.kvq_window_append(ctypes.byref(cfg), p, p, p, 0, 1, p, p, 100, None, p, 8, 1, p,
                               None) == kvq.ERR_ARG
    assert L.kvq_decode_attn_window(ctypes.byref(cfg), p, p, p, None, p, 8, 1, 100, p, 0, 8, p,
                                    p, 1 << 30, p, None) == kvq.ERR_ARG
    # workspace too small (the records come on top of the decode workspace)
    assert L.kvq_decode_attn_window(ctypes.byref(cfg), p, p, p, p, p, 8, 1, 100, p, 0, 8, p, p,
                                    kvq.decode_workspace_bytes(cfg, 1, 8, 100), p,
                                    None) == kvq.ERR_WORKSPACE
    # the one-launch window step: no RoPE flag, R >= 0, the window decode workspace
    ad = L.kvq_append_decode_window
    wsb = kvq.window_decode_workspace_bytes(cfg, 1, 8, 100)
    assert ad(ctypes.byref(cfg), p, p, p, 0, 1, p, p, 100, p, p, 8, 1, 100, p, 0, 8, p, p, wsb,
              kvq.STEP_ROPE, p, None) == kvq.ERR_ARG
    assert ad(ctypes.byref(cfg), p, p, p, 0, 1, p, p, 100, p, p, -1, 1, 100, p, 0, 8, p, p, wsb,
              0, p, None) == kvq.ERR_ARG
    assert ad(ctypes.byref(cfg), p, p, p, 0, 1, p, p, 100, None, p, 8, 1, 100, p, 0, 8, p, p, wsb,
              0, p, None) == kvq.ERR_ARG
    assert ad(ctypes.byref(cfg), p, p, p, 0, 1, p, p, 100, p, p, 8, 1, 100, p, 0, 8, p, p,
              wsb - 256, 0, p, None) == kvq.ERR_WORKSPACE


def test_argument_errors_without_gpu():
    L = kvq.lib()
    bad = kvq.make_cfg(2, 3, 3, head_dim=64)
    assert L.kvq_plan_build(ctypes.byref(bad), 0, None, 1, None) == kvq.ERR_UNSUPPORTED
    cfg = kvq.make_cfg(2, 9, 3)
    assert L.kvq_plan_build(ctypes.byref(cfg), 0, None, 1, None) == kvq.ERR_ARG
    assert b"bits_k" in L.kvq_last_error()
    cfg = kvq.make_cfg(2, 3, 3)
    assert kvq.tile_bytes(kvq.make_cfg(2, 0, 3)) == 0
    assert L.kvq_decode_attn(ctypes.byref(cfg), None, None, None, 1, 10, None, 0, 16, None, None,
                             0, None, None) == kvq.ERR_ARG
    E = -np.ones((1, 64))
    assert L.kvq_plan_build(ctypes.byref(kvq.make_cfg(1, 2, 2)), 0, E.ctypes.data, 1,
                            np.zeros(1, kvq.PLAN_DTYPE).ctypes.data) == kvq.ERR_ARG
    # n_q not a multiple of n_kv, G > 16, workspace too small: rejected before launch
    p = ctypes.c_void_p(16)
    assert L.kvq_decode_attn(ctypes.byref(cfg), p, p, p, 1, 10, p, 0, 15, p, p, 1 << 30, p,
                             None) == kvq.ERR_ARG
    assert L.kvq_decode_attn(ctypes.byref(cfg), p, p, p, 1, 10, p, 0, 34, p, p, 1 << 30, p,
                             None) == kvq.ERR_ARG
    assert L.kvq_decode_attn(ctypes.byref(cfg), p, p, p, 1, 10, p, 0, 16, p, p, 8, p,
                             None) == kvq.ERR_WORKSPACE
    # a workspace off a 16-byte boundary, and unknown step flags
    p8 = ctypes.c_void_p(24)
    assert L.kvq_decode_attn(ctypes.byref(cfg), p, p, p, 1, 10, p, 0, 16, p, p8, 1 << 30, p,
                             None) == kvq.ERR_ARG
    assert b"aligned" in L.kvq_last_error()
    assert L.kvq_append_decode(ctypes.byref(cfg), p, p, p, 0, 1, p, p, 10, 1, 10, p, 0, 16, p,
                               p8, 1 << 30, 0, 0.0, p, None) == kvq.ERR_ARG
    assert L.kvq_append_decode(ctypes.byref(cfg), p, p, p, 0, 1, p, p, 10, 1, 10, p, 0, 16, p,
                               p, 1 << 30, 4, 0.0, p, None) == kvq.ERR_ARG
    assert b"step_flags" in L.kvq_last_error()
    # RoPE: the base must exceed 1
    assert L.kvq_append_decode(ctypes.byref(cfg), p, p, p, 0, 1, p, p, 10, 1, 10, p, 0, 16, p,
                               p, 1 << 30, kvq.STEP_ROPE, 0.5, p, None) == kvq.ERR_ARG
    assert b"rope_base" in L.kvq_last_error()
    assert L.kvq_quantize_append_rope(ctypes.byref(cfg), p, p, p, 0, 1, 1, p, p, 10, 1.0, p,
                                      None) == kvq.ERR_ARG
    assert L.kvq_quantize_append(ctypes.byref(cfg), p, p, p, 7, 1, 1, p, p, 10, p,
                                 None) == kvq.ERR_ARG
    # context shards: records must be given and 16-byte aligned; n_parts >= 1
    assert L.kvq_decode_attn_partial(ctypes.byref(cfg), p, p, p, 1, 10, p, 0, 16, None, p,
                                     1 << 30, p, None) == kvq.ERR_ARG
    assert L.kvq_decode_attn_partial(ctypes.byref(cfg), p, p, p, 1, 10, p, 0, 16, p8, p,
                                     1 << 30, p, None) == kvq.ERR_ARG
    assert b"aligned" in L.kvq_last_error()
    assert L.kvq_decode_attn_partial(ctypes.byref(cfg), p, p, p, 1, 10, p, 0, 16, p, p, 8, p,
                                     None) == kvq.ERR_WORKSPACE
    assert L.kvq_combine_partials(ctypes.byref(cfg), p, 0, p, 1, 16, p, None) == kvq.ERR_ARG
    assert b"n_parts" in L.kvq_last_error()
    assert L.kvq_combine_partials(ctypes.byref(cfg), p, 2, p8, 1, 16, p, None) == kvq.ERR_ARG
    assert L.kvq_combine_partials(ctypes.byref(cfg), p, 2, p, 1, 15, p, None) == kvq.ERR_ARG
    # paged caches: page_tiles a power of two, pool aligned, capacity < 2^31 tokens
    assert kvq.page_bytes(cfg, 4) == 4 * 2 * kvq.tile_bytes(cfg)
    assert kvq.page_bytes(cfg, 3) == 0 and kvq.page_bytes(cfg, 0) == 0
    pg = kvq.Pages(16, 16, 10, 3, 8)
    assert L.kvq_paged_decode_attn(ctypes.byref(cfg), p, ctypes.byref(pg), p, 1, 10, p, 0, 16, p,
                                   p, 1 << 30, p, None) == kvq.ERR_ARG
    assert b"page_tiles" in L.kvq_last_error()
    pg = kvq.Pages(24, 16, 10, 4, 8)
    assert L.kvq_paged_quantize_append(ctypes.byref(cfg), p, p, p, 0, 1, 1, ctypes.byref(pg), p,
                                       0.0, p, None) == kvq.ERR_ARG
    assert b"aligned" in L.kvq_last_error()
    pg = kvq.Pages(16, 16, 10, 1 << 20, 1 << 10)
    assert L.kvq_paged_append_decode(ctypes.byref(cfg), p, p, p, 0, 1, ctypes.byref(pg), p, 1,
                                     10, p, 0, 16, p, p, 1 << 30, 0, 0.0, p, None) == kvq.ERR_ARG
    assert b"capacity" in L.kvq_last_error()
    pg = kvq.Pages(16, None, 10, 4, 8)
    assert L.kvq_paged_decode_attn(ctypes.byref(cfg), p, ctypes.byref(pg), p, 1, 10, p, 0, 16, p,
                                   p, 1 << 30, p, None) == kvq.ERR_ARG
    pg = kvq.Pages(16, 16, 10, 4, 8)
    assert L.kvq_paged_quantize_append(ctypes.byref(cfg), p, p, p, 0, 1, 1, ctypes.byref(pg), p,
                                       0.5, p, None) == kvq.ERR_ARG
    assert b"rope_base" in L.kvq_last_error()
    assert L.kvq_paged_decode_attn_partial(ctypes.byref(cfg), p, ctypes.byref(pg), p, 1, 10, p,
                                           0, 16, None, p, 1 << 30, p, None) == kvq.ERR_ARG
    assert L.kvq_paged_decode_attn_partial(ctypes.byref(cfg), p, ctypes.byref(pg), p, 1, 10, p,
                                           0, 16, p, p, 8, p, None) == kvq.ERR_WORKSPACE
    # zero new tokens is a no-op
    assert L.kvq_quantize_append(ctypes.byref(cfg), p, None, None, 0, 1, 0, p, p, 10, p,
                                 None) == kvq.OK


@pytest.mark.parametrize("kind", ["zero", "one_block", "tiny"])
def test_plan_build_degenerate_energies(kind):
    """Degenerate energy vectors (all zero, one nonzero block, denormal-small)
    give the oracle's plans: widths by the tie rule, zero scales where the
    energy is zero."""
    E = np.zeros((1, 64))
    if kind == "one_block":
        E[0, 17] = 3.0
    elif kind == "tiny":
        E[0] = np.ldexp(1.0, -1060) * (1 + np.arange(64))
    for bits in (1, 3, 8):
        cfg = kvq.make_cfg(1, bits, 2, v_seed=4)
        got = kvq.plan_build(cfg, 0, E)[0]
        ref = alloc.make_plan(E[0], bits, 2, 4, 0, 0)
        assert np.array_equal(got["width"].astype(int), ref.widths)
        assert np.array_equal(got["g"], ref.g) and np.array_equal(got["a_hat"], ref.a_hat)
        assert int(got["width"].sum()) == 64 * bits


def test_plan_check_accepts_built_plans_and_refuses_inconsistent_ones():
    rng = np.random.default_rng(31)
    E = np.exp(1.5 * rng.standard_normal((2, 64)) - np.arange(64) / 8.0)
    for mode in (kvq.ALLOC_GREEDY, kvq.ALLOC_UNIFORM, kvq.ALLOC_GREEDY | kvq.ALLOC_ROTATE_KEYS):
        for bits in ((1, 1), (3, 3), (8, 2)):
            cfg = kvq.make_cfg(2, *bits, v_seed=1, alloc_mode=mode)
            kvq.plan_check(cfg, kvq.plan_build(cfg, 0, E))
    cfg = kvq.make_cfg(2, 3, 3, v_seed=1)
    good = kvq.plan_build(cfg, 0, E)

    def refused(mutate, what):
        p = good.copy()
        mutate(p)
        with pytest.raises(kvq.KVQError) as ei:
            kvq.plan_check(cfg, p)
        assert what in str(ei.value)

    def bad_magic(p):
        p["magic"] = 0

    def wide_block(p):
        p["width"][0, 0] = 9

    refused(bad_magic, "magic")
    refused(wide_block, "width")
    j0, j1 = int(good["order"][0][0]), int(good["order"][0][1])

    def swap_order(p):
        p["order"][0][0], p["order"][0][1] = j1, j0
    if good["width"][0][j0] != good["width"][0][j1]:
        refused(swap_order, "inconsistent")

    def move_bit(p):  # one bit moved between blocks: widths still sum right
        w = p["width"][0]
        a = int(np.argmax(w))
        b = int(np.argmin(np.where(w < 8, w, 99)))
        w[a] -= 1
        w[b] += 1
    refused(move_bit, "inconsistent")
    def shift_segment(p):
        p["seg_off"][0, 3] += 1

    def bad_rot(p):
        p["k_rot"] = 2

    def nan_scale(p):
        p["g"][0, 5] = np.float32(np.nan)

    refused(shift_segment, "inconsistent")
    refused(bad_rot, "k_rot")
    refused(nan_scale, "scales")
    other = kvq.make_cfg(2, 2, 3, v_seed=1)
    with pytest.raises(kvq.KVQError):
        kvq.plan_check(other, good)
