"""kvq_decode_attn_noalloc: decode without a caller workspace (GPU).

The entry point is for callers that cannot allocate device memory where they
decode (graph capture, memory owned by a pool the library cannot reach, no
allocator synchronization allowed mid-step). Its split partials live in one
fixed scratch array shared by every call, so the tests check it call after
call, and across calls of different shapes, against the fp64 oracle and
against kvq_decode_attn with a fresh workspace. This file is collected last
so that a run that stops at its first failure has run every other test
already; it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle_pipeline as op
import synth
from bit_kv_cache_19_b200 import kvq
from bit_kv_cache_19_b200.runtime import PackedLayer

pytestmark = pytest.mark.gpu
TOL = 2e-3
V_SEED = 8


def _noalloc(cfg, L, max_len, q, out):
    L_ = kvq.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L_.kvq_decode_attn_noalloc(ctypes.byref(cfg), ctypes.c_void_p(L.plan_ptrs.data_ptr()),
                                      ctypes.c_void_p(L.cache_ptrs.data_ptr()),
                                      ctypes.c_void_p(L.lens.data_ptr()), q.shape[0], max_len,
                                      ctypes.c_void_p(q.data_ptr()), kvq.BF16, q.shape[1],
                                      ctypes.c_void_p(out.data_ptr()),
                                      ctypes.c_void_p(L.status.data_ptr()), stream)


def _bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


class _Case:
    """A filled layer (batch sequences of T tokens) and its oracle heads."""

    def __init__(self, seed, n_kv, batch, T, cap):
        rng = np.random.default_rng(seed)
        self.cfg = kvq.make_cfg(n_kv, 3, 3, v_seed=V_SEED)
        self.cap = cap
        self.L = PackedLayer(self.cfg, batch, cap)
        E = np.exp(rng.standard_normal((n_kv, 64)) - np.arange(64) / 8.0)
        self.L.set_plans(kvq.plan_build(self.cfg, 0, E))
        k = synth.to_bf16_bits(rng.standard_normal((batch, T, n_kv, 128)))
        v = synth.to_bf16_bits(rng.standard_normal((batch, T, n_kv, 128)))
        self.L.append(_bf16_dev(k), _bf16_dev(v))
        self.heads = []
        for b in range(batch):
            kh, vh = op.bf16_heads(k[b], v[b])
            _, hs = op.layer(kh, vh, 3, 3, V_SEED, 0, E=E, pack=False)
            self.heads.append(hs)
        self.rng = rng
        torch.cuda.synchronize()

    def query(self, G):
        batch, n_kv = len(self.heads), len(self.heads[0])
        qb = synth.to_bf16_bits(self.rng.standard_normal((batch, n_kv * G, 128)))
        return qb, _bf16_dev(qb)

    def oracle(self, qb):
        q = synth.bf16_bits_to_f64(qb)
        return np.stack([op.decode(q[b], self.heads[b]) for b in range(len(self.heads))])

    def noalloc(self, q):
        out = torch.full(q.shape, float("nan"), device="cuda")
        assert _noalloc(self.cfg, self.L, self.cap, q, out) == kvq.OK, kvq.lib().kvq_last_error()
        torch.cuda.synchronize()
        return out.cpu().numpy()

    def with_workspace(self, q):
        # kvq_decode_attn with a fresh zero-filled workspace
        return self.L.decode(q, max_len=self.cap).cpu().numpy()


def _check(case, G):
    qb, q = case.query(G)
    got = case.noalloc(q)
    assert np.isfinite(got).all()
    assert op.rel_err(got, case.oracle(qb)) <= TOL
    assert op.rel_err(got, case.with_workspace(q)) <= TOL
    assert case.L.flags() == 0


def test_noalloc_matches_oracle_twice():
    case = _Case(21, n_kv=2, batch=3, T=1500, cap=1536)
    limit = kvq.lib().kvq_decode_noalloc_scratch_bytes()
    assert kvq.decode_workspace_bytes(case.cfg, 3, 16, 1536) <= limit
    for _ in range(2):
        _check(case, G=8)


def test_noalloc_alternating_shapes():
    # shapes ordered on one stream through the same scratch: the second has
    # fewer sequences, a shorter context and a smaller query group, so its
    # counter and bucket blocks lie where the first call's split records
    # could sit if the layout depended on the shape
    big = _Case(22, n_kv=2, batch=3, T=1500, cap=1536)
    small = _Case(23, n_kv=2, batch=1, T=500, cap=512)
    _check(big, G=8)
    _check(small, G=4)
    _check(big, G=8)
    _check(small, G=8)
    _check(big, G=2)


def test_noalloc_rejects_what_does_not_fit():
    cfg = kvq.make_cfg(4, 3, 2)
    limit = kvq.lib().kvq_decode_noalloc_scratch_bytes()
    assert kvq.decode_workspace_bytes(cfg, 2048, 28, 1 << 20) > limit
    p = ctypes.c_void_p(256)
    rc = kvq.lib().kvq_decode_attn_noalloc(ctypes.byref(cfg), p, p, p, 2048, 1 << 20, p,
                                           kvq.BF16, 28, p, p, None)
    assert rc == kvq.ERR_WORKSPACE
    assert b"16 MiB" in kvq.lib().kvq_last_error()
