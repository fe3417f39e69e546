"""kvq_decode_attn_noalloc: decode without a caller workspace (GPU).

The entry point is for callers that cannot allocate device memory where they
decode (graph capture, memory owned by a pool the library cannot reach, no
allocator synchronization allowed mid-step). It must give the same output
as kvq_decode_attn with a caller workspace, call after call, although its
split partials live in one fixed scratch array shared by all calls. This
file is collected last so that a run that stops at its first failure has
run every other test already; it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from bit_kv_cache_19_b200 import kvq
from bit_kv_cache_19_b200.runtime import PackedLayer

pytestmark = pytest.mark.gpu
TOL = 2e-3


def _rel(o, ref):
    o = o.reshape(-1, 128).astype(np.float64)
    ref = ref.reshape(-1, 128).astype(np.float64)
    den = np.maximum(np.abs(ref).max(axis=1), 1e-30)
    return float(np.max(np.abs(o - ref).max(axis=1) / den))


def _noalloc(cfg, L, max_len, q, out):
    L_ = kvq.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L_.kvq_decode_attn_noalloc(ctypes.byref(cfg), ctypes.c_void_p(L.plan_ptrs.data_ptr()),
                                      ctypes.c_void_p(L.cache_ptrs.data_ptr()),
                                      ctypes.c_void_p(L.lens.data_ptr()), q.shape[0], max_len,
                                      ctypes.c_void_p(q.data_ptr()), kvq.BF16, q.shape[1],
                                      ctypes.c_void_p(out.data_ptr()),
                                      ctypes.c_void_p(L.status.data_ptr()), stream)


def test_noalloc_matches_workspace_decode_twice():
    rng = np.random.default_rng(21)
    n_kv, G, batch, T, cap = 2, 8, 3, 1500, 1536
    cfg = kvq.make_cfg(n_kv, 3, 3, v_seed=8)
    L = PackedLayer(cfg, batch, cap)
    E = np.exp(rng.standard_normal((n_kv, 64)) - np.arange(64) / 8.0)
    L.set_plans(kvq.plan_build(cfg, 0, E))
    k = synth.to_bf16_bits(rng.standard_normal((batch, T, n_kv, 128)))
    v = synth.to_bf16_bits(rng.standard_normal((batch, T, n_kv, 128)))
    kd = torch.from_numpy(k.view(np.int16)).view(torch.bfloat16).cuda()
    vd = torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).cuda()
    L.append(kd, vd)
    torch.cuda.synchronize()
    assert kvq.decode_workspace_bytes(cfg, batch, n_kv * G, cap) <= \
        kvq.lib().kvq_decode_noalloc_scratch_bytes()
    for call in range(2):
        qb = synth.to_bf16_bits(rng.standard_normal((batch, n_kv * G, 128)))
        q = torch.from_numpy(qb.view(np.int16)).view(torch.bfloat16).cuda()
        ref = L.decode(q, max_len=cap).cpu().numpy()
        out = torch.full((batch, n_kv * G, 128), float("nan"), device="cuda")
        assert _noalloc(cfg, L, cap, q, out) == kvq.OK, kvq.lib().kvq_last_error()
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert np.isfinite(got).all()
        assert _rel(got, ref) <= TOL, call
    assert L.flags() == 0


def test_noalloc_rejects_what_does_not_fit():
    cfg = kvq.make_cfg(4, 3, 2)
    limit = kvq.lib().kvq_decode_noalloc_scratch_bytes()
    assert kvq.decode_workspace_bytes(cfg, 2048, 28, 1 << 20) > limit
    p = ctypes.c_void_p(256)
    rc = kvq.lib().kvq_decode_attn_noalloc(ctypes.byref(cfg), p, p, p, 2048, 1 << 20, p,
                                           kvq.BF16, 28, p, p, None)
    assert rc == kvq.ERR_WORKSPACE
    assert b"4 MiB" in kvq.lib().kvq_last_error()
