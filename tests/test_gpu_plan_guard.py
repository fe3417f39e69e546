"""Plan records whose magic and shape are valid but whose order, K segments
or decode schedule do not follow from the widths are flagged on the device
(BAD_PLAN): kvq_quantize_append stores nothing with them, and
kvq_decode_attn and kvq_append_decode flag their output (the fused append
keeps its writes inside the token's tile record). The corruptions are
ones the host check (kvq_plan_check) also refuses, and each keeps every index
the kernels would derive from it inside the tile record (so the test is safe
even against a kernel that failed to refuse it)."""
import numpy as np
import pytest
import torch

import synth
from bit_kv_cache_19_b200 import kvq
from bit_kv_cache_19_b200.runtime import PackedLayer


def _plan(seed):
    cfg = kvq.make_cfg(1, 3, 3, v_seed=4)
    rng = np.random.default_rng(seed)
    E = np.exp(1.5 * rng.standard_normal((1, 64)) - np.arange(64) / 8.0)
    return cfg, kvq.plan_build(cfg, 0, E)


def _corruptions(plan):
    p = plan[0]
    nr = int(p["n_ranks"])
    w_of = lambda r: int(p["width"][p["order"][r]])  # noqa: E731
    out = {}
    # two ranks of different widths swapped in the order
    r = next(r for r in range(nr - 1) if w_of(r) != w_of(r + 1))
    x = plan.copy()
    x[0]["order"][[r, r + 1]] = x[0]["order"][[r + 1, r]]
    out["order_swap"] = x
    # a K segment moved by one word
    x = plan.copy()
    x[0]["seg_off"][nr // 2] += 1
    out["seg_off"] = x
    # one width raised and another lowered (same bit budget, order stale)
    lo = next(j for j in range(64) if 1 <= p["width"][j] <= 7)
    hi = next(j for j in range(63, -1, -1) if p["width"][j] >= 2 and j != lo)
    x = plan.copy()
    x[0]["width"][lo] += 1
    x[0]["width"][hi] -= 1
    out["widths"] = x
    # a half step one rank short
    hs = next(h for h in range(int(p["n_half"])) if p["hs_count"][h] >= 2)
    x = plan.copy()
    x[0]["hs_count"][hs] -= 1
    out["hs_count"] = x
    # one half step fewer
    x = plan.copy()
    x[0]["n_half"] -= 1
    out["n_half"] = x
    # a class given another valid width
    x = plan.copy()
    x[0]["cls_w"][0] = x[0]["cls_w"][0] - 1 if x[0]["cls_w"][0] > 1 else 2
    out["cls_w"] = x
    # a class's first K word moved
    x = plan.copy()
    x[0]["cls_seg0"][1] += 2
    out["cls_seg0"] = x
    return out


def test_host_check_refuses_every_corruption():
    cfg, plan = _plan(1)
    kvq.plan_check(cfg, plan)
    for name, bad in _corruptions(plan).items():
        with pytest.raises(kvq.KVQError):
            kvq.plan_check(cfg, bad)
        assert bad[0]["magic"] == plan[0]["magic"], name


@pytest.mark.gpu
def test_device_refuses_inconsistent_plans():
    cfg, plan = _plan(1)
    rng = np.random.default_rng(2)
    T = 100
    kb = synth.to_bf16_bits(rng.standard_normal((1, T, 1, 128)))
    vb = synth.to_bf16_bits(rng.standard_normal((1, T, 1, 128)))
    k = torch.from_numpy(kb.view(np.int16)).view(torch.bfloat16).cuda()
    v = torch.from_numpy(vb.view(np.int16)).view(torch.bfloat16).cuda()
    q = torch.from_numpy(synth.to_bf16_bits(rng.standard_normal((1, 8, 128))).view(np.int16))
    q = q.view(torch.bfloat16).cuda()
    # the valid plan is accepted by both kernels
    L = PackedLayer(cfg, 1, 128)
    L.set_plans(plan)
    L.append(k, v)
    out = L.decode(q)
    torch.cuda.synchronize()
    assert L.flags() == 0 and torch.isfinite(out).all()
    ws = L.workspace(8, 128)
    for name, bad in _corruptions(plan).items():
        # quantize: nothing stored
        M = PackedLayer(cfg, 1, 128)
        M.set_plans(bad, check=False)  # the device check is under test
        before = M.caches[0].clone()
        M.append(k, v)
        torch.cuda.synchronize()
        assert M.flags() & kvq.FLAG_BAD_PLAN, name
        assert torch.equal(before, M.caches[0]), name
        # decode over a cache written with the valid plan: output flagged
        L.set_plans(bad, check=False)
        L.status.zero_()
        L.decode(q, ws=ws)
        torch.cuda.synchronize()
        assert L.flags() & kvq.FLAG_BAD_PLAN, name
        # fused append + decode: flagged; the append writes only inside the
        # record of the token's tile (tile 3 of 4 here)
        n0 = int(L.lens.item())
        rec = L.caches[0].clone()
        L.status.zero_()
        L.append_decode(k[:, :1].contiguous(), v[:, :1].contiguous(), q, ws=ws)
        torch.cuda.synchronize()
        assert L.flags() & kvq.FLAG_BAD_PLAN, name
        tb = kvq.tile_bytes(cfg)
        assert torch.equal(rec[:3 * tb], L.caches[0][:3 * tb]), name
        L.caches[0].copy_(rec)
        L.lens.fill_(n0)
    # the workspace is still usable with the valid plan
    L.set_plans(plan)
    L.status.zero_()
    ref = L.decode(q)
    out = L.decode(q, ws=ws)
    torch.cuda.synchronize()
    assert L.flags() == 0
    assert torch.allclose(out, ref, rtol=1e-5, atol=1e-6)
