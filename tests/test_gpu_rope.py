"""Fused RoPE + quantize-append (pre-RoPE keys in, post-RoPE codes in the
cache) against the oracle's fp32 RoPE recipe followed by the usual
quantization (GPU): packed words and norms bit-exact, decode output within
the decode tolerance."""
import numpy as np
import pytest
import torch

import oracle_pipeline as op
import synth
from bit_kv_cache_19_b200 import kvq
from bit_kv_cache_19_b200.runtime import PackedLayer
from oracle import alloc, attn, layout, quant, rope

pytestmark = pytest.mark.gpu
TOL = 2e-3


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _oracle_heads(kpre_heads, v_heads, pos0, base, E, bk, bv, v_seed, layer):
    """Oracle records of pre-RoPE keys rotated (fp32 recipe) to positions pos0.."""
    heads = []
    for h, (kp, v) in enumerate(zip(kpre_heads, v_heads)):
        T = kp.shape[0]
        k = rope.rotate_f32(kp, pos0 + np.arange(T), base).astype(np.float64)
        plan = alloc.make_plan(E[h], bk, bv, v_seed, layer, h)
        kc, kn, _ = quant.quantize_keys(k, plan)
        vc, vn, _ = quant.quantize_values(v, plan)
        heads.append(dict(plan=plan, rec=layout.pack(kc, vc, kn, vn, plan, T),
                          khat=attn.dequant_keys(kc, kn, plan), vhat=attn.dequant_values(vc, vn, plan)))
    return heads


def _check(got, ref, T, bk, bv):
    """Code words equal (positions past T are zero on both sides); norms of
    the T tokens equal."""
    nw = 128 * (bk + bv)
    assert np.array_equal(got[:, :nw], ref[:, :nw]), "packed code words differ"
    gn = got[:, nw:].view(np.uint16).reshape(-1, 2, 32)
    rn = ref[:, nw:].view(np.uint16).reshape(-1, 2, 32)
    valid = np.arange(gn.shape[0] * 32).reshape(-1, 32) < T
    for part in range(2):
        assert np.array_equal(gn[:, part][valid], rn[:, part][valid]), "norms differ"


@pytest.mark.parametrize("wname,bits", [("qwen3b_128k", (3, 3)), ("llama8b", (2, 2)),
                                        ("qwen3b_128k", (5, 1))])
def test_quantize_append_rope_matches_oracle(wname, bits):
    wl = synth.WORKLOADS[wname]
    bk, bv = bits
    n_kv = 2
    starts, total = [0, 45, 1000], 300
    cap = max(starts) + total + 32
    cfg = kvq.make_cfg(n_kv, bk, bv, v_seed=3)
    L = PackedLayer(cfg, len(starts), cap, layer=2)
    kpre, vv = [], []
    for s, T0 in enumerate(starts):
        ks = [synth.keys_pre_rope(wl, 40 + s, 2, h, T0 + total) for h in range(n_kv)]
        vs = [synth.keys_values(wl, 40 + s, 2, h, T0 + total)[1] for h in range(n_kv)]
        kpre.append(np.stack(ks, axis=1))
        vv.append(np.stack(vs, axis=1))
    E, _ = op.energies([synth.bf16_bits_to_f64(kpre[0][:, h]) for h in range(n_kv)])
    L.set_plans(kvq.plan_build(cfg, 2, E))
    for s, T0 in enumerate(starts):  # older tokens, then the appended block
        if T0:
            kvq.quantize_append_rope(cfg, L.plan_ptrs[s:s + 1], _dev(kpre[s][:T0])[None],
                                     _dev(vv[s][:T0])[None], L.cache_ptrs[s:s + 1],
                                     L.lens[s:s + 1], cap, wl.rope_base, L.status)
    k = torch.stack([_dev(kpre[s][T0:T0 + total]) for s, T0 in enumerate(starts)])
    v = torch.stack([_dev(vv[s][T0:T0 + total]) for s, T0 in enumerate(starts)])
    L.append_rope(k, v, wl.rope_base)
    torch.cuda.synchronize()
    assert L.flags() == 0
    for s, T0 in enumerate(starts):
        T = T0 + total
        heads = _oracle_heads([synth.bf16_bits_to_f64(kpre[s][:T, h]) for h in range(n_kv)],
                              [synth.bf16_bits_to_f64(vv[s][:T, h]) for h in range(n_kv)],
                              0, wl.rope_base, E, bk, bv, 3, 2)
        for h in range(n_kv):
            _check(L.head_records(s, h, (T + 31) // 32), heads[h]["rec"], T, bk, bv)


@pytest.mark.parametrize("n_new,flags", [(1, kvq.STEP_ROPE), (7, kvq.STEP_ROPE | kvq.STEP_EARLY)])
def test_fused_step_with_pre_rope_keys(n_new, flags):
    wl = synth.WORKLOADS["qwen3b_128k"]
    n_kv, G, bk, bv = 2, 8, 3, 3
    starts = [300, 31]
    cap = 512
    cfg = kvq.make_cfg(n_kv, bk, bv, v_seed=9)
    L = PackedLayer(cfg, len(starts), cap, layer=1)
    kpre = [np.stack([synth.keys_pre_rope(wl, 60 + s, 1, h, T0 + n_new) for h in range(n_kv)], 1)
            for s, T0 in enumerate(starts)]
    vv = [np.stack([synth.keys_values(wl, 60 + s, 1, h, T0 + n_new)[1] for h in range(n_kv)], 1)
          for s, T0 in enumerate(starts)]
    E, _ = op.energies([synth.bf16_bits_to_f64(kpre[0][:, h]) for h in range(n_kv)])
    L.set_plans(kvq.plan_build(cfg, 1, E))
    for s, T0 in enumerate(starts):
        kvq.quantize_append_rope(cfg, L.plan_ptrs[s:s + 1], _dev(kpre[s][:T0])[None],
                                 _dev(vv[s][:T0])[None], L.cache_ptrs[s:s + 1], L.lens[s:s + 1],
                                 cap, wl.rope_base, L.status)
    knew = torch.stack([_dev(kpre[s][T0:T0 + n_new]) for s, T0 in enumerate(starts)])
    vnew = torch.stack([_dev(vv[s][T0:T0 + n_new]) for s, T0 in enumerate(starts)])
    qb = np.stack([synth.queries(wl, 60 + s, 1, 0, starts[s] + n_new) for s in range(len(starts))])
    out = L.append_decode(knew, vnew, _dev(qb), ws=L.workspace(n_kv * G, cap),
                          step_flags=flags, rope_base=wl.rope_base).cpu().numpy()
    torch.cuda.synchronize()
    assert L.flags() == 0
    assert L.lens.cpu().tolist() == [T0 + n_new for T0 in starts]
    for s, T0 in enumerate(starts):
        T = T0 + n_new
        heads = _oracle_heads([synth.bf16_bits_to_f64(kpre[s][:T, h]) for h in range(n_kv)],
                              [synth.bf16_bits_to_f64(vv[s][:T, h]) for h in range(n_kv)],
                              0, wl.rope_base, E, bk, bv, 9, 1)
        for h in range(n_kv):
            _check(L.head_records(s, h, (T + 31) // 32), heads[h]["rec"], T, bk, bv)
        assert op.rel_err(out[s], op.decode(synth.bf16_bits_to_f64(qb[s]), heads)) <= TOL
