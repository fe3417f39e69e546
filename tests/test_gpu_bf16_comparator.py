"""bf16 comparator kernel (dense split-K decode over an unquantized cache,
not part of the method) against the oracle's exact attention on the same
bf16 values (GPU).

Tolerance: the kernel feeds P = 2^(s - m) to the tensor cores in bf16 (8
significant bits, relative rounding <= 2^-9) while l sums the fp32 values,
so an output can move by up to ~2^-9 of max |v| when one token dominates;
4e-3 of max |o| per head bounds that with margin.
"""
import numpy as np
import pytest
import torch

import synth
from bit_kv_cache_19_b200 import kvq
from oracle import attn

pytestmark = pytest.mark.gpu
TOL = 4e-3


def _bf16(a):
    return torch.from_numpy(synth.to_bf16_bits(a).view(np.int16)).view(torch.bfloat16).cuda()


def _rel(o, ref):
    o = o.reshape(-1, 128).astype(np.float64)
    ref = ref.reshape(-1, 128).astype(np.float64)
    den = np.maximum(np.abs(ref).max(axis=1), 1e-30)
    return float(np.max(np.abs(o - ref).max(axis=1) / den))


@pytest.mark.parametrize("n_kv,G,lens,cap", [
    (2, 8, [1000, 37, 1030], 1030),   # ragged tails, a tile cut by the capacity
    (8, 4, [4096, 1], 4100),          # llama-shaped group, one-token sequence
    (1, 16, [777], 800),              # 16 query heads per KV head (two n-tiles)
    (2, 8, [0, 64], 64),              # an empty sequence gives zeros
])
def test_bf16_comparator_matches_exact_attention(n_kv, G, lens, cap):
    rng = np.random.default_rng(7 + n_kv * 100 + G + len(lens))
    B = len(lens)
    scale = np.exp(rng.standard_normal((n_kv, 1, 128)) * 0.5)
    kf = rng.standard_normal((B, n_kv, cap, 128)) * scale
    vf = rng.standard_normal((B, n_kv, cap, 128))
    qf = rng.standard_normal((B, n_kv * G, 128)) * 2.0
    k, v, q = _bf16(kf), _bf16(vf), _bf16(qf)
    kb = synth.bf16_bits_to_f64(synth.to_bf16_bits(kf))
    vb = synth.bf16_bits_to_f64(synth.to_bf16_bits(vf))
    qb = synth.bf16_bits_to_f64(synth.to_bf16_bits(qf))
    lens_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
    max_len = max(cap, 1)
    ws = torch.zeros(kvq.bf16_decode_workspace_bytes(B, n_kv, n_kv * G, max_len),
                     dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):  # the counters return to zero: a second call on the same workspace
        out = torch.full((B, n_kv * G, 128), float("nan"), device="cuda")
        kvq.bf16_decode_attn(k, v, lens_d, max_len, q, out, ws, status)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert np.isfinite(got).all(), call
        for b in range(B):
            ref = np.zeros((n_kv * G, 128))
            for h in range(n_kv):
                T = lens[b]
                ref[h * G:(h + 1) * G] = attn.attention(qb[b, h * G:(h + 1) * G], kb[b, h, :T],
                                                        vb[b, h, :T])
            if lens[b] == 0:
                assert np.all(got[b] == 0.0)
            else:
                assert _rel(got[b], ref) <= TOL, (call, b)
    assert int(status.item()) == 0
