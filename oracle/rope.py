"""RoPE on 2-D frequency blocks (oracle; test infrastructure only).

"RoPE-Aware Bit Allocation for KV-Cache Quantization", abstract: under RoPE a
key's contribution to a future attention logit decomposes into a
position-dependent sum over two-dimensional frequency blocks. With head size
d = 128 the blocks are the coordinate pairs (j, j + 64), j = 0..63 (half-split
pairing), rotated by the angle pos * theta_j with theta_j = base^(-2j/d):

    (x_j, x_{j+64}) -> (x_j cos a - x_{j+64} sin a,  x_j sin a + x_{j+64} cos a)

so that  RoPE(q, m) . RoPE(k, n) = sum_j q_j^T R(theta_j (n - m)) k_j,
with q_j = (q_j, q_{j+64}). All arithmetic fp64, except rotate_f32, the
recipe of the fused rotate-and-quantize path (pre-RoPE keys in, codes of the
rotated keys out; a reading of ours, the pages give no RoPE arithmetic): the
angles pos * theta_j in fp64, their cos and sin rounded once to fp32, then
the 2-D rotation in fp32 with every product and sum rounded (no fused
multiply-add), so the codes decided on the rotated values are exact on both
sides.
"""
import numpy as np


def thetas(base: float, d: int = 128) -> np.ndarray:
    """theta_j = base^(-2j/d) for j = 0..d/2-1 (theta_0 = 1 is the fastest)."""
    j = np.arange(d // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * j / d)


def rotate(x, pos, base: float):
    """Apply RoPE at position(s) ``pos`` to ``x[..., d]`` (fp64)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    h = d // 2
    ang = np.asarray(pos, dtype=np.float64)[..., None] * thetas(base, d)
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., :h], x[..., h:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def block_terms(q, k, m, n, base: float) -> np.ndarray:
    """Per-block logit terms q_j^T R(theta_j (n - m)) k_j of pre-RoPE q, k.

    Their sum is the RoPE logit RoPE(q, m) . RoPE(k, n).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    h = q.shape[-1] // 2
    ang = (float(n) - float(m)) * thetas(base, 2 * h)
    c, s = np.cos(ang), np.sin(ang)
    k0 = k[:h] * c - k[h:] * s
    k1 = k[:h] * s + k[h:] * c
    return q[:h] * k0 + q[h:] * k1


def rotate_f32(x, pos, base: float) -> np.ndarray:
    """RoPE as the fused quantize path computes it (float32 result).

    c = fp32(cos(pos theta_j)), s = fp32(sin(pos theta_j)) from fp64 angles;
    a' = fp32(fp32(a c) - fp32(b s)), b' = fp32(fp32(a s) + fp32(b c)).
    """
    x32 = np.asarray(x, dtype=np.float32)
    d = x32.shape[-1]
    h = d // 2
    ang = np.asarray(pos, dtype=np.float64)[..., None] * thetas(base, d)
    c = np.cos(ang).astype(np.float32)
    s = np.sin(ang).astype(np.float32)
    a, b = x32[..., :h], x32[..., h:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1).astype(np.float32)
