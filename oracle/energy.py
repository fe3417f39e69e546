"""Label-free RoPE block energy (oracle; test infrastructure only).

"RoPE-Aware Bit Allocation for KV-Cache Quantization", abstract: for each layer
and KV head Block-GTQ computes a label-free energy score for each RoPE block.
The formula is not printed. Reading adopted: the key-only second moment of
the block over the allocation window (no queries, labels or gradients),

    E_j = (1/T) sum_t (k_{t,j}^2 + k_{t,j+64}^2).

It is RoPE-invariant (a rotation keeps each block's squared length). To make
it order-independent, each squared coordinate is taken on a fixed-point grid
of 2^-32 before summation:

    S_j = sum_t sum_{i in block j} min(floor(k_{t,i}^2 * 2^32), 2^64 - 1)

an exact integer (any summation order gives the same S_j), and
E_j = fp64(S_j) * 2^-32 / T. Non-finite coordinates contribute 0 and raise
the NONFINITE flag.
"""
import numpy as np

FLAG_NONFINITE = 2
_TWO32 = float(2 ** 32)
_TWO64 = float(2 ** 64)


def square_terms(k) -> tuple:
    """floor(k^2 * 2^32) per coordinate as uint64, saturating; and a flag."""
    k = np.asarray(k, dtype=np.float64)
    fin = np.isfinite(k)
    f = np.where(fin, k, 0.0)
    f = f * f * _TWO32                     # exact: inputs have <= 24-bit significands
    sat = f >= _TWO64
    t = np.floor(np.where(sat, 0.0, f)).astype(np.uint64)
    t = np.where(sat, np.uint64(2 ** 64 - 1), t)
    flags = 0 if fin.all() else FLAG_NONFINITE
    return t, flags


def block_energy_int(k):
    """Exact integer block sums S[h][j] for keys ``k[T, H, 128]``.

    Returns (list of lists of Python ints, flags).
    """
    k = np.asarray(k, dtype=np.float64)
    T, H, d = k.shape
    half = d // 2
    t, flags = square_terms(k)
    lo = (t & np.uint64(0xFFFFFFFF)).sum(axis=0, dtype=np.uint64)    # [H, d]
    hi = (t >> np.uint64(32)).sum(axis=0, dtype=np.uint64)
    out = []
    for h in range(H):
        row = []
        for j in range(half):
            s = 0
            for i in (j, j + half):
                s += (int(hi[h, i]) << 32) + int(lo[h, i])
            row.append(s)
        out.append(row)
    return out, flags


def block_energy(k):
    """E[h][j] (fp64) and flags for keys ``k[T, H, 128]``."""
    k = np.asarray(k, dtype=np.float64)
    T = k.shape[0]
    S, flags = block_energy_int(k)
    E = np.array([[float(s) / _TWO32 / T for s in row] for row in S], dtype=np.float64)
    return E, flags


def query_weights(q, n_kv: int):
    """Query block energies averaged over each KV head's query group.

    Variant of the allocation (not the pages' label-free score): the logit
    q . k decomposes into 2-D RoPE block terms q_j . k_j, so a quantization
    error in block j reaches the logit scaled by the query's block-j energy.
    For calibration queries ``q[T, Hq, 128]`` (post-RoPE; the energy is
    RoPE-invariant) this returns Q[h][j] = (1/G) sum_{g < G} E^q_{hG+g, j}
    (sum over g in increasing order, fp64), E^q the same exact block energy
    as for keys, G = Hq / n_kv."""
    Eq, flags = block_energy(q)
    Hq = Eq.shape[0]
    G = Hq // n_kv
    Q = np.zeros((n_kv, Eq.shape[1]))
    for h in range(n_kv):
        acc = np.zeros(Eq.shape[1])
        for g in range(G):
            acc = acc + Eq[h * G + g]
        Q[h] = acc / G
    return Q, flags
