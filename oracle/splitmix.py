"""SplitMix64 counter generator for the value sign flips (oracle).

Test infrastructure only. SplitMix64 (Steele, Lea and Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014; public reference code by
S. Vigna): the n-th output (n = 0, 1, ...) of the stream with seed s is
mix(s + (n + 1) * GAMMA) mod 2^64, with GAMMA = 0x9E3779B97F4A7C15 and

    mix(z): z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9
            z = (z ^ (z >> 27)) * 0x94D049BB133111EB
            return z ^ (z >> 31)

Reading adopted for the TQ-MSE value rotation (random signs s in {+-1}^128 of
the randomised Hadamard transform, one draw per (layer, KV head)):

    key = splitmix64(v_seed, n = layer * 2^32 + kv_head)
    s_i = -1 if bit 63 of splitmix64(key, n = i) is set else +1,  i = 0..127
"""
MASK = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15


def mix(z: int) -> int:
    z &= MASK
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK
    return z ^ (z >> 31)


def splitmix64(seed: int, n: int) -> int:
    """n-th output of the SplitMix64 stream seeded with ``seed``."""
    return mix((seed + (n + 1) * GAMMA) & MASK)


def v_signs(v_seed: int, layer: int, kv_head: int, d: int = 128):
    """Sign vector (list of +-1) of the value rotation of one (layer, KV head)."""
    key = splitmix64(v_seed, (layer << 32) + kv_head)
    return [-1 if (splitmix64(key, i) >> 63) else 1 for i in range(d)]


def k_signs(v_seed: int, layer: int, kv_head: int, n: int = 128):
    """Signs of the per-width-group key rotation (when it is on): plan position
    P = 0..n-1 takes output 128 + P of the same stream as the value signs,
    -1 if its bit 63 is set."""
    key = splitmix64(v_seed, (layer << 32) + kv_head)
    return [-1 if (splitmix64(key, 128 + P) >> 63) else 1 for P in range(n)]
