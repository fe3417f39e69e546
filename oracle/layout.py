"""Packed KV tile record: pack and unpack (oracle; test infrastructure only).

"RoPE-Aware Bit Allocation for KV-Cache Quantization", abstract: the packed
K3V3 cache of the serving path reaches 3.24x compression. The layout is not
printed; this module defines the one adopted here. Code bits are counted
exactly: b_K bits per key dimension and b_V per value dimension, plus one fp16
norm per token for K and one for V (K3V3: 100 bytes per token and KV head).

The cache of one (sequence, layer, KV head) is a run of tile records, each
holding 32 consecutive tokens (token t sits in tile t // 32, position
t % 32). A record is little-endian 32-bit words:

    [K part: 128 b_K words][V part: 128 b_V words][Knorm: 32 fp16][Vnorm: 32 fp16]

K part: one segment per stored RoPE block, in plan order (see
``alloc.plan_order``). A block of width w has 2w words holding 32 fields of
2w bits; the field of token position t sits at bit offset slot_k(t) * 2w
(LSB first, bit b of the segment is bit b % 32 of word b // 32); its low w
bits are the code of coordinate j, its high w bits the code of j + 64.

V part: one segment of b_V words per rotated coordinate p = 0..127, holding
32 fields of b_V bits; token position t's code sits at bit slot_v(t) * b_V.

Slot orders (chosen so that the decode kernel's matrix-fragment registers are
filled from contiguous bits):
    slot_k(t) = 4 (t mod 8) + t div 8
    slot_v(t) = 8 ((t mod 8) div 2) + 2 (t div 8) + (t mod 2)

Bits of positions not holding a token are zero. Norm slots of such positions
are unspecified.
"""
from __future__ import annotations

import numpy as np

TILE = 32


def slot_k(t):
    t = np.asarray(t)
    return 4 * (t % 8) + t // 8


def slot_v(t):
    t = np.asarray(t)
    return 8 * ((t % 8) // 2) + 2 * (t // 8) + (t % 2)


def tile_words(bits_k: int, bits_v: int) -> int:
    return 128 * (bits_k + bits_v) + 32


def tile_bytes(bits_k: int, bits_v: int) -> int:
    return 4 * tile_words(bits_k, bits_v)


def _pack_fields(fields: np.ndarray, f: int) -> np.ndarray:
    """fields[n, 32] (slot order, < 2^f) -> words[n, f]."""
    n = fields.shape[0]
    bits = ((fields[:, :, None] >> np.arange(f)[None, None, :]) & 1).astype(np.uint8)
    by = np.packbits(bits.reshape(n, 32 * f), axis=1, bitorder="little")
    return by.view("<u4").reshape(n, f)


def _unpack_fields(words: np.ndarray, f: int) -> np.ndarray:
    """words[n, f] -> fields[n, 32] (slot order)."""
    n = words.shape[0]
    by = np.ascontiguousarray(words.astype("<u4")).view(np.uint8).reshape(n, 4 * f)
    bits = np.unpackbits(by, axis=1, bitorder="little").reshape(n, 32, f).astype(np.int64)
    return np.sum(bits << np.arange(f)[None, None, :], axis=2)


def pack(k_codes, v_codes, k_norm, v_norm, plan, length: int) -> np.ndarray:
    """Tile records [n_tiles, tile_words] (uint32) for ``length`` tokens.

    k_codes[T, 128] canonical coordinates, v_codes[T, 128] rotated coordinates,
    norms as fp16 values; T >= length. Norm slots past ``length`` are 0 here.
    """
    bk, bv = plan.bits_k, plan.bits_v
    n_tiles = (length + TILE - 1) // TILE
    W = tile_words(bk, bv)
    rec = np.zeros((n_tiles, W), dtype=np.uint32)
    pos = np.arange(n_tiles * TILE)
    valid = pos < length
    kc = np.zeros((n_tiles * TILE, 128), dtype=np.int64)
    vc = np.zeros((n_tiles * TILE, 128), dtype=np.int64)
    kc[:length] = np.asarray(k_codes)[:length]
    vc[:length] = np.asarray(v_codes)[:length]
    sk = slot_k(np.arange(TILE))
    sv = slot_v(np.arange(TILE))
    off = 0
    for j in plan.order:
        w = int(plan.widths[j])
        fld = kc[:, j] | (kc[:, j + 64] << w)
        fld = np.where(valid, fld, 0).reshape(n_tiles, TILE)
        by_slot = np.zeros_like(fld)
        by_slot[:, sk] = fld
        rec[:, off:off + 2 * w] = _pack_fields(by_slot, 2 * w)
        off += 2 * w
    assert off == 128 * bk
    for p in range(128):
        fld = np.where(valid, vc[:, p], 0).reshape(n_tiles, TILE)
        by_slot = np.zeros_like(fld)
        by_slot[:, sv] = fld
        rec[:, off:off + bv] = _pack_fields(by_slot, bv)
        off += bv
    kn = np.zeros(n_tiles * TILE, dtype=np.float16)
    vn = np.zeros(n_tiles * TILE, dtype=np.float16)
    kn[:length] = np.asarray(k_norm, dtype=np.float32)[:length].astype(np.float16)
    vn[:length] = np.asarray(v_norm, dtype=np.float32)[:length].astype(np.float16)
    rec[:, off:off + 16] = kn.view(np.uint16).reshape(n_tiles, 16, 2).astype(np.uint32) @ \
        np.array([1, 1 << 16], dtype=np.uint32)
    rec[:, off + 16:off + 32] = vn.view(np.uint16).reshape(n_tiles, 16, 2).astype(np.uint32) @ \
        np.array([1, 1 << 16], dtype=np.uint32)
    return rec


def unpack(rec, plan, length: int):
    """Inverse of ``pack``: (k_codes, v_codes, k_norm, v_norm) for ``length``
    tokens; codes of width-0 key blocks are 0; norms as float32."""
    rec = np.asarray(rec, dtype=np.uint32)
    n_tiles = rec.shape[0]
    bk, bv = plan.bits_k, plan.bits_v
    kc = np.zeros((n_tiles * TILE, 128), dtype=np.int64)
    vc = np.zeros((n_tiles * TILE, 128), dtype=np.int64)
    sk = slot_k(np.arange(TILE))
    sv = slot_v(np.arange(TILE))
    off = 0
    for j in plan.order:
        w = int(plan.widths[j])
        fld = _unpack_fields(rec[:, off:off + 2 * w], 2 * w)[:, sk].reshape(-1)
        kc[:, j] = fld & ((1 << w) - 1)
        kc[:, j + 64] = fld >> w
        off += 2 * w
    for p in range(128):
        vc[:, p] = _unpack_fields(rec[:, off:off + bv], bv)[:, sv].reshape(-1)
        off += bv
    kn = (rec[:, off:off + 16].astype(np.uint32)[:, :, None] >> np.array([0, 16])) & 0xFFFF
    vn = (rec[:, off + 16:off + 32].astype(np.uint32)[:, :, None] >> np.array([0, 16])) & 0xFFFF
    kn = kn.astype(np.uint16).reshape(-1).view(np.float16).astype(np.float32)
    vn = vn.astype(np.uint16).reshape(-1).view(np.float16).astype(np.float32)
    return kc[:length], vc[:length], kn[:length], vn[:length]
