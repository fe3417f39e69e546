"""ctypes binding of libkvq (C ABI in include/kvq.h).

Argument marshalling only: every step of the quantize and decode path runs in
the library's CUDA kernels. PyTorch supplies device memory and the current
stream. There is no fallback: if ``libkvq.so`` is missing the import of the
library raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvq.so")

OK = 0
ERR_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA = -1, -2, -3, -4
FLAG_CAPACITY, FLAG_NONFINITE, FLAG_NORM_SAT, FLAG_TIMEOUT, FLAG_BAD_PLAN = 1, 2, 4, 8, 16
FLAG_BAD_PAGE = 32
BF16, FP16, FP32 = 0, 1, 2
ALLOC_GREEDY, ALLOC_UNIFORM = 0, 1
ALLOC_ROTATE_KEYS = 0x100
STEP_EARLY = 1
STEP_ROPE = 2
PLAN_BYTES = 1024
PLAN_MAGIC = 0x5051564B

# Plan record layout (kvq.h).
PLAN_DTYPE = np.dtype([
    ("magic", "<u4"), ("bits_k", "<i4"), ("bits_v", "<i4"), ("n_ranks", "<i4"),
    ("layer", "<i4"), ("kv_head", "<i4"), ("words_k", "<i4"), ("words_v", "<i4"),
    ("g", "<f4", 64), ("a_hat", "<f4", 64), ("width", "u1", 64), ("order", "u1", 64),
    ("seg_off", "<u2", 65), ("n_half", "u1"), ("pad0", "u1"), ("hs_width", "u1", 32),
    ("hs_rank0", "u1", 32), ("hs_count", "u1", 32), ("v_sign", "<u4", 4), ("pad1", "<u4"),
    ("energy_sum", "<f8"), ("n_class", "u1"), ("pad2", "u1", 7), ("cls_w", "u1", 8),
    ("cls_hs0", "u1", 8), ("cls_nhs", "u1", 8), ("cls_last", "u1", 8), ("cls_seg0", "<u2", 8),
    ("k_sign", "<u4", 4), ("k_rot", "u1"), ("pad3", "u1", 3),
    ("tail", "u1", PLAN_BYTES - 1004),
])
assert PLAN_DTYPE.itemsize == PLAN_BYTES


class KVQError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"kvq error {code}: {msg}")
        self.code = code


class Cfg(ctypes.Structure):
    _fields_ = [("head_dim", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("bits_k", ctypes.c_int32), ("bits_v", ctypes.c_int32), ("b_max", ctypes.c_int32),
                ("alloc_mode", ctypes.c_int32), ("v_seed", ctypes.c_uint64)]


def make_cfg(n_kv_heads, bits_k, bits_v, v_seed=0, alloc_mode=ALLOC_GREEDY, head_dim=128):
    return Cfg(head_dim, n_kv_heads, bits_k, bits_v, 8, alloc_mode, v_seed)


class Pages(ctypes.Structure):
    """kvq_pages: pool, block table [batch][max_pages] (int32 page ids),
    pages in the pool, 32-token tiles per page, block-table row length."""
    _fields_ = [("pool", ctypes.c_void_p), ("block_table", ctypes.c_void_p),
                ("n_pages", ctypes.c_int64), ("page_tiles", ctypes.c_int32),
                ("max_pages", ctypes.c_int32)]


_vp, _sz, _i32, _i64, _u32p = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_int64, \
    ctypes.c_void_p
_SIGS = {
    "kvq_version": (ctypes.c_char_p, []),
    "kvq_last_error": (ctypes.c_char_p, []),
    "kvq_plan_bytes": (_sz, []),
    "kvq_tile_bytes": (_sz, [ctypes.POINTER(Cfg)]),
    "kvq_cache_bytes": (_sz, [ctypes.POINTER(Cfg), _i64]),
    "kvq_alloc_workspace_bytes": (_sz, [ctypes.POINTER(Cfg)]),
    "kvq_decode_workspace_bytes": (_sz, [ctypes.POINTER(Cfg), _i32, _i32, _i64]),
    "kvq_alloc_bits": (_i32, [ctypes.POINTER(Cfg), _i32, _vp, _i32, _i64, _vp, _sz, _vp, _vp,
                              _vp, _vp, _vp]),
    "kvq_plan_build": (_i32, [ctypes.POINTER(Cfg), _i32, _vp, _i32, _vp]),
    "kvq_codebook": (_i32, [_i32, _vp, _vp, _vp]),
    "kvq_quantize_append": (_i32, [ctypes.POINTER(Cfg), _vp, _vp, _vp, _i32, _i32, _i32, _vp, _vp,
                                   _i64, _vp, _vp]),
    "kvq_decode_attn": (_i32, [ctypes.POINTER(Cfg), _vp, _vp, _vp, _i32, _i64, _vp, _i32, _i32,
                               _vp, _vp, _sz, _vp, _vp]),
    "kvq_append_decode": (_i32, [ctypes.POINTER(Cfg), _vp, _vp, _vp, _i32, _i32, _vp, _vp, _i64,
                                 _i32, _i64, _vp, _i32, _i32, _vp, _vp, _sz, _i32,
                                 ctypes.c_double, _vp, _vp]),
    "kvq_decode_attn_noalloc": (_i32, [ctypes.POINTER(Cfg), _vp, _vp, _vp, _i32, _i64, _vp, _i32,
                                       _i32, _vp, _vp, _vp]),
    "kvq_decode_noalloc_scratch_bytes": (_sz, []),
    "kvq_bf16_decode_workspace_bytes": (_sz, [_i32, _i32, _i32, _i64]),
    "kvq_bf16_decode_attn": (_i32, [_vp, _vp, _vp, _i32, _i32, _i64, _i64, _vp, _i32, _vp, _vp, _sz,
                                    _vp, _vp]),
    "kvq_quantize_append_rope": (_i32, [ctypes.POINTER(Cfg), _vp, _vp, _vp, _i32, _i32, _i32, _vp,
                                        _vp, _i64, ctypes.c_double, _vp, _vp]),
    "kvq_decode_attn_partial": (_i32, [ctypes.POINTER(Cfg), _vp, _vp, _vp, _i32, _i64, _vp, _i32,
                                       _i32, _vp, _vp, _sz, _vp, _vp]),
    "kvq_combine_partials": (_i32, [ctypes.POINTER(Cfg), _vp, _i32, _vp, _i32, _i32, _vp, _vp]),
    "kvq_page_bytes": (_sz, [ctypes.POINTER(Cfg), _i32]),
    "kvq_plan_check": (_i32, [ctypes.POINTER(Cfg), _vp]),
    "kvq_energy_workspace_bytes": (_sz, [_i32]),
    "kvq_block_energy": (_i32, [_vp, _i32, _i64, _i32, _vp, _sz, _vp, _vp, _vp]),
    "kvq_plan_build_weighted": (_i32, [ctypes.POINTER(Cfg), _i32, _vp, _vp, _i32, _vp]),
    "kvq_paged_quantize_append": (_i32, [ctypes.POINTER(Cfg), _vp, _vp, _vp, _i32, _i32, _i32,
                                         ctypes.POINTER(Pages), _vp, ctypes.c_double, _vp, _vp]),
    "kvq_paged_decode_attn": (_i32, [ctypes.POINTER(Cfg), _vp, ctypes.POINTER(Pages), _vp, _i32,
                                     _i64, _vp, _i32, _i32, _vp, _vp, _sz, _vp, _vp]),
    "kvq_paged_decode_attn_partial": (_i32, [ctypes.POINTER(Cfg), _vp, ctypes.POINTER(Pages),
                                             _vp, _i32, _i64, _vp, _i32, _i32, _vp, _vp, _sz,
                                             _vp, _vp]),
    "kvq_paged_append_decode": (_i32, [ctypes.POINTER(Cfg), _vp, _vp, _vp, _i32, _i32,
                                       ctypes.POINTER(Pages), _vp, _i32, _i64, _vp, _i32, _i32,
                                       _vp, _vp, _sz, _i32, ctypes.c_double, _vp, _vp]),
    "kvq_debug_decode_stall": (_i32, [ctypes.c_longlong]),
    "kvq_set_decode_deterministic": (_i32, [_i32]),
    "kvq_window_bytes": (_sz, [ctypes.POINTER(Cfg), _i32]),
    "kvq_window_append": (_i32, [ctypes.POINTER(Cfg), _vp, _vp, _vp, _i32, _i32, _vp, _vp, _i64,
                                 _vp, _vp, _i32, _i32, _vp, _vp]),
    "kvq_window_decode_workspace_bytes": (_sz, [ctypes.POINTER(Cfg), _i32, _i32, _i64]),
    "kvq_decode_attn_window": (_i32, [ctypes.POINTER(Cfg), _vp, _vp, _vp, _vp, _vp, _i32, _i32,
                                      _i64, _vp, _i32, _i32, _vp, _vp, _sz, _vp, _vp]),
    "kvq_append_decode_window": (_i32, [ctypes.POINTER(Cfg), _vp, _vp, _vp, _i32, _i32, _vp, _vp,
                                        _i64, _vp, _vp, _i32, _i32, _i64, _vp, _i32, _i32, _vp,
                                        _vp, _sz, _i32, _vp, _vp]),
}
EXPORTS = tuple(_SIGS)

_lib = None


def lib():
    """The loaded libkvq (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with "
                              "`python -m bit_kv_cache_19_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(rc):
    if rc != OK:
        raise KVQError(rc, lib().kvq_last_error().decode())
    return rc


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dtype_code(t):
    import torch
    return {torch.bfloat16: BF16, torch.float16: FP16, torch.float32: FP32}[t.dtype]


# ------------------------------------------------------------ sizes, host-only
def version() -> str:
    return lib().kvq_version().decode()


def tile_bytes(cfg) -> int:
    return lib().kvq_tile_bytes(ctypes.byref(cfg))


def cache_bytes(cfg, cap_tokens) -> int:
    return lib().kvq_cache_bytes(ctypes.byref(cfg), cap_tokens)


def alloc_workspace_bytes(cfg) -> int:
    return lib().kvq_alloc_workspace_bytes(ctypes.byref(cfg))


def decode_workspace_bytes(cfg, batch, n_q_heads, max_len) -> int:
    return lib().kvq_decode_workspace_bytes(ctypes.byref(cfg), batch, n_q_heads, max_len)


def codebook(bits):
    """(centroids float32 [2^b], thresholds float32 [2^b - 1], D) of the library."""
    c = np.zeros(1 << bits, dtype=np.float32)
    t = np.zeros((1 << bits) - 1, dtype=np.float32)
    d = ctypes.c_double()
    _check(lib().kvq_codebook(bits, c.ctypes.data, t.ctypes.data, ctypes.byref(d)))
    return c, t, d.value


def plan_build(cfg, layer, E) -> np.ndarray:
    """Host plan records (PLAN_DTYPE array) from energies E[n_heads, 64]."""
    E = np.ascontiguousarray(np.asarray(E, dtype=np.float64))
    n = E.shape[0]
    out = np.zeros(n, dtype=PLAN_DTYPE)
    _check(lib().kvq_plan_build(ctypes.byref(cfg), layer, E.ctypes.data, n, out.ctypes.data))
    return out


def plan_build_weighted(cfg, layer, E, Eq) -> np.ndarray:
    """Host plans of the query-weighted variant: widths from the greedy on
    E * W, W the query energies Eq [n_q_heads, 64] averaged over each KV
    head's group (in the library); key scales from E [n_kv_heads, 64]."""
    E = np.ascontiguousarray(E, dtype=np.float64)
    Eq = np.ascontiguousarray(Eq, dtype=np.float64)
    out = np.zeros(E.shape[0], dtype=PLAN_DTYPE)
    _check(lib().kvq_plan_build_weighted(ctypes.byref(cfg), layer, E.ctypes.data, Eq.ctypes.data,
                                         Eq.shape[0], out.ctypes.data))
    return out


def block_energy(x, status=None, ws=None) -> np.ndarray:
    """Exact block energies fp64 [n_heads, 64] of a device tensor
    x [n_tokens, n_heads, 128] (e.g. calibration queries)."""
    import torch
    n_heads = x.shape[1]
    if ws is None:
        ws = torch.zeros(lib().kvq_energy_workspace_bytes(n_heads), dtype=torch.uint8,
                         device=x.device)
    E = np.zeros((n_heads, 64), dtype=np.float64)
    _check(lib().kvq_block_energy(_ptr(x), _dtype_code(x), x.shape[0], n_heads, _ptr(ws),
                                  ws.numel(), E.ctypes.data, _ptr(status), _stream()))
    return E


def plan_check(cfg, plans):
    """Raise KVQError unless every host plan record (PLAN_DTYPE array) is
    consistent (kvq_plan_check)."""
    plans = np.ascontiguousarray(plans)
    for i in range(plans.shape[0]):
        _check(lib().kvq_plan_check(ctypes.byref(cfg), plans[i:i + 1].ctypes.data))


def parse_plans(raw) -> np.ndarray:
    return np.frombuffer(bytes(raw), dtype=PLAN_DTYPE)


# ------------------------------------------------------------------ device
def ptr_array(tensors, device):
    """Device int64 tensor holding the data pointers of ``tensors``."""
    import torch
    return torch.tensor([t.data_ptr() for t in tensors], dtype=torch.int64, device=device)


def alloc_bits(cfg, layer, k, plans_dev, status=None, ws=None):
    """Energy + greedy plans of one layer. k: [T, n_kv, 128] on the device.

    Writes plans_dev (uint8 [n_kv * 1024]); returns (host plans, energies)."""
    import torch
    n_kv = cfg.n_kv_heads
    if ws is None:
        ws = torch.empty(alloc_workspace_bytes(cfg), dtype=torch.uint8, device=k.device)
    host = np.zeros(n_kv, dtype=PLAN_DTYPE)
    E = np.zeros((n_kv, 64), dtype=np.float64)
    _check(lib().kvq_alloc_bits(ctypes.byref(cfg), layer, _ptr(k), _dtype_code(k), k.shape[0],
                                _ptr(ws), ws.numel(), _ptr(plans_dev), host.ctypes.data,
                                E.ctypes.data, _ptr(status), _stream()))
    return host, E


def quantize_append(cfg, plan_ptrs, k, v, cache_ptrs, lens, cap_tokens, status):
    """Append k, v [batch, n_new, n_kv, 128] to the packed caches."""
    batch, n_new = k.shape[0], k.shape[1]
    _check(lib().kvq_quantize_append(ctypes.byref(cfg), _ptr(plan_ptrs), _ptr(k), _ptr(v),
                                     _dtype_code(k), batch, n_new, _ptr(cache_ptrs), _ptr(lens),
                                     cap_tokens, _ptr(status), _stream()))


def quantize_append_rope(cfg, plan_ptrs, k, v, cache_ptrs, lens, cap_tokens, rope_base, status):
    """Fused RoPE + append: k [batch, n_new, n_kv, 128] holds pre-RoPE keys,
    rotated to their cache positions before they are quantized."""
    batch, n_new = k.shape[0], k.shape[1]
    _check(lib().kvq_quantize_append_rope(ctypes.byref(cfg), _ptr(plan_ptrs), _ptr(k), _ptr(v),
                                          _dtype_code(k), batch, n_new, _ptr(cache_ptrs),
                                          _ptr(lens), cap_tokens, float(rope_base), _ptr(status),
                                          _stream()))


def decode_attn(cfg, plan_ptrs, cache_ptrs, lens, max_len, q, out, ws, status):
    """Packed-cache decode attention; q [batch, n_q, 128], out fp32 same shape."""
    batch, n_q = q.shape[0], q.shape[1]
    _check(lib().kvq_decode_attn(ctypes.byref(cfg), _ptr(plan_ptrs), _ptr(cache_ptrs), _ptr(lens),
                                 batch, max_len, _ptr(q), _dtype_code(q), n_q, _ptr(out), _ptr(ws),
                                 ws.numel() * ws.element_size(), _ptr(status), _stream()))


REC_FLOATS = 132  # partial-decode record: m, l, 2 unused, o_rot[128]


def decode_attn_partial(cfg, plan_ptrs, cache_ptrs, lens, max_len, q, rec, ws, status):
    """Decode over one context shard (caches holding a token range of each
    sequence) into merged records rec fp32 [batch, n_q, 132]: (m, l, -, -,
    o_rot) with 2^m l = sum_t 2^s_t and 2^m o_rot = sum_t 2^s_t v_rot_t."""
    batch, n_q = q.shape[0], q.shape[1]
    _check(lib().kvq_decode_attn_partial(ctypes.byref(cfg), _ptr(plan_ptrs), _ptr(cache_ptrs),
                                         _ptr(lens), batch, max_len, _ptr(q), _dtype_code(q), n_q,
                                         _ptr(rec), _ptr(ws), ws.numel() * ws.element_size(),
                                         _ptr(status), _stream()))


def combine_partials(cfg, plan_ptrs, recs, out):
    """Merge the stacked records recs fp32 [n_parts, batch, n_q, 132] of the
    shards of the same sequences and undo the value rotation into out fp32
    [batch, n_q, 128]."""
    n_parts, batch, n_q = recs.shape[0], recs.shape[1], recs.shape[2]
    _check(lib().kvq_combine_partials(ctypes.byref(cfg), _ptr(plan_ptrs), n_parts, _ptr(recs),
                                      batch, n_q, _ptr(out), _stream()))


def page_bytes(cfg, page_tiles) -> int:
    return lib().kvq_page_bytes(ctypes.byref(cfg), page_tiles)


def make_pages(pool, block_table, n_pages, page_tiles):
    """kvq_pages over a device pool (n_pages pages of page_bytes) and a device
    block table int32 [batch, max_pages]."""
    return Pages(pool.data_ptr(), block_table.data_ptr(), n_pages, page_tiles,
                 block_table.shape[1])


def paged_quantize_append(cfg, plan_ptrs, k, v, pages, lens, status, rope_base=0.0):
    """kvq_quantize_append into paged caches (rope_base > 1: pre-RoPE keys)."""
    batch, n_new = k.shape[0], k.shape[1]
    _check(lib().kvq_paged_quantize_append(ctypes.byref(cfg), _ptr(plan_ptrs), _ptr(k), _ptr(v),
                                           _dtype_code(k), batch, n_new, ctypes.byref(pages),
                                           _ptr(lens), float(rope_base), _ptr(status),
                                           _stream()))


def paged_decode_attn(cfg, plan_ptrs, pages, lens, max_len, q, out, ws, status):
    """kvq_decode_attn over paged caches."""
    batch, n_q = q.shape[0], q.shape[1]
    _check(lib().kvq_paged_decode_attn(ctypes.byref(cfg), _ptr(plan_ptrs), ctypes.byref(pages),
                                       _ptr(lens), batch, max_len, _ptr(q), _dtype_code(q), n_q,
                                       _ptr(out), _ptr(ws), ws.numel() * ws.element_size(),
                                       _ptr(status), _stream()))


def paged_decode_attn_partial(cfg, plan_ptrs, pages, lens, max_len, q, rec, ws, status):
    """kvq_decode_attn_partial over paged caches: records fp32 [batch, n_q, 132]."""
    batch, n_q = q.shape[0], q.shape[1]
    _check(lib().kvq_paged_decode_attn_partial(ctypes.byref(cfg), _ptr(plan_ptrs),
                                               ctypes.byref(pages), _ptr(lens), batch, max_len,
                                               _ptr(q), _dtype_code(q), n_q, _ptr(rec), _ptr(ws),
                                               ws.numel() * ws.element_size(), _ptr(status),
                                               _stream()))


def paged_append_decode(cfg, plan_ptrs, k, v, pages, lens, max_len, q, out, ws, status,
                        step_flags=0, rope_base=0.0):
    """kvq_append_decode over paged caches."""
    batch, n_q = q.shape[0], q.shape[1]
    n_new = 0 if k is None else k.shape[1]
    _check(lib().kvq_paged_append_decode(ctypes.byref(cfg), _ptr(plan_ptrs), _ptr(k), _ptr(v),
                                         _dtype_code(k) if k is not None else BF16, n_new,
                                         ctypes.byref(pages), _ptr(lens), batch, max_len,
                                         _ptr(q), _dtype_code(q), n_q, _ptr(out), _ptr(ws),
                                         ws.numel() * ws.element_size(), step_flags,
                                         float(rope_base), _ptr(status), _stream()))


def append_decode(cfg, plan_ptrs, k, v, cache_ptrs, lens, cap_tokens, max_len, q, out, ws,
                  status, step_flags=0, rope_base=0.0):
    """Append k, v [batch, n_new, n_kv, 128] and decode q [batch, n_q, 128] in one launch.

    step_flags=STEP_EARLY: stream the caches before the previous kernel ends
    (only when that kernel writes neither these caches nor these lengths);
    STEP_ROPE: k holds pre-RoPE keys, rotated with base rope_base."""
    batch, n_q = q.shape[0], q.shape[1]
    n_new = 0 if k is None else k.shape[1]
    _check(lib().kvq_append_decode(ctypes.byref(cfg), _ptr(plan_ptrs), _ptr(k), _ptr(v),
                                   _dtype_code(k) if k is not None else BF16, n_new,
                                   _ptr(cache_ptrs), _ptr(lens), cap_tokens, batch, max_len,
                                   _ptr(q), _dtype_code(q), n_q, _ptr(out), _ptr(ws),
                                   ws.numel() * ws.element_size(), step_flags,
                                   float(rope_base), _ptr(status), _stream()))


def decode_attn_noalloc(cfg, plan_ptrs, cache_ptrs, lens, max_len, q, out, status):
    """kvq_decode_attn without a caller workspace: the split partials go to
    the library's fixed 16 MiB device scratch (for callers that cannot
    allocate device memory where they decode). Calls must not overlap on the
    GPU; the first call on a device must precede any stream capture."""
    batch, n_q = q.shape[0], q.shape[1]
    _check(lib().kvq_decode_attn_noalloc(ctypes.byref(cfg), _ptr(plan_ptrs), _ptr(cache_ptrs),
                                         _ptr(lens), batch, max_len, _ptr(q), _dtype_code(q), n_q,
                                         _ptr(out), _ptr(status), _stream()))


def bf16_decode_workspace_bytes(batch, n_kv_heads, n_q_heads, max_len) -> int:
    return lib().kvq_bf16_decode_workspace_bytes(batch, n_kv_heads, n_q_heads, max_len)


def bf16_decode_attn(k, v, lens, max_len, q, out, ws, status):
    """bf16 comparator (not the method): dense split-K decode attention over
    k, v [batch, n_kv, cap, 128] bf16 with q [batch, n_q, 128] bf16 into out
    [batch, n_q, 128] fp32."""
    batch, n_kv, cap = k.shape[0], k.shape[1], k.shape[2]
    _check(lib().kvq_bf16_decode_attn(_ptr(k), _ptr(v), _ptr(lens), batch, n_kv, cap, max_len,
                                      _ptr(q), q.shape[1], _ptr(out), _ptr(ws),
                                      ws.numel() * ws.element_size(), _ptr(status), _stream()))


def window_bytes(cfg, R) -> int:
    """Bytes of one sequence's recent-token window of R slots."""
    return lib().kvq_window_bytes(ctypes.byref(cfg), R)


def window_decode_workspace_bytes(cfg, batch, n_q_heads, max_len) -> int:
    return lib().kvq_window_decode_workspace_bytes(ctypes.byref(cfg), batch, n_q_heads, max_len)


def window_append(cfg, plan_ptrs, k, v, cache_ptrs, lens, cap_tokens, win_ptrs, wlens, R,
                  status):
    """Append k, v [batch, n_new, n_kv, 128]: the oldest tokens beyond the
    R-token window are quantize-appended, the rest enter the window ring."""
    batch, n_new = k.shape[0], k.shape[1]
    _check(lib().kvq_window_append(ctypes.byref(cfg), _ptr(plan_ptrs), _ptr(k), _ptr(v),
                                   _dtype_code(k), n_new, _ptr(cache_ptrs), _ptr(lens),
                                   cap_tokens, _ptr(win_ptrs), _ptr(wlens), R, batch,
                                   _ptr(status), _stream()))


def append_decode_window(cfg, plan_ptrs, k, v, cache_ptrs, lens, cap_tokens, win_ptrs, wlens, R,
                         max_len, q, out, ws, status, step_flags=0):
    """Window append of k, v [batch, n_new, n_kv, 128] then decode of q
    [batch, n_q, 128]; one launch for n_new = 1."""
    batch, n_new = k.shape[0], k.shape[1]
    _check(lib().kvq_append_decode_window(ctypes.byref(cfg), _ptr(plan_ptrs), _ptr(k), _ptr(v),
                                          _dtype_code(k), n_new, _ptr(cache_ptrs), _ptr(lens),
                                          cap_tokens, _ptr(win_ptrs), _ptr(wlens), R, batch,
                                          max_len, _ptr(q), _dtype_code(q), q.shape[1], _ptr(out),
                                          _ptr(ws), ws.numel() * ws.element_size(), step_flags,
                                          _ptr(status), _stream()))


def decode_attn_window(cfg, plan_ptrs, cache_ptrs, lens, win_ptrs, wlens, R, max_len, q, out,
                       ws, status):
    """Decode q [batch, n_q, 128] over the packed tokens and the window tokens."""
    batch, n_q = q.shape[0], q.shape[1]
    _check(lib().kvq_decode_attn_window(ctypes.byref(cfg), _ptr(plan_ptrs), _ptr(cache_ptrs),
                                        _ptr(lens), _ptr(win_ptrs), _ptr(wlens), R, batch,
                                        max_len, _ptr(q), _dtype_code(q), n_q, _ptr(out),
                                        _ptr(ws), ws.numel() * ws.element_size(), _ptr(status),
                                        _stream()))
