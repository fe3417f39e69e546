"""Device-memory plumbing around libkvq (PyTorch tensors; no compute here).

``PackedLayer`` owns, for one layer and a batch of sequences, the plan
records, the packed caches, their pointer arrays, the lengths and the status
word, and forwards to the C-ABI calls; ``sharded_decode`` is the one
exchange step of a decode whose context is split over ranks.
"""
from __future__ import annotations

import collections

import numpy as np
import torch

from . import kvq


class PackedLayer:
    """One layer's packed caches for a batch of sequences. ``window=R > 0``
    adds a recent-token window per sequence: the R most recent tokens stay
    exact (appended with ``append_window``, decoded with ``decode_window``);
    ``lens`` then counts the packed tokens and ``wlens`` the window's."""

    def __init__(self, cfg, batch: int, cap_tokens: int, device="cuda", layer: int = 0,
                 window: int = 0):
        self.cfg = cfg
        self.batch = batch
        self.cap = cap_tokens
        self.layer = layer
        self.device = torch.device(device)
        n_kv = cfg.n_kv_heads
        self.plans = torch.zeros(n_kv * kvq.PLAN_BYTES, dtype=torch.uint8, device=self.device)
        nbytes = kvq.cache_bytes(cfg, cap_tokens)
        self.caches = [torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
                       for _ in range(batch)]
        self.cache_ptrs = kvq.ptr_array(self.caches, self.device)
        self.plan_ptrs = kvq.ptr_array([self.plans] * batch, self.device)
        self.lens = torch.zeros(batch, dtype=torch.int32, device=self.device)
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.plans_host = None
        self.energy = None
        self.window = window
        self.wlens = torch.zeros(batch, dtype=torch.int32, device=self.device)
        self.wins, self.win_ptrs = [], None
        if window > 0:
            wb = kvq.window_bytes(cfg, window)
            self.wins = [torch.zeros(wb // 4, dtype=torch.float32, device=self.device)
                         for _ in range(batch)]
            self.win_ptrs = kvq.ptr_array(self.wins, self.device)

    # -------------------------------------------------------------- calls
    def alloc_bits(self, k):
        """Plans from keys k [T, n_kv, 128] (device)."""
        self.plans_host, self.energy = kvq.alloc_bits(self.cfg, self.layer, k, self.plans,
                                                      self.status)
        return self.plans_host

    def alloc_bits_query_weighted(self, k, q_calib):
        """Query-weighted variant: key energies of k [T, n_kv, 128] and query
        energies of calibration queries q_calib [Tq, n_q, 128] (both device
        tensors, both by the library's energy kernel); the library averages
        the query energies over each KV head's group and runs the greedy on
        the products."""
        E = kvq.block_energy(k, self.status)
        Eq = kvq.block_energy(q_calib, self.status)
        self.set_plans(kvq.plan_build_weighted(self.cfg, self.layer, E, Eq))
        self.energy = E
        return self.plans_host

    def set_plans(self, plans_host: np.ndarray, check: bool = True):
        """Use host plan records (e.g. from kvq.plan_build); checked on the
        host first (kvq_plan_check) unless check=False."""
        if check:
            kvq.plan_check(self.cfg, plans_host)
        raw = torch.from_numpy(np.frombuffer(plans_host.tobytes(), dtype=np.uint8).copy())
        self.plans.copy_(raw.to(self.device))
        self.plans_host = plans_host

    def append(self, k, v):
        """k, v [batch, n_new, n_kv, 128] (device) appended after each length."""
        kvq.quantize_append(self.cfg, self.plan_ptrs, k, v, self.cache_ptrs, self.lens, self.cap,
                            self.status)

    def append_rope(self, k_pre, v, rope_base):
        """Pre-RoPE keys k_pre, values v [batch, n_new, n_kv, 128] (device):
        each key is rotated to its cache position, then appended."""
        kvq.quantize_append_rope(self.cfg, self.plan_ptrs, k_pre, v, self.cache_ptrs, self.lens,
                                 self.cap, rope_base, self.status)

    def append_window(self, k, v):
        """k, v [batch, n_new, n_kv, 128] (device) through the recent-token
        window: tokens older than the window's R are quantize-appended."""
        kvq.window_append(self.cfg, self.plan_ptrs, k, v, self.cache_ptrs, self.lens, self.cap,
                          self.win_ptrs, self.wlens, self.window, self.status)

    def decode_window(self, q, out=None, ws=None, max_len=None):
        """q [batch, n_q, 128] -> fp32 [batch, n_q, 128] over the packed and
        the window tokens."""
        max_len = self.cap if max_len is None else max_len
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=self.device)
        if ws is None:
            n = kvq.window_decode_workspace_bytes(self.cfg, self.batch, q.shape[1], max_len)
            ws = torch.zeros(n, dtype=torch.uint8, device=self.device)
        kvq.decode_attn_window(self.cfg, self.plan_ptrs, self.cache_ptrs, self.lens,
                               self.win_ptrs, self.wlens, self.window, max_len, q, out, ws,
                               self.status)
        return out

    def append_decode_window(self, k, v, q, out=None, ws=None, max_len=None, step_flags=0):
        """One window step: append k, v [batch, n_new, n_kv, 128] through the
        window and decode q [batch, n_q, 128] over packed + window tokens (one
        launch for n_new = 1)."""
        max_len = self.cap if max_len is None else max_len
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=self.device)
        if ws is None:
            n = kvq.window_decode_workspace_bytes(self.cfg, self.batch, q.shape[1], max_len)
            ws = torch.zeros(n, dtype=torch.uint8, device=self.device)
        kvq.append_decode_window(self.cfg, self.plan_ptrs, k, v, self.cache_ptrs, self.lens,
                                 self.cap, self.win_ptrs, self.wlens, self.window, max_len, q, out,
                                 ws, self.status, step_flags)
        return out

    def window_rows(self, seq: int):
        """The window ring of one sequence on the host: keys, values fp32
        [R, n_kv, 128] (slot t mod R holds token t)."""
        R, n_kv = self.window, self.cfg.n_kv_heads
        w = self.wins[seq].cpu().numpy().reshape(2, R, n_kv, 128)
        return w[0], w[1]

    def decode(self, q, out=None, ws=None, max_len=None):
        """q [batch, n_q, 128] -> fp32 [batch, n_q, 128]."""
        max_len = self.cap if max_len is None else max_len
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=self.device)
        if ws is None:
            ws = self.workspace(q.shape[1], max_len)
        kvq.decode_attn(self.cfg, self.plan_ptrs, self.cache_ptrs, self.lens, max_len, q, out, ws,
                        self.status)
        return out

    def append_decode(self, k, v, q, out=None, ws=None, max_len=None, step_flags=0,
                      rope_base=0.0):
        """Fused serving step: append k, v [batch, n_new, n_kv, 128], then decode q."""
        max_len = self.cap if max_len is None else max_len
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=self.device)
        if ws is None:
            ws = self.workspace(q.shape[1], max_len)
        kvq.append_decode(self.cfg, self.plan_ptrs, k, v, self.cache_ptrs, self.lens, self.cap,
                          max_len, q, out, ws, self.status, step_flags, rope_base)
        return out

    def decode_partial(self, q, rec=None, ws=None, max_len=None):
        """Decode over this layer's caches as one context shard: merged
        records fp32 [batch, n_q, 132] (m, l, -, -, o_rot) for combine()."""
        max_len = self.cap if max_len is None else max_len
        if rec is None:
            rec = torch.empty((q.shape[0], q.shape[1], kvq.REC_FLOATS), dtype=torch.float32,
                              device=self.device)
        if ws is None:
            ws = self.workspace(q.shape[1], max_len)
        kvq.decode_attn_partial(self.cfg, self.plan_ptrs, self.cache_ptrs, self.lens, max_len, q,
                                rec, ws, self.status)
        return rec

    def combine(self, recs, out=None):
        """Outputs fp32 [batch, n_q, 128] from the stacked records
        [n_parts, batch, n_q, 132] of the shards of these sequences."""
        if out is None:
            out = torch.empty(recs.shape[1:3] + (128,), dtype=torch.float32, device=self.device)
        kvq.combine_partials(self.cfg, self.plan_ptrs, recs, out)
        return out

    def decode_sharded(self, q, group=None, max_len=None):
        """Context-sharded decode: this rank's caches hold one token range of
        each sequence (ranks in sequence order); one all-gather of records."""
        return sharded_decode(lambda: self.decode_partial(q, max_len=max_len), self.combine, group)

    def workspace(self, n_q: int, max_len: int):
        """Decode workspace, zero-filled (its arrival counters must start at 0)."""
        n = kvq.decode_workspace_bytes(self.cfg, self.batch, n_q, max_len)
        return torch.zeros(n, dtype=torch.uint8, device=self.device)

    # ------------------------------------------------------------ inspect
    def head_records(self, seq: int, head: int, n_tiles: int) -> np.ndarray:
        """Tile records [n_tiles, tile_bytes / 4] (uint32) of one head, on the host."""
        tb = kvq.tile_bytes(self.cfg)
        raw = self.caches[seq][: n_tiles * self.cfg.n_kv_heads * tb].view(
            n_tiles, self.cfg.n_kv_heads, tb)[:, head].contiguous().cpu().numpy()
        return raw.view("<u4").reshape(n_tiles, tb // 4)

    def flags(self) -> int:
        return int(self.status.item()) & 0xFFFFFFFF


def sharded_decode(partial, combine, group=None):
    """One exchange step of a context-sharded decode.

    partial() returns this rank's records [batch, n_q, 132] for its token
    range; the records of all ranks are gathered in rank order (one
    all-gather, a few KB per sequence) and combine(stacked) turns them into
    the outputs over the whole context, identical on every rank."""
    import torch.distributed as dist
    rec = partial()
    world = dist.get_world_size(group)
    recs = torch.empty((world,) + tuple(rec.shape), dtype=rec.dtype, device=rec.device)
    dist.all_gather(list(recs.unbind(0)), rec.contiguous(), group=group)
    return combine(recs)


class PageAllocator:
    """Host-side page bookkeeping of a paged cache: the block table
    [batch][max_pages] (int32 page ids, -1 = none) and a free list. Pages are
    handed out in order (or in a caller's order) as sequences grow and come
    back when a sequence is released."""

    def __init__(self, n_pages: int, page_tiles: int, batch: int, max_pages: int):
        self.n_pages = n_pages
        self.page_tiles = page_tiles
        self.table = np.full((batch, max_pages), -1, dtype=np.int32)
        self.free = collections.deque(range(n_pages))
        self.used = set()
        self.n_held = [0] * batch

    def reserve(self, seq: int, n_tokens: int, order=None):
        """Pages for the first n_tokens tokens of sequence seq (from the free
        list, or taken from `order`, a list consumed from the front; pages in
        use are skipped)."""
        need = -(-n_tokens // (32 * self.page_tiles))
        if need > self.table.shape[1]:
            raise ValueError(f"{n_tokens} tokens exceed the block-table row")
        while self.n_held[seq] < need:
            g = None
            while g is None:
                if order is not None:
                    if not order:
                        break
                    c = int(order.pop(0))
                else:
                    if not self.free:
                        break
                    c = self.free.popleft()
                if c not in self.used:
                    g = c
            if g is None:
                raise MemoryError("page pool exhausted")
            self.used.add(g)
            self.table[seq, self.n_held[seq]] = g
            self.n_held[seq] += 1

    def release(self, seq: int):
        held = self.table[seq, :self.n_held[seq]].tolist()
        self.used.difference_update(held)
        self.free.extend(held)
        self.table[seq, :] = -1
        self.n_held[seq] = 0


class PagedLayer:
    """One layer's packed caches for a batch of sequences in pages of a shared
    pool: the pool, the block table (device) and a host-side page allocator.
    Pages are handed out in order from a free list as sequences grow
    (``reserve``) and returned by ``release``; the kernels only follow the
    block table."""

    def __init__(self, cfg, batch: int, n_pages: int, page_tiles: int, max_pages: int,
                 device="cuda", layer: int = 0):
        self.cfg = cfg
        self.batch = batch
        self.layer = layer
        self.device = torch.device(device)
        self.page_tiles = page_tiles
        self.n_pages = n_pages
        nb = kvq.page_bytes(cfg, page_tiles)
        if nb == 0:
            raise ValueError(f"page_tiles {page_tiles}: a power of two, 1..2^20")
        self.pool = torch.zeros(n_pages * nb, dtype=torch.uint8, device=self.device)
        self.alloc = PageAllocator(n_pages, page_tiles, batch, max_pages)
        self.table = torch.from_numpy(self.alloc.table.copy()).to(self.device)
        self.pages = kvq.make_pages(self.pool, self.table, n_pages, page_tiles)
        self.plans = torch.zeros(cfg.n_kv_heads * kvq.PLAN_BYTES, dtype=torch.uint8,
                                 device=self.device)
        self.plan_ptrs = kvq.ptr_array([self.plans] * batch, self.device)
        self.lens = torch.zeros(batch, dtype=torch.int32, device=self.device)
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.plans_host = None

    @property
    def table_host(self):
        return self.alloc.table

    @property
    def cap(self) -> int:
        return self.alloc.table.shape[1] * self.page_tiles * 32

    # ---------------------------------------------------------- pages
    def reserve(self, seq: int, n_tokens: int, order=None):
        """Pages for the first n_tokens tokens of sequence seq; uploads the table."""
        self.alloc.reserve(seq, n_tokens, order)
        self.table.copy_(torch.from_numpy(self.alloc.table))

    def release(self, seq: int):
        """Return a sequence's pages to the free list and empty it."""
        self.alloc.release(seq)
        self.table.copy_(torch.from_numpy(self.alloc.table))
        self.lens[seq] = 0

    # ---------------------------------------------------------- calls
    def alloc_bits(self, k):
        """Plans from keys k [T, n_kv, 128] (device), as PackedLayer.alloc_bits."""
        self.plans_host, self.energy = kvq.alloc_bits(self.cfg, self.layer, k, self.plans,
                                                      self.status)
        return self.plans_host

    def set_plans(self, plans_host: np.ndarray, check: bool = True):
        if check:
            kvq.plan_check(self.cfg, plans_host)
        raw = torch.from_numpy(np.frombuffer(plans_host.tobytes(), dtype=np.uint8).copy())
        self.plans.copy_(raw.to(self.device))
        self.plans_host = plans_host

    def append(self, k, v, rope_base=0.0):
        """k, v [batch, n_new, n_kv, 128]; the pages must have been reserved."""
        kvq.paged_quantize_append(self.cfg, self.plan_ptrs, k, v, self.pages, self.lens,
                                  self.status, rope_base)

    def decode(self, q, out=None, ws=None, max_len=None):
        max_len = self.cap if max_len is None else max_len
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=self.device)
        if ws is None:
            ws = self.workspace(q.shape[1], max_len)
        kvq.paged_decode_attn(self.cfg, self.plan_ptrs, self.pages, self.lens, max_len, q, out,
                              ws, self.status)
        return out

    def decode_partial(self, q, rec=None, ws=None, max_len=None):
        """This pool's sequences as one context shard: records [batch, n_q, 132]."""
        max_len = self.cap if max_len is None else max_len
        if rec is None:
            rec = torch.empty((q.shape[0], q.shape[1], kvq.REC_FLOATS), dtype=torch.float32,
                              device=self.device)
        if ws is None:
            ws = self.workspace(q.shape[1], max_len)
        kvq.paged_decode_attn_partial(self.cfg, self.plan_ptrs, self.pages, self.lens, max_len,
                                      q, rec, ws, self.status)
        return rec

    def combine(self, recs, out=None):
        """Outputs [batch, n_q, 128] from stacked shard records [n_parts, batch, n_q, 132]."""
        if out is None:
            out = torch.empty(recs.shape[1:3] + (128,), dtype=torch.float32, device=self.device)
        kvq.combine_partials(self.cfg, self.plan_ptrs, recs, out)
        return out

    def decode_sharded(self, q, group=None, max_len=None):
        """Context-sharded decode over ranks (this rank's pool holds its range)."""
        return sharded_decode(lambda: self.decode_partial(q, max_len=max_len), self.combine, group)

    def append_decode(self, k, v, q, out=None, ws=None, max_len=None, step_flags=0,
                      rope_base=0.0):
        max_len = self.cap if max_len is None else max_len
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=self.device)
        if ws is None:
            ws = self.workspace(q.shape[1], max_len)
        kvq.paged_append_decode(self.cfg, self.plan_ptrs, k, v, self.pages, self.lens, max_len,
                                q, out, ws, self.status, step_flags, rope_base)
        return out

    def workspace(self, n_q: int, max_len: int):
        n = kvq.decode_workspace_bytes(self.cfg, self.batch, n_q, max_len)
        return torch.zeros(n, dtype=torch.uint8, device=self.device)

    def head_records(self, seq: int, head: int, n_tiles: int) -> np.ndarray:
        """Tile records [n_tiles, tile_bytes / 4] of one head, gathered
        through the block table (host)."""
        tb = kvq.tile_bytes(self.cfg)
        n_kv = self.cfg.n_kv_heads
        pool = self.pool.cpu().numpy().reshape(self.n_pages, self.page_tiles, n_kv, tb)
        out = np.empty((n_tiles, tb), dtype=np.uint8)
        for t in range(n_tiles):
            g = self.table_host[seq, t // self.page_tiles]
            out[t] = pool[g, t % self.page_tiles, head]
        return out.view("<u4").reshape(n_tiles, tb // 4)

    def flags(self) -> int:
        return int(self.status.item()) & 0xFFFFFFFF
