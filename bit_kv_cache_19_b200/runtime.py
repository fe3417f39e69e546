"""Device-memory plumbing around libkvq (PyTorch tensors; no compute here).

``PackedLayer`` owns, for one layer and a batch of sequences, the plan
records, the packed caches, their pointer arrays, the lengths and the status
word, and forwards to the C-ABI calls; ``sharded_decode`` is the one
exchange step of a decode whose context is split over ranks.
"""
from __future__ import annotations

import numpy as np
import torch

from . import kvq


class PackedLayer:
    def __init__(self, cfg, batch: int, cap_tokens: int, device="cuda", layer: int = 0):
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

    # -------------------------------------------------------------- calls
    def alloc_bits(self, k):
        """Plans from keys k [T, n_kv, 128] (device)."""
        self.plans_host, self.energy = kvq.alloc_bits(self.cfg, self.layer, k, self.plans,
                                                      self.status)
        return self.plans_host

    def set_plans(self, plans_host: np.ndarray):
        """Use host plan records (e.g. from kvq.plan_build)."""
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
