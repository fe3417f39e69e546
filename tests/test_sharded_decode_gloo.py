"""Context-sharded decode, host side, on CPU: two and three gloo ranks.

Each rank holds one token range of the same sequences; its records go
through runtime.sharded_decode's all-gather (rank order) and are combined.
The per-rank records and the combine are the oracle's here (no GPU), in the
library's record format (m, l, -, -, o): with m = lse2 and l = 1, 2^m l is
the range's sum of 2^s and 2^m o its weighted value sum. The result must be
attention over the whole context on every rank.
"""
import os
import sys

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
T, N_KV, G = 200, 2, 4


def _inputs():
    rng = np.random.default_rng(9)
    q = rng.standard_normal((N_KV * G, 128)) * 1.5
    k = rng.standard_normal((T, N_KV, 128))
    v = rng.standard_normal((T, N_KV, 128))
    return q, k, v


def _oracle_combine(recs):
    from oracle import attn
    r = recs.numpy()[:, 0]                  # [world, n_q, 132], batch of one
    with np.errstate(divide="ignore"):
        lse = r[:, :, 0] + np.log2(r[:, :, 1])
    out = np.zeros((N_KV * G, 128))
    for h in range(N_KV):
        sl = slice(h * G, (h + 1) * G)
        out[sl] = attn.combine_ranges(lse[:, sl], r[:, sl, 4:])
    return torch.from_numpy(out)[None]


def _worker(rank, world, port, cuts, out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from oracle import attn
    from bit_kv_cache_19_b200 import runtime

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v = _inputs()
        a, b = cuts[rank], cuts[rank + 1]

        def partial():
            rec = np.zeros((1, N_KV * G, 132))
            for h in range(N_KV):
                sl = slice(h * G, (h + 1) * G)
                lse, o = attn.range_record(q[sl], k[a:b, h], v[a:b, h])
                rec[0, sl, 0] = lse
                rec[0, sl, 1] = np.where(lse == -np.inf, 0.0, 1.0)
                rec[0, sl, 4:] = o
            return torch.from_numpy(rec)

        out[rank] = runtime.sharded_decode(partial, _oracle_combine).numpy()
    finally:
        dist.destroy_process_group()


def _run(cuts, port):
    world = len(cuts) - 1
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, cuts, out), nprocs=world,
                       start_method="spawn", join=True)
    return [out[r] for r in range(world)]


def test_two_ranks_combine_to_whole_context():
    from oracle import attn
    q, k, v = _inputs()
    ref = attn.decode(q, [k[:, h] for h in range(N_KV)], [v[:, h] for h in range(N_KV)])
    for cuts, port in (([0, 123, T], 29531), ([0, 0, T], 29532)):
        got = _run(cuts, port)
        for g in got:
            assert np.max(np.abs(g[0] - ref)) < 1e-12


def test_three_ranks_with_ragged_ranges():
    from oracle import attn
    q, k, v = _inputs()
    ref = attn.decode(q, [k[:, h] for h in range(N_KV)], [v[:, h] for h in range(N_KV)])
    got = _run([0, 33, 34, T], 29533)
    for g in got:
        assert np.max(np.abs(g[0] - ref)) < 1e-12
