"""Host logic of the multi-GPU bench on CPU: two gloo ranks (world size 2).

The path shards by (sequence, layer, KV head) with no data exchange, so
bench.py runs one replica per GPU; what crosses ranks is only the timing:
the job's time is the max over ranks and the value counts every rank's
units. The reference arm runs on rank 0 alone.
"""
import io
import os
import sys
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # a per-rank time: the slowest rank's is the job's
        t = bench.rank_max(1.5 + rank, dist)
        # weak scaling: every rank processed the same units
        rate = bench.job_rate(1000.0, world, t)
        seeds = [bench.rank_seed(3, rank, b) for b in range(4)]
        # the reference arm prints on rank 0 only (its work is stubbed here)
        buf = io.StringIO()
        orig = bench.oracle_sample
        bench.oracle_sample = lambda wl, seconds_target, seed: {
            "value": 1.0, "cores": 1, "sample": "stub", "seconds": 0.0}
        try:
            with redirect_stdout(buf):
                args = type("A", (), {"steps": 2, "warmup": 1, "seed": 0})()
                bench.run_reference(args, bench.synth.WORKLOADS["tiny"], rank, world)
        finally:
            bench.oracle_sample = orig
        dist.barrier()
        out[rank] = (t, rate, seeds, buf.getvalue())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_max_value_sum_reference_rank0():
    world, port = 2, 29517
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn",
                       join=True)
    (t0, r0, s0, p0), (t1, r1, s1, p1) = out[0], out[1]
    assert t0 == t1 == 2.5
    assert r0 == r1 == pytest.approx(2 * 1000.0 / 2.5e-3)
    assert not set(s0) & set(s1)          # ranks hold different sequences
    assert '"impl": "reference"' in p0 and '"n_gpus": 2' in p0
    assert p1 == ""                       # other ranks exit without work


def test_single_process_helpers():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.rank_max(4.0, None) == 4.0
    assert bench.job_rate(10.0, 1, 1.0) == pytest.approx(1e4)


def test_percentiles_and_code_hash():
    sys.path.insert(0, ROOT)
    import bench

    st = bench.percentiles([5.0, 1.0, 3.0, 2.0, 4.0])
    assert (st["n"], st["min"], st["p50"], st["max"]) == (5, 1.0, 3.0, 5.0)
    assert st["mean"] == pytest.approx(3.0)
    # the traffic record is keyed by code, not comments or layout
    a = "int f(int x) {  // one\n  /* two\n three */ return x + 1;\n}\n"
    b = "int f(int x) {\n\n  return x + 1;   // other words\n}"
    c = "int f(int x) { return x + 2; }"
    assert bench.code_only(a) == bench.code_only(b) != bench.code_only(c)
    assert len(bench.decode_source_hash()) == 16
