"""The C ABI from plain C (no Python, no torch): a host-only program is
compiled with gcc against include/kvq.h, linked to the in-tree libkvq.so and
run on the CPU; its printed facts are checked against the Python binding and
the oracle."""
import os
import shutil
import subprocess

import numpy as np
import pytest

from bit_kv_cache_19_b200 import kvq
from oracle import lloydmax

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_host_abi_from_c(tmp_path):
    kvq.lib()  # raises if the library was not built
    exe = tmp_path / "kvq_host_abi"
    libdir = os.path.dirname(kvq.LIB_PATH)
    subprocess.run(["gcc", "-O1", "-std=c99", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "kvq_host_abi.c"), "-L", libdir, "-lkvq",
                    f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    facts = {line.split()[0]: line.split()[1:] for line in out.splitlines() if line.strip()}
    cfg = kvq.make_cfg(2, 3, 3, v_seed=7)
    assert facts["version"][0] == "kvq"
    assert int(facts["plan_bytes"][0]) == kvq.PLAN_BYTES
    assert int(facts["tile_bytes"][0]) == kvq.tile_bytes(cfg) == 32 * 100
    assert int(facts["cache_bytes_128k"][0]) == kvq.cache_bytes(cfg, 131072)
    assert int(facts["page_bytes_16"][0]) == 16 * 2 * 3200
    c0, t3, d3 = (float(x) for x in facts["codebook3"])
    assert c0 == pytest.approx(float(lloydmax.centroids(3)[0]), abs=1e-6)
    assert t3 == pytest.approx(float(lloydmax.thresholds(3)[3]), abs=1e-6)
    assert d3 == pytest.approx(0.03454, abs=1e-5)
    assert int(facts["plan_width_sum"][0]) == 64 * 3
    assert int(facts["corrupt_plan_check"][0]) == kvq.ERR_ARG
    assert "width" in " ".join(facts["corrupt_plan_check"][1:])
    assert int(facts["head_dim_64"][0]) == kvq.ERR_UNSUPPORTED
