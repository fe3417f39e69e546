"""The C ABI on the GPU from plain C (no Python, no torch in the process that
computes): tests/c/kvq_device_abi.c allocates with cudaMalloc and runs
kvq_alloc_bits -> kvq_quantize_append -> kvq_decode_attn on one sequence.
Its plans must equal the oracle's and its outputs the fp64 oracle within
2e-3."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle_pipeline as op
import synth
from bit_kv_cache_19_b200 import kvq
from test_gpu_parity import check_plan

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")
TOL = 2e-3


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_device_abi_from_c(tmp_path):
    kvq.lib()  # raises if the library was not built
    exe = tmp_path / "kvq_device_abi"
    libdir = os.path.dirname(kvq.LIB_PATH)
    subprocess.run(["gcc", "-O1", "-std=c99", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(CUDA, "include"),
                    os.path.join(ROOT, "tests", "c", "kvq_device_abi.c"), "-L", libdir, "-lkvq",
                    "-L", os.path.join(CUDA, "lib64"), "-lcudart", f"-Wl,-rpath,{libdir}",
                    f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}", "-o", str(exe)], check=True)
    n_kv, bits_k, bits_v, T, G, v_seed = 2, 3, 3, 1000, 8, 9
    rng = np.random.default_rng(41)
    E0 = np.exp(rng.standard_normal((n_kv, 64)) - np.arange(64) / 8.0)
    sig = np.sqrt(np.concatenate([E0, E0], axis=1) / 2)
    kb = synth.to_bf16_bits(rng.standard_normal((T, n_kv, 128)) * sig[None])
    vb = synth.to_bf16_bits(rng.standard_normal((T, n_kv, 128)))
    qb = synth.to_bf16_bits(rng.standard_normal((n_kv * G, 128)))
    inp, outp = tmp_path / "in.bin", tmp_path / "out.bin"
    with open(inp, "wb") as f:
        f.write(np.array([n_kv, bits_k, bits_v, T, n_kv * G, v_seed], dtype=np.int32).tobytes())
        f.write(kb.tobytes())
        f.write(vb.tobytes())
        f.write(qb.tobytes())
    r = subprocess.run([str(exe), str(inp), str(outp)], capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.stdout, r.stderr)
    raw = open(outp, "rb").read()
    res = np.frombuffer(raw[:20], dtype=np.int32)
    assert list(res) == [kvq.OK, kvq.OK, kvq.OK, 0, T]
    out = np.frombuffer(raw[20:20 + n_kv * G * 512], dtype=np.float32).reshape(n_kv * G, 128)
    plans = np.frombuffer(raw[20 + n_kv * G * 512:], dtype=kvq.PLAN_DTYPE)
    kh, vh = op.bf16_heads(kb, vb)
    E, heads = op.layer(kh, vh, bits_k, bits_v, v_seed, 0, pack=False)
    for h in range(n_kv):
        check_plan(plans[h], heads[h]["plan"])
    ref = op.decode(synth.bf16_bits_to_f64(qb), heads)
    assert op.rel_err(out, ref) <= TOL
