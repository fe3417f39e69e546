"""Plain, slow CPU oracle for RoPE-aware packed KV-cache quantization.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it. The
product path (``bit_kv_cache_19_b200`` and its CUDA library) never imports,
links or runs anything here, and this package imports nothing from the product.

Source of the method: "RoPE-Aware Bit Allocation for KV-Cache Quantization"
(Block-GTQ), abstract. The abstract states the method in prose only: per
(layer, KV head) label-free energy of each RoPE 2-D block, greedy integer bit
allocation by marginal gain under a matched K/V budget, quantization built on
TurboQuant-MSE, and a packed-cache decode path. Every piece it leaves open is
fixed here as a recorded reading (energy formula, distortion model, codebooks,
norm, packing layout); each module says which.

Modules (each function cites the passage it follows):

* ``lloydmax`` - Gaussian Lloyd-Max codebooks and distortion D(b).
* ``rope``     - RoPE rotation of 2-D frequency blocks and the block form of
                 the query-key logit.
* ``energy``   - label-free block energy (exact integer accumulation).
* ``alloc``    - greedy marginal-gain bit allocation and the per-head plan.
* ``splitmix`` - SplitMix64 counter generator for the value sign flips.
* ``quant``    - TQ-MSE style quantizers for keys (per-block widths) and
                 values (randomised Hadamard, uniform width), with the fp32
                 decision arithmetic written out step by step.
* ``layout``   - the packed tile record: pack and unpack.
* ``attn``     - dequantization and exact softmax attention in fp64.
* ``window``   - the recent-token window: which tokens stay exact, decode
                 over the packed and the exact tokens together.

Floating point is fp64 except where a quantization decision is taken: there
the arithmetic is IEEE fp32 in a fixed order so that codes are reproducible
bit for bit.
"""
