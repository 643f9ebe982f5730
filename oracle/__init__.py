"""CPU oracle for the a8w8 block-scaled FP8 GEMM path -- TEST INFRASTRUCTURE ONLY.

This package is the slow, plain, obviously-correct restatement of what the
GPU path computes. It exists to check the CUDA kernels, never to stand in for
them: only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import it. The product package
``fp8_block_scaled_a8w8_b200`` never imports it and shares no code with it
(the only shared module is the seeded input generator
``fp8_block_scaled_a8w8_b200.inputs``, which holds none of the method's
arithmetic).

Everything is numpy in float64 unless a step is defined in a narrower type
(the activation quantiser works in IEEE float32, as the kernel must, so that
the fp8 codes can be compared bit for bit).

Sources (web pages, cited by title and section):

* [cookbook#8] "Why aiter#5069's measured -25% kernel win moved serving
  throughput by 0.0%" (sglang-amd-cookbook PR #8): GLM-5.2-FP8 is block
  quantised with ``weight_block_size: [128,128]`` and so takes
  ``gemm_a8w8_blockscale*``; the tuned lookup walks exact M -> size band ->
  nextPow2 -> give up (M=6016 runs the 8192 row); the coverage census counts
  hits/misses deduplicated by (M, N, K, table, padded_M, library).
* [aiter#7752] "[Perf] Retune gfx942 Qwen3.8-27B a8w8 blockscale decode rows
  for cold weights" (ROCm/aiter PR #7752), sections "Kernel" and
  "PR-specific question": the decode shapes, the getPaddedM walk, relative L2
  against an fp32 reference of 1.7e-3 (bf16 output-rounding floor) vs 2.5e-3
  with split-K bf16 atomics.
* [aiter#7247] ROCm/aiter PR #7247 (gfx1250 DSv4.1 tuned rows), "Test Result":
  error ratio = fraction of outputs outside tolerance against a reference GEMM.

Modules:
  e4m3      -- OCP FP8 E4M3 codec from the bit-level format definition
  bf16      -- round-to-nearest-even to bfloat16 from float64
  quant     -- per-token 1x128 activation quantiser, 128x128 weight quantiser
  gemm      -- a8w8 block-scaled GEMM and plain bf16 GEMM in float64
  metrics   -- relative L2, error ratio, bf16 ulp
  norm      -- fused residual add + RMSNorm + activation quantisation
  mx        -- MX32 variant: E8M0 scales, 1x32 activation groups, 32x32 weight blocks
  dispatch  -- the padded-M lookup walk and the census deduplication rule

Parity status of every function is listed in each module's header; every
function here is pinned by a ``-m "not gpu"`` test in ``tests/test_oracle_*.py``
against something other than itself.
"""

from . import e4m3, bf16, quant, gemm, metrics, dispatch, norm, mx  # noqa: F401
