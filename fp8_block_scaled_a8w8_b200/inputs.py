"""Seeded synthetic inputs and the workload list.

This module only draws random numbers and names shapes; it holds none of the
GEMM's or the quantisers' arithmetic, so both the CUDA path and the CPU oracle
may use it. Shapes are the ones the pages measure: the Qwen3.8-27B decode
projections of [aiter#7752] "Kernel" (o_proj/out_proj N=5120 K=6144, qkv
14336x5120, in_proj_qkvz 16384x5120, gate_up 34816x5120), the dense prefill M
that chunked prefill produces ([cookbook#8]: M up to 8192, M=6016), and the
small-N BF16 router/indexer GEMMs of [cookbook#8] and [aiter#7247]
"Technical Details". No dataset is read; all values are synthetic.

Recipe (every draw uses numpy's default_rng (PCG64)):
  activations  A ~ N(0, 1) drawn in float32, optionally 1% of the K channels
               (rng.choice(K, K // 100, replace=False)) multiplied by 20, then
               rounded to bfloat16 (torch's RN-even cast);
  weights      W ~ N(0, sigma) in float32, sigma = 0.02;
  raw codes    uniform random e4m3 codes that are finite (0x7F/0xFF excluded);
  raw scales   uniform in [2^e, 2^(e+1)), e uniform in {-10..-2}, float32.
"""

from __future__ import annotations

import numpy as np
import torch

SIGMA_W = 0.02

# (N, K) of the decode / prefill projections.
DECODE_NK = [(5120, 6144), (14336, 5120), (16384, 5120), (34816, 5120)]
DECODE_MS = [1, 2, 3, 4, 8, 9, 16]
PREFILL_NK = [(14336, 5120), (34816, 5120)]
PREFILL_MS = [2048, 6016, 8192]
LADDER_NK = (5120, 6144)
# small-N bf16 GEMMs: (N, K, fp32 output?)
BF16_NK = [(256, 6144, False), (32, 6144, False), (384, 5120, False), (1024, 5120, True), (128, 512, False)]
BF16_MS = [1, 32, 576, 4096, 16384]
# the MX32 (32x32 E8M0 scale block) GEMMs of [aiter#7247] "Technical Details" and its
# microbenchmark table: dense (N, K) at M = 48 and 768, batched b = 8 (1024, 4096) at M = 16
MX32_NK = [(1792, 5120), (4608, 5120), (5120, 2304), (5120, 8192), (32768, 1280)]
MX32_MS = [48, 768]
MX32_BATCHED = (8, 1024, 4096)
MX32_BATCHED_MS = [16, 64]
# the fused residual add + RMSNorm + quantisation step feeding the decode / prefill GEMMs
NORM_KS = [5120, 6144]
NORM_MS = [1, 16, 2048, 8192]
# the target lm_head of [aiter#7247] "Technical Details" / microbenchmark table (bf16 out)
LM_HEAD_NK = (32320, 5120)
LM_HEAD_MS = [24, 384, 1536, 2304, 3072]

WORKLOADS = {
    "decode_m1_n5120_k6144": "single a8w8 blockscale GEMM M=1, N=5120, K=6144, seed 0",
    "decode_sweep": "a8w8 blockscale decode sweep, M in {1,2,3,4,8,9,16} x (N,K) in "
                    "{(5120,6144),(14336,5120),(16384,5120),(34816,5120)}, weights rotated over >= 512 MiB",
    "prefill": "a8w8 blockscale prefill, M in {2048,6016,8192} x (N,K) in {(14336,5120),(34816,5120)}, "
               "1% outlier channels x20",
    "ladder": "a8w8 blockscale dense M ladder, 512 M drawn from 1..8192 on (N,K)=(5120,6144)",
    "bf16_small_n": "bf16 x bf16 small-N GEMMs, M in {1,32,576,4096,16384} x (N,K) in "
                    "{(256,6144),(32,6144),(384,5120),(1024,5120) fp32 out,(128,512)}",
    "mx32": "MX32 a8w8 GEMM (E8M0 scales, 1x32 / 32x32 blocks), M in {48,768} x (N,K) in "
            "{(1792,5120),(4608,5120),(5120,2304),(5120,8192),(32768,1280)}, weights rotated over >= 512 MiB",
    "mx32_batched": "batched MX32 a8w8 GEMM, b=8, (N,K)=(1024,4096), M in {16,64}, weights rotated over >= 512 MiB",
    "add_rmsnorm_quant": "fused residual add + RMSNorm + 1x128 fp8 quantisation, M in {1,16,2048,8192} x "
                         "K in {5120,6144}",
    "lm_head": "bf16 x bf16 large-N lm_head GEMM, M in {24,384,1536,2304,3072} on (N,K)=(32320,5120), bf16 out",
}


def decode_seed_w(nk_index: int) -> int:
    return 100 + nk_index


def decode_seed_a(nk_index: int, m_index: int) -> int:
    return 200 + 10 * nk_index + m_index


def activation_bf16(M: int, K: int, seed: int, outliers: bool = False) -> torch.Tensor:
    """[M, K] bfloat16 CPU tensor."""
    rng = np.random.default_rng(seed)
    a = rng.standard_normal((M, K), dtype=np.float32)
    if outliers:
        ch = rng.choice(K, K // 100, replace=False)
        a[:, ch] *= np.float32(20.0)
    return torch.from_numpy(a).to(torch.bfloat16)


def weight_f32(N: int, K: int, seed: int, sigma: float = SIGMA_W) -> torch.Tensor:
    """[N, K] float32 CPU tensor."""
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((N, K), dtype=np.float32)
    w *= np.float32(sigma)
    return torch.from_numpy(w)


def weight_bf16(N: int, K: int, seed: int, sigma: float = SIGMA_W) -> torch.Tensor:
    return weight_f32(N, K, seed, sigma).to(torch.bfloat16)


def m1_n5120_k6144(seed: int = 0):
    """Single GEMM M=1, N=5120, K=6144: one generator, A drawn first, then W."""
    M, N, K = 1, 5120, 6144
    rng = np.random.default_rng(seed)
    a = rng.standard_normal((M, K), dtype=np.float32)
    w = rng.standard_normal((N, K), dtype=np.float32) * np.float32(SIGMA_W)
    return torch.from_numpy(a).to(torch.bfloat16), torch.from_numpy(w)


def ladder_ms(seed: int = 3, count: int = 512, max_m: int = 8192) -> list:
    rng = np.random.default_rng(seed)
    ms = rng.choice(np.arange(1, max_m + 1), size=count, replace=False)
    return sorted(int(m) for m in ms)


def random_e4m3_codes(shape, seed: int, max_code: int = 0x7E) -> np.ndarray:
    """Uniform finite e4m3 codes with magnitude code <= max_code (0x7E = 448)."""
    rng = np.random.default_rng(seed)
    mag = rng.integers(0, max_code + 1, size=shape, dtype=np.int64)
    sign = rng.integers(0, 2, size=shape, dtype=np.int64) << 7
    return (mag | sign).astype(np.uint8)


def random_scales(shape, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    mant = rng.uniform(0.5, 1.0, size=shape)
    e = rng.integers(-10, -1, size=shape)
    return np.ldexp(mant, e + 1).astype(np.float32)
