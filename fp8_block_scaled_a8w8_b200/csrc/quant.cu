// Activation (per token, 1x128 group) and weight (128x128 block) quantisers.
//
// scale = amax / 448 and code = e4m3_rn_satfinite(x / scale), both divisions IEEE
// float32 round-to-nearest (__fdiv_rn), the conversion the hardware
// cvt.rn.satfinite.e4m3x2.f32 -- so the codes and scales equal the CPU
// oracle's bit for bit. A group whose amax is 0 gets scale 0 and codes +-0.
// ([cookbook#8]: the checkpoint is block quantised, weight_block_size [128,128].)
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace fp8bs {

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ float quant_div(float x, float s) { return s == 0.f ? x : __fdiv_rn(x, s); }

__device__ __forceinline__ uint32_t cvt4_e4m3(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return (lo & 0xFFFFu) | (hi << 16);
}

// One half-warp per group: 16 lanes x 8 bf16 = 128 values; a warp takes two groups.
__global__ void __launch_bounds__(256) quant_act_kernel(const uint16_t* __restrict__ x, int64_t M, int64_t K,
                                                        int64_t ld_x, uint8_t* __restrict__ q,
                                                        float* __restrict__ scale) {
  pdl_trigger();
  pdl_wait();
  const int64_t G = K / 128;
  const int64_t total = M * G;
  const int lane = threadIdx.x & 31;
  const int half = lane >> 4;
  const int hl = lane & 15;
  const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  for (int64_t gp = warp * 2; gp < total; gp += nwarps * 2) {
    const int64_t gi = gp + half;
    const bool valid = gi < total;
    const int64_t m = valid ? gi / G : 0;
    const int64_t g = valid ? gi - m * G : 0;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (valid) v = ld_nc_v4(x + m * ld_x + g * 128 + hl * 8);
    float f[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                  bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
    for (int off = 8; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const float s = __fdiv_rn(amax, 448.f);
    if (valid) {
      uint2 out;
      out.x = cvt4_e4m3(quant_div(f[0], s), quant_div(f[1], s), quant_div(f[2], s), quant_div(f[3], s));
      out.y = cvt4_e4m3(quant_div(f[4], s), quant_div(f[5], s), quant_div(f[6], s), quant_div(f[7], s));
      *reinterpret_cast<uint2*>(q + m * K + g * 128 + hl * 8) = out;
      if (hl == 0) scale[m * G + g] = s;
    }
  }
}

// One CTA (256 threads) per 128x128 block; thread t owns row t/2, 64 columns.
__global__ void __launch_bounds__(256) quant_weight_kernel(const float* __restrict__ w, int64_t N, int64_t K,
                                                           uint8_t* __restrict__ q, float* __restrict__ scale) {
  pdl_trigger();
  pdl_wait();
  const int64_t G = K / 128;
  const int64_t nb = blockIdx.y;
  const int64_t g = blockIdx.x;
  const int t = threadIdx.x;
  const int64_t row = nb * 128 + (t >> 1);
  const int64_t col = g * 128 + (t & 1) * 64;
  const bool valid = row < N;
  float4 v[16];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    v[i] = valid ? __ldg(reinterpret_cast<const float4*>(w + row * K + col) + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)), fmaxf(fabsf(v[i].z), fabsf(v[i].w))));
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  __shared__ float red[8];
  if ((t & 31) == 0) red[t >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
  const float s = __fdiv_rn(amax, 448.f);
  if (t == 0) scale[nb * G + g] = s;
  if (!valid) return;
  uint32_t packed[16];
#pragma unroll
  for (int i = 0; i < 16; ++i)
    packed[i] = cvt4_e4m3(quant_div(v[i].x, s), quant_div(v[i].y, s), quant_div(v[i].z, s), quant_div(v[i].w, s));
  uint4* dst = reinterpret_cast<uint4*>(q + row * K + col);
#pragma unroll
  for (int i = 0; i < 4; ++i) dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
}

// Fused residual add + RMSNorm + activation quantisation (the add_rmsnorm_quant step of
// [mi210 docs/43] "43-ck-int8-gemm-gfx90a.md", Rounds 40-41, which feeds the GEMM), one
// CTA per token row:
//   h = bf16(float(x) + float(residual))          -> residual_out (may alias residual)
//   r = 1 / sqrt(sum(h^2) / K + eps)              (float32; IEEE sqrt and division)
//   y = (h * r) * gamma                           (float32)
//   q, a_scale = the 1x128 activation quantiser of y (as quant_act_kernel)
// Thread t holds the 16-byte vectors t, t + T, ... (T threads, at most kNormVpt vectors
// each), so every load of the row is in flight at once and a half-warp covers one
// 128-wide group; the sum of squares is reduced by warp shuffles and across warps in
// shared memory. y stays in registers and is quantised straight from float32.
constexpr int kNormVpt = 4;

template <int VPT>
__global__ void __launch_bounds__(1024) add_rmsnorm_quant_kernel(const uint16_t* x, const uint16_t* res,
                                                                 const uint16_t* __restrict__ gamma, float eps,
                                                                 uint16_t* res_out, uint8_t* __restrict__ q,
                                                                 float* __restrict__ scale, int64_t M, int64_t K) {
  __shared__ float warp_ss[32];
  __shared__ float s_rinv;
  pdl_trigger();
  pdl_wait();
  const int64_t row = blockIdx.x;
  const int T = blockDim.x, t = threadIdx.x, lane = t & 31, w = t >> 5;
  const int64_t nv = K / 8;
  const int64_t base = row * K;
  float f[VPT][8];
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int64_t v = t + int64_t(j) * T;
#pragma unroll
    for (int i = 0; i < 8; ++i) f[j][i] = 0.f;
    if (v < nv) {
      // plain loads: residual and residual_out may be the same buffer
      const uint4 xa = *reinterpret_cast<const uint4*>(x + base + 8 * v);
      const uint4 ra = *reinterpret_cast<const uint4*>(res + base + 8 * v);
      const uint32_t xw[4] = {xa.x, xa.y, xa.z, xa.w}, rw[4] = {ra.x, ra.y, ra.z, ra.w};
      uint32_t hw[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(__fadd_rn(bf16_lo(xw[i]), bf16_lo(rw[i])),
                                                        __fadd_rn(bf16_hi(xw[i]), bf16_hi(rw[i])));
        hw[i] = *reinterpret_cast<const uint32_t*>(&h2);
        f[j][2 * i] = bf16_lo(hw[i]);
        f[j][2 * i + 1] = bf16_hi(hw[i]);
        ss = __fmaf_rn(f[j][2 * i], f[j][2 * i], ss);
        ss = __fmaf_rn(f[j][2 * i + 1], f[j][2 * i + 1], ss);
      }
      *reinterpret_cast<uint4*>(res_out + base + 8 * v) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    }
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, off));
  if (lane == 0) warp_ss[w] = ss;
  __syncthreads();
  if (t == 0) {
    float tot = 0.f;
    for (int i = 0; i < (T >> 5); ++i) tot = __fadd_rn(tot, warp_ss[i]);  // in warp order
    s_rinv = __fdiv_rn(1.f, __fsqrt_rn(__fadd_rn(__fdiv_rn(tot, float(K)), eps)));
  }
  __syncthreads();
  const float rinv = s_rinv;
  const int64_t G = K / 128;
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int64_t v = t + int64_t(j) * T;
    const bool valid = v < nv;
    if (valid) {
      const uint4 ga = ld_nc_v4(gamma + 8 * v);
      const uint32_t gw[4] = {ga.x, ga.y, ga.z, ga.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        f[j][2 * i] = __fmul_rn(__fmul_rn(f[j][2 * i], rinv), bf16_lo(gw[i]));
        f[j][2 * i + 1] = __fmul_rn(__fmul_rn(f[j][2 * i + 1], rinv), bf16_hi(gw[i]));
      }
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[j][i]));
#pragma unroll
    for (int off = 8; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const float s = __fdiv_rn(amax, 448.f);
    if (valid) {
      uint2 out;
      out.x = cvt4_e4m3(quant_div(f[j][0], s), quant_div(f[j][1], s), quant_div(f[j][2], s), quant_div(f[j][3], s));
      out.y = cvt4_e4m3(quant_div(f[j][4], s), quant_div(f[j][5], s), quant_div(f[j][6], s), quant_div(f[j][7], s));
      *reinterpret_cast<uint2*>(q + base + 8 * v) = out;
      if ((lane & 15) == 0) scale[row * G + v / 16] = s;
    }
  }
}

int launch_add_rmsnorm_quant(const void* x, const void* residual, const void* gamma, float eps, void* residual_out,
                             void* q, float* scale, int64_t M, int64_t K, void* stream) {
  const int64_t nv = K / 8;
  const int64_t per = (nv + 1023) / 1024;  // vectors per thread at 1024 threads
  if (per > kNormVpt || M > 0x7FFFFFFF) return int(cudaErrorInvalidValue);
  // Many rows are bound by the bytes each SM keeps in flight. One vector per thread keeps
  // three rows resident per SM while a row has at most 682 vectors (3 x 682 threads <= 2048);
  // longer rows (K = 6144: 768 threads, two rows an SM) take two vectors per thread, which
  // fits four rows under the register file (measured on a B200 at M = 2048..8192: K = 6144
  // 87.6 -> 75.6 us, while K = 5120 and small M run faster with one vector per thread).
  const int vpt = per <= 1 ? ((nv > 682 && M >= 256) ? 2 : 1) : per <= 2 ? 2 : 4;
  const int threads = int(((nv + vpt - 1) / vpt + 31) / 32 * 32);
  auto args = [&](auto kernel) {
    return launch_kernel(kernel, dim3(unsigned(M)), dim3(threads), 0, stream, static_cast<const uint16_t*>(x),
                         static_cast<const uint16_t*>(residual), static_cast<const uint16_t*>(gamma), eps,
                         static_cast<uint16_t*>(residual_out), static_cast<uint8_t*>(q), scale, M, K);
  };
  if (vpt == 1) return args(add_rmsnorm_quant_kernel<1>);
  if (vpt == 2) return args(add_rmsnorm_quant_kernel<2>);
  return args(add_rmsnorm_quant_kernel<4>);
}

// ---------------------------------------------------------------- MX32 quantisers
// MX32 variant ([aiter#7247] "Motivation": 32x32 weight scale blocks): E8M0 scales
// (value 2^(code - 127)) on 1x32 activation groups and 32x32 weight blocks. The exponent
// is the smallest that keeps the group within the e4m3 range, read exactly from the
// bits of r = amax / 448 (one IEEE float32 division): e = ceil(log2 r); code = e + 127
// clamped to [0, 254]; amax == 0 gives code 0. Codes are e4m3_rn_satfinite(x * 2^-e), an
// exact power-of-two scaling (rounded once only where the product is float32-subnormal).
__device__ __forceinline__ int mx_code_for_amax(float amax) {
  if (amax == 0.f) return 0;
  const uint32_t b = __float_as_uint(__fdiv_rn(amax, 448.f));
  const int ex = int((b >> 23) & 0xFFu);
  const uint32_t man = b & 0x7FFFFFu;
  int e;
  if (ex != 0) {
    e = ex - 127 + (man != 0 ? 1 : 0);
  } else {  // subnormal ratio: ceil(log2(man * 2^-149))
    const int top = 31 - __clz(int(man));
    e = -149 + top + ((man & ((1u << top) - 1u)) != 0 ? 1 : 0);
  }
  return min(max(e + 127, 0), 254);
}
// 2^-e as float32 for e = code - 127: its biased exponent is 254 - code (code 254 gives the
// subnormal 2^-127).
__device__ __forceinline__ float mx_inv_scale(int code) {
  const int pe = 254 - code;  // in [0, 254]
  return pe >= 1 ? __uint_as_float(uint32_t(pe) << 23) : __uint_as_float(0x00400000u);  // 2^-127 for pe == 0
}

// Activations: 4 lanes x 8 bf16 per 32-wide group (quarter-warp shuffles for the amax).
__global__ void __launch_bounds__(256) quant_act_mx32_kernel(const uint16_t* __restrict__ x, int64_t M, int64_t K,
                                                             int64_t ld_x, uint8_t* __restrict__ q,
                                                             uint8_t* __restrict__ ecode) {
  pdl_trigger();
  pdl_wait();
  const int64_t G = K / 32;
  const int64_t total = M * G;  // groups
  const int64_t tid = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nthreads = int64_t(gridDim.x) * blockDim.x;
  // thread -> (group gi = idx / 4, part = idx % 4); every lane of a quarter-warp iterates together
  for (int64_t idx = tid; idx < (total * 4 + 31) / 32 * 32; idx += nthreads) {
    const int64_t gi = idx >> 2;
    const int part = int(idx & 3);
    const bool valid = gi < total;
    const int64_t m = valid ? gi / G : 0;
    const int64_t g = valid ? gi - m * G : 0;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (valid) v = ld_nc_v4(x + m * ld_x + g * 32 + part * 8);
    float f[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                  bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const int code = mx_code_for_amax(amax);
    const float inv = mx_inv_scale(code);
    if (valid) {
      uint2 out;
      out.x = cvt4_e4m3(__fmul_rn(f[0], inv), __fmul_rn(f[1], inv), __fmul_rn(f[2], inv), __fmul_rn(f[3], inv));
      out.y = cvt4_e4m3(__fmul_rn(f[4], inv), __fmul_rn(f[5], inv), __fmul_rn(f[6], inv), __fmul_rn(f[7], inv));
      *reinterpret_cast<uint2*>(q + m * K + g * 32 + part * 8) = out;
      if (part == 0) ecode[m * G + g] = uint8_t(code);
    }
  }
}

// Weights: one warp per 32x32 block, lane = row; the block's amax is a warp maximum.
__global__ void __launch_bounds__(256) quant_weight_mx32_kernel(const float* __restrict__ w, int64_t N, int64_t K,
                                                                uint8_t* __restrict__ q, uint8_t* __restrict__ ecode) {
  pdl_trigger();
  pdl_wait();
  const int64_t G = K / 32, NB = (N + 31) / 32;
  const int lane = threadIdx.x & 31;
  const int64_t blk = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (blk >= NB * G) return;
  const int64_t nb = blk / G, g = blk - nb * G;
  const int64_t row = nb * 32 + lane;
  const bool valid = row < N;
  float4 v[8];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[i] = valid ? __ldg(reinterpret_cast<const float4*>(w + row * K + g * 32) + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)), fmaxf(fabsf(v[i].z), fabsf(v[i].w))));
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const int code = mx_code_for_amax(amax);
  const float inv = mx_inv_scale(code);
  if (lane == 0) ecode[nb * G + g] = uint8_t(code);
  if (!valid) return;
  uint32_t packed[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    packed[i] = cvt4_e4m3(__fmul_rn(v[i].x, inv), __fmul_rn(v[i].y, inv), __fmul_rn(v[i].z, inv), __fmul_rn(v[i].w, inv));
  uint4* dst = reinterpret_cast<uint4*>(q + row * K + g * 32);
  dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
}

int launch_quant_act_mx32(const void* x, int64_t M, int64_t K, int64_t ld_x, void* q, void* ecode, void* stream) {
  const int64_t threads_needed = M * (K / 32) * 4;
  const int64_t cap = int64_t(device_sm_count()) * 8;
  const int blocks = int(std::min<int64_t>((threads_needed + 255) / 256, cap));
  return launch_kernel(quant_act_mx32_kernel, dim3(std::max(blocks, 1)), dim3(256), 0, stream,
                       static_cast<const uint16_t*>(x), M, K, ld_x, static_cast<uint8_t*>(q),
                       static_cast<uint8_t*>(ecode));
}

int launch_quant_weight_mx32(const float* w, int64_t N, int64_t K, void* q, void* ecode, void* stream) {
  const int64_t blocks = ((N + 31) / 32) * (K / 32);  // one warp each, 8 per CTA
  return launch_kernel(quant_weight_mx32_kernel, dim3(unsigned((blocks + 7) / 8)), dim3(256), 0, stream, w, N, K,
                       static_cast<uint8_t*>(q), static_cast<uint8_t*>(ecode));
}

int launch_quant_act(const void* x, int64_t M, int64_t K, int64_t ld_x, void* q, float* scale, void* stream) {
  const int64_t groups = M * (K / 128);
  const int64_t need = (groups + 15) / 16;  // 16 groups per 256-thread block per pass
  const int64_t cap = int64_t(device_sm_count()) * 8;
  const int blocks = int(need < cap ? need : cap);
  return launch_kernel(quant_act_kernel, dim3(blocks), dim3(256), 0, stream, static_cast<const uint16_t*>(x), M, K,
                       ld_x, static_cast<uint8_t*>(q), scale);
}

int launch_quant_weight(const float* w, int64_t N, int64_t K, void* q, float* scale, void* stream) {
  dim3 grid(unsigned(K / 128), unsigned((N + 127) / 128));
  return launch_kernel(quant_weight_kernel, grid, dim3(256), 0, stream, w, N, K, static_cast<uint8_t*>(q), scale);
}

}  // namespace fp8bs

namespace fp8bs {

// ---------------------------------------------------------------- tiled weight layout
// The e4m3 weight [N, K] rearranged into 16 KiB tiles, one per (128-row block b, 128-wide
// K group g), tile (b, g) at byte (b * G + g) * 16384; inside a tile row r's 128 bytes sit
// in the 128-byte-swizzled order the tensor core's K-major shared-memory operand uses
// (16-byte chunk c of row r at chunk c ^ (r % 8)). So a tile is one contiguous copy that
// lands in shared memory ready for the MMA -- the role of the pages' pre-shuffled B
// ("bpreshuffle", [aiter#7247]), for this hardware. Rows past N and the padding block that
// makes the block count even are zero. One CTA per tile, 256 threads, 4 x 16 bytes each.
__global__ void __launch_bounds__(256) tile_weight_kernel(const uint8_t* __restrict__ w, int64_t N, int64_t K,
                                                          uint8_t* __restrict__ wt) {
  pdl_trigger();
  pdl_wait();
  const int64_t G = K / 128;
  const int64_t tile = blockIdx.x;
  const int64_t b = tile / G, g = tile - b * G;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int ci = threadIdx.x + 256 * k;  // destination 16-byte chunk of the tile
    const int r = ci >> 3, c = (ci & 7) ^ (r & 7);
    const int64_t row = b * 128 + r;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (row < N) v = ld_nc_v4(w + row * K + g * 128 + c * 16);
    *reinterpret_cast<uint4*>(wt + tile * 16384 + ci * 16) = v;
  }
}

size_t tiled_weight_bytes(int64_t N, int64_t K) {
  const int64_t nblk = (N + 127) / 128;
  return size_t((nblk + 1) / 2 * 2) * size_t(K / 128) * 16384;
}

int launch_tile_weight(const void* w, int64_t N, int64_t K, void* wt, void* stream) {
  const int64_t nblk_pad = ((N + 127) / 128 + 1) & ~int64_t(1);
  const int64_t tiles = nblk_pad * (K / 128);
  if (tiles >= (int64_t(1) << 31)) return int(cudaErrorInvalidValue);
  return launch_kernel(tile_weight_kernel, dim3(unsigned(tiles)), dim3(256), 0, stream,
                       static_cast<const uint8_t*>(w), N, K, static_cast<uint8_t*>(wt));
}

}  // namespace fp8bs
