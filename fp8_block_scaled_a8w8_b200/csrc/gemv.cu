// Weight-streaming split-K GEMM for small M (decode): the cost is reading W from HBM
// once ([aiter#7752] "[Perf] Retune gfx942 Qwen3.8-27B a8w8 blockscale decode rows for
// cold weights": in a decode step the weights come from HBM), and the whole GPU must
// take part even at M = 1 ([mi210 docs/43] section 3: at M = 1 a tile heuristic that
// emits too few workgroups leaves most of the card idle).
//
// Work split ("stream-K"): W is cut into units of 16 rows x one 128-wide K group (2 KB
// of e4m3; for bf16, 16 rows x 64 columns). Units are ordered tile-major (all groups
// of rows 0..15, then rows 16..31, ...) and the active warps take equal contiguous
// ranges of them, so every warp streams the same number of bytes whatever the shape.
// A warp that covers a whole 16-row tile writes its output directly; a tile shared by
// several warps is finished by the last one to arrive (an atomic counter per tile), which
// sums the others' float32 partials in warp order -- a fixed order, so results are
// bit-reproducible -- writes the output, and zeroes the partials it read and the tile's
// counter, so the whole workspace is zero-filled again when the kernel ends.
//
// Math: swap-AB mma.sync.m16n8k32 (e4m3 -> f32): 16 W rows are the MMA's M, up to 8
// tokens its N. Inside one MMA the 32 k positions may be matched between A and B in any
// consistent order, so each thread feeds raw 16-byte loads straight into fragments:
// lane (gid, tig) loads W rows gid and gid+8 and token gid at k = base + c*64 + tig*16,
// and MMA (c, h) takes bytes 8h..8h+7 of those loads. Each group's four MMAs land in a
// fresh float32 fragment that is then scaled by a_scale[token, g] * w_scale[row/128, g]
// and added to the running sum, the block-scale definition term by term.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace fp8bs {

constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = kGemvThreads / 32;

struct GemvArgs {
  const uint8_t* A;        // [M, K] e4m3 (or bf16 bytes)
  const float* a_scale;    // [M, G]
  const uint8_t* W;        // [N, K]
  const float* w_scale;    // [ceil(N/128), G]
  void* out;               // [M, N] bf16 or f32
  int M, N, K;
  int row_bytes;           // K * element size
  int groups;              // units per 16-row tile
  int n_active_warps;
  float* part;             // [2 * n_active_warps][NB * 4 * 32]
  unsigned* counter;       // [N / 16]
  int out_fp32;
};

__device__ __forceinline__ int64_t warp_of_unit(int64_t u, int64_t U, int64_t W) { return ((u + 1) * W - 1) / U; }

template <bool kFp8, int NB>
__device__ __forceinline__ void store_out(const GemvArgs& p, int t, int lane, const float (&acc)[NB][4]) {
  const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
  for (int nb = 0; nb < NB; ++nb)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int token = nb * 8 + 2 * tig + (i & 1);
      const int n = t * 16 + gid + (i >= 2 ? 8 : 0);
      if (token < p.M) {
        if (p.out_fp32)
          static_cast<float*>(p.out)[int64_t(token) * p.N + n] = acc[nb][i];
        else
          static_cast<__nv_bfloat16*>(p.out)[int64_t(token) * p.N + n] = __float2bfloat16_rn(acc[nb][i]);
      }
    }
}

template <bool kFp8, int NB, int D>
__global__ void __launch_bounds__(kGemvThreads) gemv_kernel(const GemvArgs p) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int w = blockIdx.x * kGemvWarps + (threadIdx.x >> 5);
  if (w >= p.n_active_warps) return;
  const int G = p.groups;
  const int64_t T = p.N >> 4;
  const int64_t U = T * G;
  const int64_t Wn = p.n_active_warps;
  const int64_t u0 = U * w / Wn, u1 = U * (w + 1) / Wn;
  const int first_tile = int(u0 / G);
  constexpr int kUnitBytes = 128;  // per row per unit

  // ---- register ring of D units in flight
  uint4 wa[D][2], wb[D][2], act[D][NB][2];
  float sa[D][NB][2], sw[D];

  // load cursor (tile, group) of the next unit to fetch
  int lt = int(u0 / G), lg = int(u0 - int64_t(lt) * G);
  auto load_unit = [&](int s) {
    const uint8_t* wr = p.W + (int64_t(lt) * 16 + gid) * p.row_bytes + lg * kUnitBytes + tig * 16;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      wa[s][c] = ld_stream_v4(wr + c * 64);
      wb[s][c] = ld_stream_v4(wr + 8 * int64_t(p.row_bytes) + c * 64);
    }
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const int token = nb * 8 + gid;
#pragma unroll
      for (int c = 0; c < 2; ++c)
        act[s][nb][c] = token < p.M ? ld_nc_v4(p.A + int64_t(token) * p.row_bytes + lg * kUnitBytes + tig * 16 + c * 64)
                                    : make_uint4(0, 0, 0, 0);
      if (kFp8) {
        const int t0 = nb * 8 + 2 * tig;
        sa[s][nb][0] = t0 < p.M ? __ldg(p.a_scale + int64_t(t0) * G + lg) : 0.f;
        sa[s][nb][1] = t0 + 1 < p.M ? __ldg(p.a_scale + int64_t(t0 + 1) * G + lg) : 0.f;
      }
    }
    if (kFp8) sw[s] = __ldg(p.w_scale + int64_t(lt >> 3) * G + lg);
    if (++lg == G) {
      lg = 0;
      ++lt;
    }
  };

  float acc[NB][4];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[nb][i] = 0.f;

#pragma unroll
  for (int s = 0; s < D; ++s)
    if (u0 + s < u1) load_unit(s);

  int ct = int(u0 / G), cg = int(u0 - int64_t(ct) * G);  // compute cursor
  for (int64_t ub = u0; ub < u1; ub += D) {
#pragma unroll
    for (int s = 0; s < D; ++s) {
      const int64_t u = ub + s;
      if (u < u1) {
        // ---- math for unit u (slot s)
        if (kFp8) {
          float d[NB][4];
#pragma unroll
          for (int nb = 0; nb < NB; ++nb)
#pragma unroll
            for (int i = 0; i < 4; ++i) d[nb][i] = 0.f;
#pragma unroll
          for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint32_t a0 = h ? wa[s][c].z : wa[s][c].x, a2 = h ? wa[s][c].w : wa[s][c].y;
              const uint32_t a1 = h ? wb[s][c].z : wb[s][c].x, a3 = h ? wb[s][c].w : wb[s][c].y;
#pragma unroll
              for (int nb = 0; nb < NB; ++nb) {
                const uint32_t b0 = h ? act[s][nb][c].z : act[s][nb][c].x;
                const uint32_t b1 = h ? act[s][nb][c].w : act[s][nb][c].y;
                mma_e4m3_16832(d[nb], a0, a1, a2, a3, b0, b1);
              }
            }
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            const float s0 = sa[s][nb][0] * sw[s], s1 = sa[s][nb][1] * sw[s];
            acc[nb][0] = fmaf(d[nb][0], s0, acc[nb][0]);
            acc[nb][1] = fmaf(d[nb][1], s1, acc[nb][1]);
            acc[nb][2] = fmaf(d[nb][2], s0, acc[nb][2]);
            acc[nb][3] = fmaf(d[nb][3], s1, acc[nb][3]);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint32_t a0 = h ? wa[s][c].z : wa[s][c].x, a2 = h ? wa[s][c].w : wa[s][c].y;
              const uint32_t a1 = h ? wb[s][c].z : wb[s][c].x, a3 = h ? wb[s][c].w : wb[s][c].y;
#pragma unroll
              for (int nb = 0; nb < NB; ++nb) {
                const uint32_t b0 = h ? act[s][nb][c].z : act[s][nb][c].x;
                const uint32_t b1 = h ? act[s][nb][c].w : act[s][nb][c].y;
                mma_bf16_16816(acc[nb], a0, a1, a2, a3, b0, b1);
              }
            }
        }
        // ---- refill slot s with unit u + D
        if (u + D < u1) load_unit(s);

        // ---- tile boundary: flush
        const bool tile_end = (cg == G - 1) || (u == u1 - 1);
        if (tile_end) {
          const int t = ct;
          const bool full = int64_t(t) * G >= u0 && cg == G - 1;
          if (full) {
            store_out<kFp8, NB>(p, t, lane, acc);
          } else {
            const int slot = 2 * w + (t == first_tile ? 0 : 1);
            float* dst = p.part + int64_t(slot) * (NB * 4 * 32);
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
#pragma unroll
              for (int i = 0; i < 4; ++i) __stcg(dst + (nb * 4 + i) * 32 + lane, acc[nb][i]);
            __threadfence();
            __syncwarp();
            unsigned old = 0;
            if (lane == 0) old = atomicAdd(p.counter + t, 1u);
            old = __shfl_sync(0xffffffffu, old, 0);
            const int64_t wf = warp_of_unit(int64_t(t) * G, U, Wn);
            const int64_t wl = warp_of_unit(int64_t(t + 1) * G - 1, U, Wn);
            if (old == unsigned(wl - wf)) {
              __threadfence();
              float sum[NB][4];
#pragma unroll
              for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                for (int i = 0; i < 4; ++i) sum[nb][i] = 0.f;
              // contributors' partials in warp order (a fixed order), kRB warps' loads in flight
              constexpr int kRB = NB == 1 ? 8 : NB == 2 ? 4 : 2;
              for (int64_t w0 = wf; w0 <= wl; w0 += kRB) {
                float v[kRB][NB][4];
                float* srcs[kRB];
#pragma unroll
                for (int j = 0; j < kRB; ++j) {
                  const int64_t ww = w0 + j;
                  const int ft = int((U * ww / Wn) / G);
                  srcs[j] = p.part + int64_t(2 * ww + (t == ft ? 0 : 1)) * (NB * 4 * 32);
#pragma unroll
                  for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                    for (int i = 0; i < 4; ++i) v[j][nb][i] = ww <= wl ? __ldcg(srcs[j] + (nb * 4 + i) * 32 + lane) : 0.f;
                }
#pragma unroll
                for (int j = 0; j < kRB; ++j) {
#pragma unroll
                  for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                    for (int i = 0; i < 4; ++i) sum[nb][i] += v[j][nb][i];
                  if (w0 + j <= wl) {
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                      for (int i = 0; i < 4; ++i)
                        __stcg(srcs[j] + (nb * 4 + i) * 32 + lane, 0.f);  // leave the workspace zero-filled
                  }
                }
              }
              store_out<kFp8, NB>(p, t, lane, sum);
              if (lane == 0) p.counter[t] = 0u;
            }
          }
#pragma unroll
          for (int nb = 0; nb < NB; ++nb)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[nb][i] = 0.f;
        }
        if (++cg == G) {
          cg = 0;
          ++ct;
        }
      }
    }
  }
}

// ---------------------------------------------------------------- host side
template <bool kFp8, int NB, int D>
static int occupancy() {
  static int occ = -1;
  static std::once_flag once;
  std::call_once(once, [] {
    int o = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, gemv_kernel<kFp8, NB, D>, kGemvThreads, 0) != cudaSuccess)
      o = 1;
    occ = std::max(1, o);
  });
  return occ;
}

static int gemv_nb(int64_t M) { return int((M + 7) / 8); }

// Warps the kernel runs with: one full wave of co-resident CTAs, but at least
// kMinUnitsPerWarp units per warp. (A small weight spread one unit per warp leaves every
// 16-row tile with dozens of contributors, and the finishing warp's sum over them, not
// the weight stream, sets the time.)
constexpr int64_t kMinUnitsPerWarp = 8;
static int64_t gemv_active_warps(int64_t units, int occ) {
  const int64_t warps = int64_t(device_sm_count()) * occ * kGemvWarps;
  return std::max<int64_t>(1, std::min(warps, units / kMinUnitsPerWarp));
}

template <bool kFp8, int NB>
static int gemv_occ_for_depth(int depth) {
  switch (depth) {
    case 2: return occupancy<kFp8, NB, 2>();
    case 3: return occupancy<kFp8, NB, 3>();
    default: return occupancy<kFp8, NB, 4>();
  }
}

template <bool kFp8>
static int gemv_occ(int nb, int depth) {
  switch (nb) {
    case 1: return gemv_occ_for_depth<kFp8, 1>(depth);
    case 2: return gemv_occ_for_depth<kFp8, 2>(depth);
    case 3: return gemv_occ_for_depth<kFp8, 3>(depth);
    default: return gemv_occ_for_depth<kFp8, 4>(depth);
  }
}

size_t gemv_workspace_bytes(int op, int64_t M, int64_t N, int64_t K, const KernelConfig& cfg) {
  const bool fp8 = op == FP8BS_OP_A8W8_BLOCKSCALE;
  const int nb = gemv_nb(M);
  const int64_t groups = fp8 ? K / 128 : K / 64;
  const int64_t units = (N / 16) * groups;
  const int occ = fp8 ? gemv_occ<true>(nb, cfg.gemv_depth) : gemv_occ<false>(nb, cfg.gemv_depth);
  const int64_t warps = gemv_active_warps(units, occ);
  return kCounterBytes + size_t(2 * warps) * nb * 4 * 32 * sizeof(float);
}

template <bool kFp8, int NB, int D>
static int launch_gemv_t(GemvArgs a, void* stream) {
  const int occ = occupancy<kFp8, NB, D>();
  const int64_t units = int64_t(a.N / 16) * a.groups;
  a.n_active_warps = int(gemv_active_warps(units, occ));
  const int blocks = (a.n_active_warps + kGemvWarps - 1) / kGemvWarps;
  return launch_kernel(gemv_kernel<kFp8, NB, D>, dim3(blocks), dim3(kGemvThreads), 0, stream, a);
}

template <bool kFp8, int NB>
static int launch_gemv_depth(const KernelConfig& cfg, const GemvArgs& a, void* stream) {
  switch (cfg.gemv_depth) {
    case 2: return launch_gemv_t<kFp8, NB, 2>(a, stream);
    case 3: return launch_gemv_t<kFp8, NB, 3>(a, stream);
    default: return launch_gemv_t<kFp8, NB, 4>(a, stream);
  }
}

template <bool kFp8>
static int launch_gemv_nb(const KernelConfig& cfg, const GemvArgs& a, void* stream) {
  if (a.N / 16 > kMaxCounters) return int(cudaErrorInvalidValue);
  switch (gemv_nb(a.M)) {
    case 1: return launch_gemv_depth<kFp8, 1>(cfg, a, stream);
    case 2: return launch_gemv_depth<kFp8, 2>(cfg, a, stream);
    case 3: return launch_gemv_depth<kFp8, 3>(cfg, a, stream);
    case 4: return launch_gemv_depth<kFp8, 4>(cfg, a, stream);
    default: return int(cudaErrorInvalidValue);
  }
}

static GemvArgs make_args(const void* A, const float* a_scale, const void* W, const float* w_scale, void* out,
                          int64_t M, int64_t N, int64_t K, void* ws, bool fp8, int out_fp32) {
  GemvArgs a{};
  a.A = static_cast<const uint8_t*>(A);
  a.a_scale = a_scale;
  a.W = static_cast<const uint8_t*>(W);
  a.w_scale = w_scale;
  a.out = out;
  a.M = int(M);
  a.N = int(N);
  a.K = int(K);
  a.row_bytes = int(fp8 ? K : 2 * K);
  a.groups = int(fp8 ? K / 128 : K / 64);
  a.counter = static_cast<unsigned*>(ws);
  a.part = reinterpret_cast<float*>(static_cast<char*>(ws) + kCounterBytes);
  a.out_fp32 = out_fp32;
  return a;
}

int launch_gemv_a8w8(const KernelConfig& cfg, const void* A, const float* a_scale, const void* W,
                     const float* w_scale, void* out, int64_t M, int64_t N, int64_t K, void* ws, void* stream) {
  return launch_gemv_nb<true>(cfg, make_args(A, a_scale, W, w_scale, out, M, N, K, ws, true, 0), stream);
}

int launch_gemv_bf16(const KernelConfig& cfg, const void* A, const void* W, void* out, int out_fp32, int64_t M,
                     int64_t N, int64_t K, void* ws, void* stream) {
  return launch_gemv_nb<false>(cfg, make_args(A, nullptr, W, nullptr, out, M, N, K, ws, false, out_fp32), stream);
}

}  // namespace fp8bs
