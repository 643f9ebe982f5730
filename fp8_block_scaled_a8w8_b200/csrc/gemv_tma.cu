// Weight-streaming split-K GEMM for decode M (<= 32), fed by TMA.
//
// Decode is bound by reading W from HBM once ([aiter#7752] "[Perf] Retune gfx942
// Qwen3.8-27B a8w8 blockscale decode rows for cold weights": in a decode step the
// weights come from HBM), and every SM must take part even at M = 1 ([mi210 docs/43]
// section 3: too few workgroups at M = 1 leave most of the card idle). Keeping enough
// bytes in flight per SM is the whole game, so the loads are TMA copies into a deep
// shared-memory ring instead of register-held loads:
//
//   warp 8        producer: per unit, one TMA box of W (128 rows x 128 bytes = one
//                 128-wide K group of one 128-row weight block, i.e. exactly one
//                 w_scale entry) and one box of A (the 8*NB token rows of that group;
//                 rows past M are zero-filled by the TMA unit), 128-byte swizzle
//   warps 0..7    consumers: warp w multiplies rows 16w..16w+15 of the W box with the
//                 token box (mma.sync m16n8k32 e4m3 -> f32, swap-AB: W rows are the
//                 MMA's M, tokens its N), scales the group's partial by
//                 a_scale[token, g] * w_scale[block, g] and accumulates in registers.
//
// Units (128-row block, K group) are ordered block-major and split into equal
// contiguous ranges, one per CTA ("stream-K"), so every SM streams the same bytes for
// any shape. A block covered by one CTA is written directly; a block shared by several
// CTAs is finished by the last to arrive (atomic counter per block), which sums the
// float32 partials in CTA order -- fixed, so results are bit-reproducible -- writes the
// bf16 output and resets the block's counter to zero. Partial sums are always
// overwritten before their counter is incremented, so they need no clearing; the
// counters live in a fixed region at the start of the workspace and are left at zero. A CTA leaves partial sums for at most two blocks (the first and last of
// its range); both are plain stores while streaming, published together at the end of
// the range by one acq_rel atomic per block after a CTA barrier, so nothing stalls the
// stream mid-range.
//
// Fragment layout: inside one MMA the 32 k positions may be paired between A and B in
// any consistent order. Lane (gid, tig) takes bytes [32*tig, 32*tig + 32) of its rows
// (W rows gid, gid+8; token gid) for every group; MMA (c, h) uses bytes 16c + 8h ..
// 16c + 8h + 7 of that slice. Under the 128-byte swizzle (16-byte chunk index XOR row
// mod 8) the chunks 2*tig + c of rows gid and gid+1 are all distinct, so each quarter
// warp's 16-byte shared loads are bank-conflict free.
//
// Every wait is bounded (kWaitLimitNs); on expiry the CTA raises its abort flag and the
// status word, drains its in-flight TMA copies (bounded) and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace fp8bs {

FP8BS_DEFINE_STATUS(gemv_tma)

constexpr int kGtConsumers = 8;
constexpr int kGtThreads = 32 * (kGtConsumers + 1);
constexpr int kGtRows = 16 * kGtConsumers;  // W rows per block

template <int NB>
struct GtCfg {
  static constexpr int kWBytes = kGtRows * 128;
  static constexpr int kABytes = 8 * NB * 128;
  static constexpr int kAAlloc = (kABytes + 1023) / 1024 * 1024;  // keeps every tile 1024-byte aligned
  static constexpr int kStageBytes = kWBytes + kAAlloc;
  static constexpr int kStages = (200 * 1024) / kStageBytes > 12 ? 12 : (200 * 1024) / kStageBytes;
  // scale staging region: a_scale as [G][8 * NB] (zero past M) then w_scale of the CTA's units
  static constexpr int kScaleBytes = 24 * 1024;
  static constexpr size_t kSmemBytes = size_t(kStages) * kStageBytes + 1024 + 256 + kScaleBytes;
  static_assert(kSmemBytes <= 232448, "exceeds the per-CTA shared-memory limit");
};

struct GtParams {
  const float* a_scale;  // [M, G]
  const float* w_scale;  // [nblk, G]
  __nv_bfloat16* out;    // [M, N]
  int M, N, G, nblk;
  int n_ctas;
  int static_w;          // W / w_scale are not written by any kernel still in flight
  float* part;           // [2 * n_ctas][8 warps][NB * 4][32]
  unsigned* counter;     // [nblk]
};

__device__ __forceinline__ int64_t cta_of_unit(int64_t u, int64_t U, int64_t C) { return ((u + 1) * C - 1) / U; }

__device__ __forceinline__ void consumer_bar() { asm volatile("bar.sync 1, %0;" ::"n"(32 * kGtConsumers) : "memory"); }

template <int NB>
__device__ __forceinline__ void gt_store(const GtParams& p, int b, int w, int lane, const float (&v)[NB][4]) {
  const int gid = lane >> 2, tig = lane & 3;
  const int n0 = b * kGtRows + 16 * w + gid;
  if (n0 >= p.N) return;  // N % 16 == 0: rows n0 and n0 + 8 are both in or both out
#pragma unroll
  for (int nb = 0; nb < NB; ++nb)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int token = nb * 8 + 2 * tig + (i & 1);
      if (token < p.M) p.out[int64_t(token) * p.N + n0 + (i >= 2 ? 8 : 0)] = __float2bfloat16_rn(v[nb][i]);
    }
}

// Finish block b if this CTA was its last contributor (arrival count old == contributors - 1):
// sum the contributors' partials in CTA order (a fixed order: bit-reproducible results),
// kBatch contributors' loads in flight at a time, store the output, reset the block's counter.
// Contributor cc > cf of block b started its range inside b (its slot 0); the first
// contributor cf used slot 0 only if its range started exactly at b's first unit, else b
// was its last block (slot 1).
template <int NB>
__device__ __forceinline__ void gt_finish_block(const GtParams& p, int b, unsigned old, int64_t U, int64_t Cn,
                                                int64_t G, int w, int lane) {
  const int64_t cf = cta_of_unit(int64_t(b) * G, U, Cn);
  const int64_t cl = cta_of_unit(int64_t(b + 1) * G - 1, U, Cn);
  if (old != unsigned(cl - cf)) return;
  const int cf_slot = (U * cf / Cn >= int64_t(b) * G) ? 0 : 1;
  float sum[NB][4];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb)
#pragma unroll
    for (int i = 0; i < 4; ++i) sum[nb][i] = 0.f;
  constexpr int kBatch = NB <= 2 ? 8 : 4;  // 4 * NB * kBatch floats held per thread
  for (int64_t c0 = cf; c0 <= cl; c0 += kBatch) {
    float v[kBatch][NB][4];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int64_t cc = c0 + j;
      const int64_t sl = 2 * cc + (cc == cf ? cf_slot : 0);
      const float* src = p.part + (sl * kGtConsumers + w) * (NB * 4 * 32);
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int i = 0; i < 4; ++i) v[j][nb][i] = cc <= cl ? __ldcg(src + (nb * 4 + i) * 32 + lane) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j)
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int i = 0; i < 4; ++i) sum[nb][i] += v[j][nb][i];
  }
  gt_store<NB>(p, b, w, lane, sum);
  if (w == 0 && lane == 0) p.counter[b] = 0u;
}

// kScalesSmem: every CTA's scales fit the staging region (else each unit reads its scales
// from global memory; only very large K or N get there)
template <int NB, bool kScalesSmem>
__global__ void __launch_bounds__(kGtThreads, 1)
    gemv_tma_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmA, const GtParams p) {
  using C = GtCfg<NB>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + size_t(S) * C::kStageBytes);  // full[S], empty[S]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * S);
  volatile unsigned* red_slot = reinterpret_cast<volatile unsigned*>(bars + 2 * S) + 1;  // [2]
  float* sa_s = reinterpret_cast<float*>(smem + size_t(S) * C::kStageBytes + 256);  // [G][8 * NB]

  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t G = p.G;
  const int64_t U = int64_t(p.nblk) * G;
  const int64_t Cn = p.n_ctas;
  const int cta = blockIdx.x;
  const int64_t u0 = U * cta / Cn, u1 = U * (cta + 1) / Cn;
  const int first_blk = int(u0 / G);
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + S + s); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), kGtConsumers);
    }
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&tmW);
    prefetch_tensormap(&tmA);
  }
  __syncthreads();

  if (warp == kGtConsumers) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int last_it[12];
      for (int s = 0; s < S; ++s) last_it[s] = -1;
      int b = first_blk, g = int(u0 - int64_t(first_blk) * G);
      int it = 0;
      int64_t u = u0;
      if (p.static_w) {
        // The weights are not produced by an earlier kernel, so the first ring's worth of
        // W boxes is fetched before waiting for the previous kernel: this overlaps the
        // weight stream with the previous kernel's tail. Activation boxes (produced by the
        // previous kernel) follow the wait.
        const int pre = int(u1 - u0 < S ? u1 - u0 : int64_t(S));
        int pb = b, pg = g;
        for (int j = 0; j < pre; ++j) {
          const uint32_t w_dst = smem_u32(smem + size_t(j) * C::kStageBytes);
          mbar_arrive_expect_tx(full_bar(j), C::kWBytes + C::kABytes);
          tma_load_2d(w_dst, &tmW, full_bar(j), pg * 128, pb * kGtRows);
          if (++pg == G) {
            pg = 0;
            ++pb;
          }
        }
        pdl_wait();
        for (int j = 0; j < pre; ++j, ++u, ++it) {
          const uint32_t w_dst = smem_u32(smem + size_t(j) * C::kStageBytes);
          tma_load_2d(w_dst + C::kWBytes, &tmA, full_bar(j), g * 128, 0);
          last_it[j] = it;
          if (++g == G) {
            g = 0;
            ++b;
          }
        }
      } else {
        pdl_wait();
      }
      for (; u < u1; ++u, ++it) {
        const int s = it % S;
        if (!mbar_wait_bounded(empty_bar(s), ((it / S) & 1) ^ 1, abort_flag, &g_status)) break;
        const uint32_t w_dst = smem_u32(smem + size_t(s) * C::kStageBytes);
        mbar_arrive_expect_tx(full_bar(s), C::kWBytes + C::kABytes);
        tma_load_2d(w_dst, &tmW, full_bar(s), g * 128, b * kGtRows);
        tma_load_2d(w_dst + C::kWBytes, &tmA, full_bar(s), g * 128, 0);
        last_it[s] = it;
        if (++g == G) {
          g = 0;
          ++b;
        }
      }
      for (int s = 0; s < S; ++s) {  // drain (bounded): every issued copy has landed
        if (last_it[s] < 0) continue;
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(full_bar(s), (last_it[s] / S) & 1))
          if (globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicOr(&g_status, kStatusTimeout);
            break;
          }
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    pdl_wait();  // activations, scales and the workspace come from earlier kernels
    const int w = warp;
    const int gid = lane >> 2, tig = lane & 3;
    float acc[NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[nb][i] = 0.f;
    int b = first_blk, g = int(u0 - int64_t(first_blk) * G);
    // fragment byte offsets inside a stage (swizzled chunks 2*tig + c of rows gid / gid+8 / token)
    uint32_t off_w[2], off_a[2];
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const uint32_t chunk = uint32_t(((2 * tig + c) ^ gid) << 4);
      off_w[c] = uint32_t((16 * w + gid) * 128) + chunk;
      off_a[c] = uint32_t(C::kWBytes + gid * 128) + chunk;
    }
    // Stage the scales this CTA needs in shared memory: one global round trip here instead
    // of one per unit on the stream's critical path. a_scale goes in as [G][8 * NB] (zero
    // for tokens past M, so the loop needs no guard); w_scale is [nblk, G] row-major, so
    // unit u's weight scale is w_scale[u] and the CTA's are one contiguous run.
    constexpr int kRows = 8 * NB;
    float* sw_s = sa_s + G * kRows;
    if (kScalesSmem) {
      const int tid = threadIdx.x;  // consumers are threads 0 .. 32 * kGtConsumers - 1
      for (int i = tid; i < kRows * G; i += 32 * kGtConsumers) {
        const int t = i / int(G), gg = i - t * int(G);
        sa_s[gg * kRows + t] = t < p.M ? __ldg(p.a_scale + i) : 0.f;
      }
      for (int j = tid; j < u1 - u0; j += 32 * kGtConsumers) sw_s[j] = __ldg(p.w_scale + u0 + j);
      consumer_bar();
    }
    int pend0 = -1, pend1 = -1;  // blocks this CTA left partial sums for (at most its first and last)
    int n_pending = 0;
    int it = 0;
    bool aborted = false;
    for (int64_t u = u0; u < u1; ++u, ++it) {
      const int s = it % S;
      float sa[NB][2], sw;
      if (kScalesSmem) {
        const float* r = sa_s + g * kRows + 2 * tig;
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          const float2 v = *reinterpret_cast<const float2*>(r + nb * 8);
          sa[nb][0] = v.x;
          sa[nb][1] = v.y;
        }
        sw = sw_s[u - u0];
      } else {
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          const int t0 = nb * 8 + 2 * tig;
          sa[nb][0] = t0 < p.M ? __ldg(p.a_scale + int64_t(t0) * G + g) : 0.f;
          sa[nb][1] = t0 + 1 < p.M ? __ldg(p.a_scale + int64_t(t0 + 1) * G + g) : 0.f;
        }
        sw = __ldg(p.w_scale + int64_t(b) * G + g);
      }
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(full_bar(s), (it / S) & 1, abort_flag, &g_status))) {
        aborted = true;
        break;
      }
      const uint8_t* st = smem + size_t(s) * C::kStageBytes;
      uint4 wa[2], wb[2], av[NB][2];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        wa[c] = *reinterpret_cast<const uint4*>(st + off_w[c]);
        wb[c] = *reinterpret_cast<const uint4*>(st + off_w[c] + 8 * 128);
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) av[nb][c] = *reinterpret_cast<const uint4*>(st + off_a[c] + nb * 8 * 128);
      }
      // A warp works through one unit at a time, so the latency of dependent MMAs is exposed:
      // the four k slices (c, h) of a token tile accumulate separately (summed below) for
      // NB <= 2, in two chains for NB = 3; at NB = 4 the register budget leaves one chain per
      // tile (four independent tiles).
      constexpr int kChains = NB <= 2 ? 4 : (NB == 3 ? 2 : 1);
      float d[kChains][NB][4];
#pragma unroll
      for (int c = 0; c < kChains; ++c)
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
          for (int i = 0; i < 4; ++i) d[c][nb][i] = 0.f;
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const uint32_t a0 = h ? wa[c].z : wa[c].x, a2 = h ? wa[c].w : wa[c].y;
          const uint32_t a1 = h ? wb[c].z : wb[c].x, a3 = h ? wb[c].w : wb[c].y;
#pragma unroll
          for (int nb = 0; nb < NB; ++nb)
            mma_e4m3_16832(d[(2 * h + c) % kChains][nb], a0, a1, a2, a3, h ? av[nb][c].z : av[nb][c].x,
                           h ? av[nb][c].w : av[nb][c].y);
        }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty_bar(s));  // the MMAs consumed the stage's bytes
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        const float s0 = sa[nb][0] * sw, s1 = sa[nb][1] * sw;
        float dd[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          dd[i] = d[0][nb][i];
          if (kChains >= 2) dd[i] += d[kChains >= 2 ? 1 : 0][nb][i];
          if (kChains == 4) dd[i] += d[kChains == 4 ? 2 : 0][nb][i] + d[kChains == 4 ? 3 : 0][nb][i];
        }
        acc[nb][0] = fmaf(dd[0], s0, acc[nb][0]);
        acc[nb][1] = fmaf(dd[1], s1, acc[nb][1]);
        acc[nb][2] = fmaf(dd[2], s0, acc[nb][2]);
        acc[nb][3] = fmaf(dd[3], s1, acc[nb][3]);
      }

      if (g == G - 1 || u == u1 - 1) {
        // ---- block b ends here (or the CTA's range does)
        const bool whole = int64_t(b) * G >= u0 && g == G - 1;
        if (whole) {
          gt_store<NB>(p, b, w, lane, acc);
        } else {
          // partial sum: a plain store now; publishing it (and finding out whether this CTA
          // finishes the block) waits until the end of the range, so no barrier or atomic
          // stalls the stream here
          const int slot = 2 * cta + (b == first_blk ? 0 : 1);
          float* dst = p.part + (int64_t(slot) * kGtConsumers + w) * (NB * 4 * 32);
#pragma unroll
          for (int nb = 0; nb < NB; ++nb)
#pragma unroll
            for (int i = 0; i < 4; ++i) __stcg(dst + (nb * 4 + i) * 32 + lane, acc[nb][i]);
          if (n_pending == 0)
            pend0 = b;
          else
            pend1 = b;
          ++n_pending;
        }
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[nb][i] = 0.f;
      }
      if (++g == G) {
        g = 0;
        ++b;
      }
    }
    // ---- publish the partial sums; the last contributor of a block reduces it
    consumer_bar();  // every consumer thread's partial stores happen before the release below
    if (w == 0 && lane < n_pending) {
      const int pb = lane == 0 ? pend0 : pend1;
      red_slot[lane] = aborted ? 0u : atom_add_acq_rel_gpu(p.counter + pb, 1u);
    }
    consumer_bar();
    if (!aborted) {
      if (n_pending > 0) gt_finish_block<NB>(p, pend0, red_slot[0], U, Cn, G, w, lane);
      if (n_pending > 1) gt_finish_block<NB>(p, pend1, red_slot[1], U, Cn, G, w, lane);
    }
  }
  __syncthreads();
}

// ---------------------------------------------------------------- host side
static int gt_ctas(int64_t M, int64_t N, int64_t K) {
  (void)M;
  const int64_t units = ((N + kGtRows - 1) / kGtRows) * (K / 128);
  return int(std::min<int64_t>(device_sm_count(), units));
}

size_t gemv_tma_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  const int nb = int((M + 7) / 8);
  return kCounterBytes + size_t(2) * gt_ctas(M, N, K) * kGtConsumers * nb * 4 * 32 * sizeof(float);
}

template <int NB, bool kScalesSmem>
static int launch_gt_impl(const void* A, const float* a_scale, const void* W, const float* w_scale, void* out, int64_t M,
                     int64_t N, int64_t K, void* ws, int static_w, void* stream) {
  using Cc = GtCfg<NB>;
  if ((N + kGtRows - 1) / kGtRows > kMaxCounters) return int(cudaErrorInvalidValue);
  if (const int attr = set_max_dynamic_smem(reinterpret_cast<const void*>(gemv_tma_kernel<NB, kScalesSmem>),
                                            int(Cc::kSmemBytes)))
    return attr;
  CUtensorMap mw, ma;
  if (!make_tma_2d_kmajor(&mw, W, true, N, K, kGtRows) || !make_tma_2d_kmajor(&ma, A, true, M, K, 8 * NB))
    return int(cudaErrorInvalidValue);
  GtParams p{};
  p.a_scale = a_scale;
  p.w_scale = w_scale;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.M = int(M);
  p.N = int(N);
  p.G = int(K / 128);
  p.nblk = int((N + kGtRows - 1) / kGtRows);
  p.n_ctas = gt_ctas(M, N, K);
  p.static_w = static_w;
  p.counter = static_cast<unsigned*>(ws);
  p.part = reinterpret_cast<float*>(static_cast<char*>(ws) + kCounterBytes);
  return launch_kernel(gemv_tma_kernel<NB, kScalesSmem>, dim3(p.n_ctas), dim3(kGtThreads), Cc::kSmemBytes, stream, mw, ma, p);
}

template <int NB>
static int launch_gt(const void* A, const float* a_scale, const void* W, const float* w_scale, void* out, int64_t M,
                     int64_t N, int64_t K, void* ws, int static_w, void* stream) {
  const int64_t G = K / 128;
  const int64_t units = (N + kGtRows - 1) / kGtRows * G;
  const int64_t ctas = gt_ctas(M, N, K);
  const int64_t max_units = (units + ctas - 1) / ctas;
  if ((G * 8 * NB + max_units) * int64_t(sizeof(float)) <= GtCfg<NB>::kScaleBytes)
    return launch_gt_impl<NB, true>(A, a_scale, W, w_scale, out, M, N, K, ws, static_w, stream);
  return launch_gt_impl<NB, false>(A, a_scale, W, w_scale, out, M, N, K, ws, static_w, stream);
}

int launch_gemv_tma_a8w8(const void* A, const float* a_scale, const void* W, const float* w_scale, void* out,
                         int64_t M, int64_t N, int64_t K, void* ws, int static_w, void* stream) {
  switch ((M + 7) / 8) {
    case 1: return launch_gt<1>(A, a_scale, W, w_scale, out, M, N, K, ws, static_w, stream);
    case 2: return launch_gt<2>(A, a_scale, W, w_scale, out, M, N, K, ws, static_w, stream);
    case 3: return launch_gt<3>(A, a_scale, W, w_scale, out, M, N, K, ws, static_w, stream);
    case 4: return launch_gt<4>(A, a_scale, W, w_scale, out, M, N, K, ws, static_w, stream);
    default: return int(cudaErrorInvalidValue);
  }
}

// ---------------------------------------------------------------- allocation-free variant
// Some callers cannot allocate device memory at the point where they issue a GEMM: code
// running under an allocator that is frozen or owned by someone else (a serving engine
// whose memory pool was sized once at start-up, a plugin inside a host framework, code
// that must not trigger an allocation-induced synchronisation), or code with no handle on
// an allocator at all. For them the weight-streaming kernel can take its split-K scratch
// from a fixed array that is part of the loaded library image instead of a caller-owned
// workspace. Every GPU that loads the library holds this array until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB: counters + partial sums
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array on the current device (looked up once per device;
// the array's host-side name is not a device address). nullptr if the lookup failed.
static void* noalloc_scratch_ptr() {
  static void* ptrs[64];
  static cudaError_t errs[64];
  static std::once_flag once[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::call_once(once[dev], [dev] {
    void* p = nullptr;
    errs[dev] = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    ptrs[dev] = errs[dev] == cudaSuccess ? p : nullptr;
  });
  return ptrs[dev];
}

int launch_gemv_tma_noalloc(const void* A, const float* a_scale, const void* W, const float* w_scale, void* out,
                            int64_t M, int64_t N, int64_t K, void* stream, int* too_big) {
  *too_big = 0;
  if (M > kGemvMaxM || gemv_tma_workspace_bytes(M, N, K) > kNoAllocScratchBytes ||
      (N + kGtRows - 1) / kGtRows > kMaxCounters) {
    *too_big = 1;
    return int(cudaErrorInvalidValue);
  }
  void* scratch = noalloc_scratch_ptr();
  if (!scratch) return int(cudaErrorInvalidSymbol);
  // The array keeps whatever the previous call left in it; the arrival counters this call
  // uses must start at zero, so clear them (partial sums are always written before read).
  const size_t counter_bytes = size_t((N + kGtRows - 1) / kGtRows) * sizeof(unsigned);
  cudaError_t e = cudaMemsetAsync(scratch, 0, counter_bytes, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return int(e);
  return launch_gemv_tma_a8w8(A, a_scale, W, w_scale, out, M, N, K, scratch, 0, stream);
}

}  // namespace fp8bs
