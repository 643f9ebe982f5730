// Weight-streaming split-K GEMM for decode M (<= 32) on the 5th-generation tensor cores.
//
// Decode reads every weight byte once from HBM and does little arithmetic per byte
// ([aiter#7752] "[Perf] Retune gfx942 Qwen3.8-27B a8w8 blockscale decode rows for cold
// weights": in a decode step the weights come from HBM), so all SMs stream their share
// of W ([mi210 docs/43] section 3: at M = 1 too few workgroups leave the card idle) and
// the arithmetic must never hold the stream up. The work split is the one of the
// mma.sync weight-streaming kernel: a unit is one 128-row weight block x one 128-wide K
// group (exactly one w_scale entry), units are ordered block-major and cut into equal
// contiguous ranges, one per CTA ("stream-K"), and a block shared by several CTAs is
// finished by its last contributor, which sums the float32 partials in CTA order (a
// fixed order: bit-reproducible results).
//
// The products run on tcgen05 with the operands swapped ("swap AB"): the weight box is
// the MMA's A operand (M = 128 weight rows), the token box its B operand (N = 32 token
// slots; TMA zero-fills the rows past M), both K-major with the 128-byte swizzle the
// TMA wrote. An issuing thread issues a unit's four K = 32 MMAs into one of eight
// 32-column TMEM buffers and commits; the epilogue warps take finished buffers with tcgen05.ld
// (TMEM lane = weight row = thread), multiply the unit's float32 partial by
// a_scale[token, g] * w_scale[block, g] and accumulate in registers -- the block-scale
// definition group by group ([cookbook#8]: 128x128 weight blocks, 1x128 activation
// groups). The tensor core runs up to eight units ahead of the epilogue.
//
//   warp 0        TMA producer: per unit one weight box (128 rows x 128 bytes) and one
//                 token box (NT rows x 128 bytes); with static weights the first few
//                 weight boxes are fetched before the grid-dependency wait
//   warp 1        TMEM allocator; lane 0 issues the MMAs of even units
//   warp 2        lane 0 issues the MMAs of odd units
//   warp 3        only takes part in the split-K reduction
//   warps 4..7    epilogue: warp 4 + q reads TMEM lanes 32q .. 32q + 31
//
// The CTA's scales are staged in shared memory once (a_scale as [G][NT], NT >= M token
// columns, zero past M; its run of w_scale, which is [nblk, G] row-major, so unit u's
// weight scale is w_scale[u]); shapes whose scales do not fit the staging region go to
// the mma.sync kernel instead.
//
// A CTA uses 112 KB of shared memory and 256 TMEM columns, so two fit on an SM: the
// next call's CTAs become resident while this call's still stream and fetch their first
// weight boxes during its tail. Every CTA takes at least 8 units (small weights are not
// split into dozens of contributors per block).
//
// The bf16 GEMM (kBf16) runs the same kernel: a unit is 128 weight rows x 64 bf16
// columns (the same 128-byte rows), the products are kind::f16, there are no scales, and
// the output may be float32.
//
// Every wait is bounded (kWaitLimitNs); on expiry the CTA raises its abort flag and the
// device status word, every role leaves its loop, in-flight TMA copies and MMAs are
// drained (bounded), TMEM is freed and the CTA exits without publishing partial sums.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace fp8bs {

FP8BS_DEFINE_STATUS(gemv_umma)

constexpr int kGuThreads = 256;
constexpr int kGuRows = 128;                          // weight rows per block = MMA M = TMEM lanes
constexpr int kGuSlots = 32;                          // token slots = MMA N
constexpr int kGuBufs = 8;                            // TMEM accumulator buffers
constexpr int kGuTmemCols = kGuBufs * kGuSlots;       // 256
constexpr int kGuWBytes = kGuRows * 128;              // 16 KiB weight box
constexpr int kGuABytes = kGuSlots * 128;             // 4 KiB token slots per stage
constexpr int kGuStageBytes = kGuWBytes + kGuABytes;  // multiple of 1024: every box stays aligned
// Two CTAs fit on an SM (shared memory, registers, 2 x 256 TMEM columns), so the next
// call's CTAs become resident while this call's are still streaming and fetch their first
// weight boxes during its tail: the HBM stream does not pause between calls.
constexpr int kGuCtasPerSm = 2;
constexpr int kGuStages = 5;
// Weight boxes fetched before the grid-dependency wait (static weights). Each SM's
// requests are served roughly in issue order, so everything issued after the wait (the
// token boxes, the activation scales) lands only once these have: fetch about what
// the gap before the wait can absorb, not the whole ring.
constexpr int kGuPrefetch = 4;
// (An L2 prefetch of the following units before the wait was measured: it made N = 5120
// and N = 14336 calls 5% slower and N = 34816 calls no faster, so it is not done.)
// The weight boxes are loaded with the evict-first L2 policy: they are read once per call.
// MMA issuing threads (lane 0 of warps 1 .. kGuIssuers): issuer i takes the units with
// it % kGuIssuers == i. One thread spends longer issuing a unit's MMAs, waits and commits
// than the HBM needs to deliver the unit's 16 KiB; two keep up.
constexpr int kGuIssuers = 2;
constexpr int kGuBarBytes = 512;
constexpr int kGuScaleBytes = 8 * 1024;
constexpr size_t kGuSmemBytes = size_t(kGuStages) * kGuStageBytes + kGuBarBytes + kGuScaleBytes + 1024;
static_assert(kGuStageBytes % 1024 == 0, "stage alignment");
static_assert((2 * kGuStages + 2 * kGuBufs + kGuIssuers) * 8 + 13 * 4 <= kGuBarBytes, "barrier region (misc: 13 words)");
static_assert(kGuBufs % kGuIssuers == 0, "a TMEM buffer always belongs to the same issuer");
static_assert(kGuIssuers >= 1 && kGuIssuers <= 2, "issuers are lane 0 of warps 1 and 2");
static_assert(kGuCtasPerSm * (kGuSmemBytes + 1024) <= 233472, "two CTAs must fit an SM's shared memory");
static_assert(kGuCtasPerSm * kGuTmemCols <= 512, "two CTAs must fit an SM's TMEM");
static_assert(kGuPrefetch <= kGuStages, "prefetch within the ring");
constexpr uint32_t kGuIdesc = make_idesc(kFmtE4M3, kFmtE4M3, kGuRows, kGuSlots);
constexpr uint32_t kGuIdescBf16 = make_idesc(kFmtBF16, kFmtBF16, kGuRows, kGuSlots);
// A CTA takes at least this many units: a small weight spread over every SM would leave
// each block with dozens of split-K contributors to sum.
constexpr int64_t kGuMinUnitsPerCta = 8;

struct GuParams {
  const float* a_scale;  // [M, G]
  const float* w_scale;  // [nblk, G]
  void* out;             // [M, N] bf16 (or float32 when out_fp32)
  int M, N, G, nblk;
  int n_ctas;
  int static_w;          // W / w_scale are not written by any kernel still in flight
  float* part;           // [2 * n_ctas][kGuSlots][kGuRows]
  unsigned* counter;     // [nblk]
  int out_fp32;          // bf16 GEMM only
  const uint8_t* wt;     // tiled weights (16 KiB tiles, see tile_weight_kernel), or null
};

__device__ __forceinline__ void gu_put(const GuParams& p, int64_t idx, float v) {
  if (p.out_fp32)
    static_cast<float*>(p.out)[idx] = v;
  else
    static_cast<__nv_bfloat16*>(p.out)[idx] = __float2bfloat16_rn(v);
}

__device__ __forceinline__ int64_t gu_cta_of_unit(int64_t u, int64_t U, int64_t C) { return ((u + 1) * C - 1) / U; }

__device__ __forceinline__ void gu_epilogue_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// Ordering barrier between the epilogue's weight-scale loads and the producer's prefetch
// (128 epilogue threads arrive, the producer warp's 32 wait).
__device__ __forceinline__ void gu_order_bar_arrive() { asm volatile("bar.arrive 2, 160;" ::: "memory"); }
__device__ __forceinline__ void gu_order_bar_sync() { asm volatile("bar.sync 2, 160;" ::: "memory"); }

template <int NT>
__device__ __forceinline__ void gu_tmem_ld(uint32_t taddr, uint32_t (&r)[NT]) {
  if constexpr (NT == 8)
    tmem_ld_32x32b_x8(taddr, r);
  else if constexpr (NT == 16)
    tmem_ld_32x32b_x16(taddr, r);
  else
    tmem_ld_32x32b_x32(taddr, r);
}

// Split-K finish, by a contributor fixed in advance: block b is finished by the CTA
// whose range holds b's last unit (cl). For that CTA b is its first block, so a CTA
// finishes at most one block, and the other contributors cf .. cl - 1 only publish their
// partial (a release add on the block's counter, no round trip). The finisher waits
// (bounded) until all of them have arrived, then all 256 threads sum the contributors'
// partials in CTA order, kB contributors' loads in flight at a time, store the output and
// reset the counter. Thread tid owns weight row tid % 128 and tokens tid / 128 + 2j.
// Contributor cc > cf started its range inside b (its slot 0); the first contributor cf
// used slot 0 only if its range started exactly at b's first unit, else b was its last
// block (slot 1).
struct GuFinish {
  int blk;       // block this CTA finishes, or -1
  int others;    // contributors before this CTA (cl - cf)
  int cf;        // first contributor
  int cf_slot;   // its slot for b
};

__device__ __forceinline__ GuFinish gu_finish_plan(int64_t cta, int64_t u0, int64_t u1, int64_t U, int64_t Cn,
                                                   int64_t G) {
  GuFinish f{-1, 0, 0, 0};
  const int64_t b = u0 / G;
  if (b * G < u0 && (b + 1) * G <= u1) {  // starts before this range and ends inside it
    f.blk = int(b);
    f.cf = int(gu_cta_of_unit(b * G, U, Cn));
    f.others = int(cta - f.cf);
    f.cf_slot = (U * f.cf / Cn >= b * G) ? 0 : 1;
  }
  return f;
}

template <int NT>
__device__ __forceinline__ void gu_finish_block(const GuParams& p, const GuFinish& f) {
  constexpr int kE = NT * kGuRows / kGuThreads;  // elements per thread
  constexpr int kB = kE >= 16 ? 4 : kE >= 8 ? 6 : 8;
  const int tid = threadIdx.x;
  const int r = tid & (kGuRows - 1);
  const int t0 = tid >> 7;
  const int cf = f.cf, cl = f.cf + f.others;
  float sum[kE];
#pragma unroll
  for (int j = 0; j < kE; ++j) sum[j] = 0.f;
  for (int c0 = cf; c0 <= cl; c0 += kB) {
    float v[kB][kE];
#pragma unroll
    for (int jj = 0; jj < kB; ++jj) {
      const int cc = c0 + jj;
      const int64_t sl = 2 * cc + (cc == cf ? f.cf_slot : 0);
      const float* src = p.part + sl * (kGuSlots * kGuRows) + r;
#pragma unroll
      for (int j = 0; j < kE; ++j) {
        const int t = t0 + 2 * j;
        v[jj][j] = (cc <= cl && t < p.M) ? __ldcg(src + t * kGuRows) : 0.f;
      }
    }
#pragma unroll
    for (int jj = 0; jj < kB; ++jj)
#pragma unroll
      for (int j = 0; j < kE; ++j) sum[j] += v[jj][j];
  }
  const int n = f.blk * kGuRows + r;
  if (n < p.N) {
#pragma unroll
    for (int j = 0; j < kE; ++j) {
      const int t = t0 + 2 * j;
      if (t < p.M) gu_put(p, int64_t(t) * p.N + n, sum[j]);
    }
  }
  if (tid == 0) p.counter[f.blk] = 0u;
}

// NT: token columns the epilogue reads per unit (8, 16 or 32 >= M).
// kBf16: the bf16 GEMM (out = A W^T): a unit is 128 weight rows x 64 bf16 columns (the
// same 128-byte rows), kind::f16 products, no scales.
template <int NT, bool kBf16>
__global__ void __launch_bounds__(kGuThreads, kGuCtasPerSm)
    gemv_umma_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmA, const GuParams p) {
  constexpr int S = kGuStages;
  constexpr int B = kGuBufs;
  // The token box has NT rows (rows past M read as zero); MMA column n depends only on
  // token row n, so slots NT..31 may hold anything: their columns are never read.
  constexpr uint32_t kTx = kGuWBytes + NT * 128;
  constexpr int kX = kBf16 ? 64 : 128;  // TMA x step per unit, in elements (128 bytes)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + size_t(S) * kGuStageBytes);  // full[S] empty[S] tfull[B] tempty[B] drain
  uint32_t* misc = reinterpret_cast<uint32_t*>(bars + 2 * S + 2 * B + kGuIssuers);
  uint32_t* tmem_slot = misc;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  volatile int* pend_s = reinterpret_cast<volatile int*>(misc + 2);             // n_pending, block 0, block 1
  volatile int* passed = reinterpret_cast<volatile int*>(misc + 7);  // units whose full-barrier wait has passed
  volatile int* plan_s = reinterpret_cast<volatile int*>(misc + 8);   // GuFinish: blk, others, cf, cf_slot
  volatile int* fin_ok = reinterpret_cast<volatile int*>(misc + 12);
  float* sa_s = reinterpret_cast<float*>(smem + size_t(S) * kGuStageBytes + kGuBarBytes);  // [G][NT]

  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t G = p.G;
  const int64_t U = int64_t(p.nblk) * G;
  const int64_t Cn = p.n_ctas;
  const int cta = blockIdx.x;
  const int64_t u0 = U * cta / Cn, u1 = U * (cta + 1) / Cn;
  const int n_units = int(u1 - u0);
  const int first_blk = int(u0 / G);
  float* sw_s = sa_s + G * NT;  // [n_units]
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + S + s); };
  auto tfull_bar = [&](int b) { return smem_u32(bars + 2 * S + b); };
  auto tempty_bar = [&](int b) { return smem_u32(bars + 2 * S + B + b); };
  auto drain_bar = [&](int i) { return smem_u32(bars + 2 * S + 2 * B + i); };
  // Bounded spin until units 0 .. it-1 have passed their full-barrier wait.
  auto wait_passed = [&](int it) {
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t i = 1; *passed < it; ++i) {
      if ((i & 63u) == 0) {
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
          *abort_flag = 1;
          atomicOr(&g_status, kStatusTimeout);
          return false;
        }
      }
    }
    return true;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < B; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 4);  // one arrival per epilogue warp
    }
    for (int i = 0; i < kGuIssuers; ++i) mbar_init(drain_bar(i), 1);
    *abort_flag = 0;
    pend_s[0] = 0;
    *passed = 0;
    fence_barrier_init();
    prefetch_tensormap(&tmW);
    prefetch_tensormap(&tmA);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kGuTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (!kBf16 && p.static_w) gu_order_bar_sync();  // the epilogue's w_scale requests go out first
    if (lane == 0) {
      int last_it[kGuStages];
      for (int s = 0; s < S; ++s) last_it[s] = -1;
      int b = first_blk, g = int(u0 - int64_t(first_blk) * G);
      int it = 0;
      const uint64_t w_policy = l2_policy_evict_first();
      if (!kBf16 && p.static_w) {
        // The weights are not produced by an earlier kernel: fetch the first ring's worth
        // of weight boxes before waiting for the previous kernel, overlapping its tail.
        const int pre = n_units < kGuPrefetch ? n_units : kGuPrefetch;
        int pb = b, pg = g;
        for (int j = 0; j < pre; ++j) {
          const uint32_t dst = smem_u32(smem + size_t(j) * kGuStageBytes);
          mbar_arrive_expect_tx(full_bar(j), kTx);
          if (p.wt)  // tiled weights: the unit is one contiguous 16 KiB tile
            bulk_load_hint(dst, p.wt + (int64_t(pb) * G + pg) * 16384, 16384, full_bar(j), w_policy);
          else
            tma_load_2d_hint(dst, &tmW, full_bar(j), pg * kX, pb * kGuRows, w_policy);
          if (++pg == G) {
            pg = 0;
            ++pb;
          }
        }
        pdl_wait();
        for (int j = 0; j < pre; ++j, ++it) {
          const uint32_t dst = smem_u32(smem + size_t(j) * kGuStageBytes);
          tma_load_2d(dst + kGuWBytes, &tmA, full_bar(j), g * kX, 0);
          last_it[j] = it;
          if (++g == G) {
            g = 0;
            ++b;
          }
        }
      } else {
        pdl_wait();
      }
      for (; it < n_units; ++it) {
        const int s = it % S;
        if (!mbar_wait_bounded(empty_bar(s), ((it / S) & 1) ^ 1, abort_flag, &g_status)) break;
        const uint32_t dst = smem_u32(smem + size_t(s) * kGuStageBytes);
        mbar_arrive_expect_tx(full_bar(s), kTx);
        if (p.wt)
          bulk_load_hint(dst, p.wt + (int64_t(b) * G + g) * 16384, 16384, full_bar(s), w_policy);
        else
          tma_load_2d_hint(dst, &tmW, full_bar(s), g * kX, b * kGuRows, w_policy);
        tma_load_2d(dst + kGuWBytes, &tmA, full_bar(s), g * kX, 0);
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
  } else if (warp >= 1 && warp <= kGuIssuers) {
    // ------------------------------------------------------------ MMA issuers
    pdl_wait();  // the bounded waits below start once the previous kernel has completed
    if (lane == 0) {
      const int me = warp - 1;
      bool issued = false;
      for (int it = me; it < n_units; it += kGuIssuers) {
        const int s = it % S;
        // Units pass their full-barrier wait in unit order: an issuer that ran a whole ring
        // ahead of the other would otherwise test stage s's barrier while it still holds an
        // older phase of the same parity and take stale bytes. (Stages and TMEM buffers are
        // then also reused strictly in order.)
        if (kGuIssuers > 1 && !wait_passed(it)) break;
        if (!mbar_wait_bounded(full_bar(s), (it / S) & 1, abort_flag, &g_status)) break;
        if (kGuIssuers > 1) *passed = it + 1;
        const int buf = it % B;
        if (!mbar_wait_bounded(tempty_bar(buf), ((it / B) & 1) ^ 1, abort_flag, &g_status)) break;
        tc_fence_after();
        const uint32_t st = smem_u32(smem + size_t(s) * kGuStageBytes);
        const uint64_t adesc = sw128_kmajor_desc(st);
        const uint64_t bdesc = sw128_kmajor_desc(st + kGuWBytes);
        const uint32_t d_tmem = tmem_base + uint32_t(buf * kGuSlots);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {  // 32 bytes of K per MMA: 32 e4m3 or 16 bf16
          if constexpr (kBf16)
            umma_f16(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, kGuIdescBf16, kk > 0);
          else
            umma_f8f6f4(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, kGuIdesc, kk > 0);
        }
        issued = true;
        umma_commit(empty_bar(s));    // the stage's bytes are consumed once these MMAs complete
        umma_commit(tfull_bar(buf));  // the unit's partial is in TMEM
      }
      if (issued) {  // drain: every MMA issued by this thread has completed once drain_bar flips
        umma_commit(drain_bar(me));
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(drain_bar(me), 0))
          if (globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicOr(&g_status, kStatusTimeout);
            break;
          }
      }
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ split-K plan (off the tail)
    if (lane == 0) {
      const GuFinish f = gu_finish_plan(cta, u0, u1, U, Cn, G);
      plan_s[0] = f.blk;
      plan_s[1] = f.others;
      plan_s[2] = f.cf;
      plan_s[3] = f.cf_slot;
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue warps 4..7
    const int q = warp - 4;
    const int r = 32 * q + lane;  // weight row within the block = TMEM lane
    const uint32_t lane_addr = tmem_base + (uint32_t(32 * q) << 16);
    const int et = threadIdx.x - 128;
    // Stage the scales: the CTA's run of w_scale (static weights: requested before the
    // producer's weight prefetch, which waits on the ordering barrier) and a_scale as
    // [G][NT] (written by the previous kernel: after the grid-dependency wait), each
    // thread's loads issued together.
    if (kBf16) {
      pdl_wait();  // the activations and the workspace come from earlier kernels
    } else if (p.static_w) {  // (fp8 only: the bf16 GEMM has no static-weight flag)
      float v[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) v[k] = et + 128 * k < n_units ? __ldg(p.w_scale + u0 + et + 128 * k) : 0.f;
      gu_order_bar_arrive();
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (et + 128 * k < n_units) sw_s[et + 128 * k] = v[k];
      for (int j = et + 512; j < n_units; j += 128) sw_s[j] = __ldg(p.w_scale + u0 + j);
      pdl_wait();  // activation scales and the workspace come from earlier kernels
    } else {
      pdl_wait();  // so may the weight scales
      for (int j = et; j < n_units; j += 128) sw_s[j] = __ldg(p.w_scale + u0 + j);
    }
    constexpr int kPer = 8;
    for (int base = 0; base < (kBf16 ? 0 : NT * int(G)); base += 128 * kPer) {
      float v[kPer];
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int i = base + 128 * k + et;  // = t * G + gg
        const int t = i / int(G);
        v[k] = (i < NT * int(G) && t < p.M) ? __ldg(p.a_scale + i) : 0.f;
      }
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int i = base + 128 * k + et;
        const int t = i / int(G), gg = i - t * int(G);
        if (i < NT * int(G)) sa_s[gg * NT + t] = v[k];
      }
    }
    gu_epilogue_bar();

    float acc[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t] = 0.f;
    int b = first_blk, g = int(u0 - int64_t(first_blk) * G);
    int n_pending = 0, pend0 = -1, pend1 = -1;
    for (int it = 0; it < n_units; ++it) {
      const int buf = it % B;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(tfull_bar(buf), (it / B) & 1, abort_flag, &g_status))) break;
      tc_fence_after();
      uint32_t d[NT];
      gu_tmem_ld<NT>(lane_addr + uint32_t(buf * kGuSlots), d);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(buf));  // the buffer may take the next unit
      if constexpr (kBf16) {
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[t] += __uint_as_float(d[t]);
      } else {
      const float sw = sw_s[it];
      const float* sa = sa_s + g * NT;
#pragma unroll
      for (int t = 0; t < NT; t += 4) {
        const float4 s4 = *reinterpret_cast<const float4*>(sa + t);
        acc[t + 0] = fmaf(__uint_as_float(d[t + 0]), s4.x * sw, acc[t + 0]);
        acc[t + 1] = fmaf(__uint_as_float(d[t + 1]), s4.y * sw, acc[t + 1]);
        acc[t + 2] = fmaf(__uint_as_float(d[t + 2]), s4.z * sw, acc[t + 2]);
        acc[t + 3] = fmaf(__uint_as_float(d[t + 3]), s4.w * sw, acc[t + 3]);
      }
      }
      if (g == G - 1 || it == n_units - 1) {
        // ---- block b ends here (or the CTA's range does)
        const bool whole = int64_t(b) * G >= u0 && g == G - 1;
        if (whole) {
          const int n = b * kGuRows + r;
          if (n < p.N) {
#pragma unroll
            for (int t = 0; t < NT; ++t)
              if (t < p.M) gu_put(p, int64_t(t) * p.N + n, acc[t]);
          }
        } else {
          // partial sum: a plain store now, published after the loop
          const int slot = 2 * cta + (b == first_blk ? 0 : 1);
          float* dst = p.part + int64_t(slot) * (kGuSlots * kGuRows) + r;
#pragma unroll
          for (int t = 0; t < NT; ++t)
            if (t < p.M) __stcg(dst + t * kGuRows, acc[t]);
          if (n_pending == 0)
            pend0 = b;
          else
            pend1 = b;
          ++n_pending;
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[t] = 0.f;
      }
      if (++g == G) {
        g = 0;
        ++b;
      }
    }
    if (threadIdx.x == 128) {
      pend_s[1] = pend0;
      pend_s[2] = pend1;
      pend_s[0] = n_pending;
    }
  }

  // ---- every warp: free TMEM, publish the partial sums, finish the blocks this CTA completes
  __syncwarp();
  tc_fence_before();
  __syncthreads();  // TMEM reads, partial stores and the pending list are complete
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kGuTmemCols);
  }
  pdl_wait();  // warp 3 has not waited yet; the tail writes the workspace and the output
  if (*abort_flag) return;
  const GuFinish f{plan_s[0], plan_s[1], plan_s[2], plan_s[3]};
  // publish the partial sums of the blocks this CTA does not finish (at most two)
  const int n_pending = pend_s[0];
  if (threadIdx.x < n_pending && pend_s[1 + threadIdx.x] != f.blk)
    red_add_release_gpu(p.counter + pend_s[1 + threadIdx.x], 1u);
  if (f.blk < 0) return;
  if (threadIdx.x == 0) {  // bounded wait for the other contributors
    bool ok = true;
    const unsigned long long t0 = globaltimer_ns();
    while (ld_acquire_gpu(p.counter + f.blk) != unsigned(f.others)) {
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        atomicOr(&g_status, kStatusTimeout);
        ok = false;
        break;
      }
    }
    *fin_ok = ok;
  }
  __syncthreads();
  if (*fin_ok) gu_finish_block<NT>(p, f);
}

// ---------------------------------------------------------------- host side
static int gu_ctas(int64_t N, int64_t K, bool bf16) {
  const int64_t units = ((N + kGuRows - 1) / kGuRows) * (K / (bf16 ? 64 : 128));
  return int(std::max<int64_t>(1, std::min<int64_t>(device_sm_count(), units / kGuMinUnitsPerCta)));
}

static bool gu_scales_fit(int64_t M, int64_t N, int64_t K) {
  const int64_t G = K / 128;
  const int64_t units = ((N + kGuRows - 1) / kGuRows) * G;
  const int64_t ctas = gu_ctas(N, K, false);
  const int64_t max_units = (units + ctas - 1) / ctas;
  const int64_t nt = M <= 8 ? 8 : M <= 16 ? 16 : 32;
  return (G * nt + max_units) * int64_t(sizeof(float)) <= kGuScaleBytes;
}

static size_t gu_own_workspace(int64_t N, int64_t K, bool bf16) {
  return kCounterBytes + size_t(2) * gu_ctas(N, K, bf16) * kGuSlots * kGuRows * sizeof(float);
}

size_t gemv_umma_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  return std::max(gu_own_workspace(N, K, false), gemv_tma_workspace_bytes(M, N, K));  // fallback kernel's need
}

size_t gemv_umma_bf16_workspace_bytes(int64_t, int64_t N, int64_t K) { return gu_own_workspace(N, K, true); }

template <int NT, bool kBf16>
static int launch_gu(const void* A, const float* a_scale, const void* W, const float* w_scale, void* out, int64_t M,
                     int64_t N, int64_t K, void* ws, int static_w, int out_fp32, void* stream, bool tiled_w = false) {
  // the carveout is a hint; the dynamic shared-memory limit is required (per device)
  if (const int attr = set_max_dynamic_smem(reinterpret_cast<const void*>(gemv_umma_kernel<NT, kBf16>),
                                            int(kGuSmemBytes)))
    return attr;
  static std::once_flag carve_once;
  std::call_once(carve_once, [] {
    (void)cudaFuncSetAttribute(gemv_umma_kernel<NT, kBf16>, cudaFuncAttributePreferredSharedMemoryCarveout,
                               int(cudaSharedmemCarveoutMaxShared));
  });
  CUtensorMap mw, ma;
  if (!make_tma_2d_kmajor(&ma, A, !kBf16, M, K, NT)) return int(cudaErrorInvalidValue);
  if (tiled_w)
    mw = ma;  // (unused: the weight tiles are plain copies)
  else if (!make_tma_2d_kmajor(&mw, W, !kBf16, N, K, kGuRows))
    return int(cudaErrorInvalidValue);
  GuParams p{};
  p.a_scale = a_scale;
  p.w_scale = w_scale;
  p.out = out;
  p.M = int(M);
  p.N = int(N);
  p.G = int(K / (kBf16 ? 64 : 128));
  p.nblk = int((N + kGuRows - 1) / kGuRows);
  p.n_ctas = gu_ctas(N, K, kBf16);
  p.static_w = kBf16 ? 0 : static_w;
  p.out_fp32 = kBf16 ? out_fp32 : 0;
  p.counter = static_cast<unsigned*>(ws);
  p.part = reinterpret_cast<float*>(static_cast<char*>(ws) + kCounterBytes);
  p.wt = tiled_w ? static_cast<const uint8_t*>(W) : nullptr;
  return launch_kernel(gemv_umma_kernel<NT, kBf16>, dim3(p.n_ctas), dim3(kGuThreads), kGuSmemBytes, stream, mw, ma, p);
}

int launch_gemv_umma_a8w8(const void* A, const float* a_scale, const void* W, const float* w_scale, void* out,
                          int64_t M, int64_t N, int64_t K, void* ws, int static_w, void* stream, bool tiled_w) {
  if (M < 1 || M > kGemvMaxM || (N + kGuRows - 1) / kGuRows > kMaxCounters) return int(cudaErrorInvalidValue);
  if (!gu_scales_fit(M, N, K)) {
    if (tiled_w) return int(cudaErrorNotSupported);  // (the mma.sync kernel reads the standard layout only)
    return launch_gemv_tma_a8w8(A, a_scale, W, w_scale, out, M, N, K, ws, static_w, stream);
  }
  if (M <= 8) return launch_gu<8, false>(A, a_scale, W, w_scale, out, M, N, K, ws, static_w, 0, stream, tiled_w);
  if (M <= 16) return launch_gu<16, false>(A, a_scale, W, w_scale, out, M, N, K, ws, static_w, 0, stream, tiled_w);
  return launch_gu<32, false>(A, a_scale, W, w_scale, out, M, N, K, ws, static_w, 0, stream, tiled_w);
}

bool gemv_umma_reads_tiles(int64_t M, int64_t N, int64_t K) { return M >= 1 && M <= kGemvMaxM && gu_scales_fit(M, N, K); }

int launch_gemv_umma_bf16(const void* A, const void* W, void* out, int out_fp32, int64_t M, int64_t N, int64_t K,
                          void* ws, void* stream) {
  if (M < 1 || M > kGemvMaxM || K % 64 != 0 || (N + kGuRows - 1) / kGuRows > kMaxCounters)
    return int(cudaErrorInvalidValue);
  if (M <= 8) return launch_gu<8, true>(A, nullptr, W, nullptr, out, M, N, K, ws, 0, out_fp32, stream);
  if (M <= 16) return launch_gu<16, true>(A, nullptr, W, nullptr, out, M, N, K, ws, 0, out_fp32, stream);
  return launch_gu<32, true>(A, nullptr, W, nullptr, out, M, N, K, ws, 0, out_fp32, stream);
}

}  // namespace fp8bs
