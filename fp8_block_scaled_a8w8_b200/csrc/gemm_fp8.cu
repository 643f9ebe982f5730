// Tensor-core GEMM for prefill-sized M with a wide promotion epilogue: a8w8 block scale
// on tcgen05.mma (kind::f8f6f4), TMEM accumulators, operands staged by TMA with the
// 128-byte swizzle; persistent and warp-specialised.
//
//   warp 0        TMA producer: per K group one 128-row A box and one BN-row W box
//   warp 1        TMEM allocator and MMA issuer (one thread)
//   warps 2-3     idle (they complete warpgroup 0)
//   warps 4..19   promotion epilogue, four warpgroups
//
// The block-scale definition applies a different scale to every 128-wide K group
// ([cookbook#8]: 128x128 weight blocks, 1x128 activation groups), so a group's fp32
// partial cannot stay in the tensor core's accumulator: every group's four K = 32 MMAs
// write a fresh partial P_g into one of the TMEM buffers, and the epilogue reads it back
// and adds a_scale[row, g] * w_scale[col / 128, g] * P_g into float32 registers. Reading
// P_g back is the cost that decides the speed: 128 x BN float32 per group, against 2 x BN
// cycles of MMA per group. Sixteen epilogue warps (each 32 TMEM lanes x BN/4 columns)
// keep enough TMEM loads in flight to drain a buffer well inside one group's MMA time,
// release it as soon as the data is in registers, and then scale and accumulate with
// packed two-wide FMAs (fma.rn.f32x2, IEEE-identical to two fmaf). With BN = 256 two
// buffers fill the 512 TMEM columns; with BN = 128 there are four.
//
// Split K (for shapes whose tiles leave SMs idle): a work item is (tile, K range); each
// split stores its float32 partial tile and the tile is finished by the shared split-K
// finish (splitk.cuh): with one item per CTA every split sums its own share of the tile
// once all have published, otherwise the last split to arrive sums it. The partials are
// added in split order -- a fixed order, so results are bit-reproducible -- and rounded
// once to bf16.
//
// Every wait is bounded by a limit passed in the kernel parameters (1 s by default); a
// wait that gives up raises the CTA's abort flag and the device status word, the roles
// leave their loops, in-flight TMA copies and MMAs are drained (bounded) and TMEM is
// freed before the CTA exits. For testing, the producer of CTA 0 can be told to skip one
// K group's loads (nothing ever fills that stage, so the MMA issuer's wait runs out).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"
#include "splitk.cuh"

namespace fp8bs {

FP8BS_DEFINE_STATUS(fp8)

constexpr int kF8Threads = 640;  // 5 warpgroups
constexpr int kF8EpiWarps = 16;
constexpr int kF8EpiThreads = 32 * kF8EpiWarps;
// Registers: the launch gives every thread kF8LaunchRegs (checked by the build);
// warpgroup 0 drops to kF8ProducerRegs and the four epilogue warpgroups rise to
// kF8EpilogueRegs, which together use no more than the launch's 640 * kF8LaunchRegs.
constexpr int kF8LaunchRegs = 96;
constexpr int kF8ProducerRegs = 32;
constexpr int kF8EpilogueRegs = 112;
static_assert(128 * kF8ProducerRegs + kF8EpiThreads * kF8EpilogueRegs <= kF8Threads * kF8LaunchRegs, "register split");
constexpr int kF8BM = 128;
constexpr int kF8OutBytesPerWarp = 2048;  // output staging per epilogue warp (32 x 32 bf16)
constexpr int kF8OutBytes = kF8EpiWarps * kF8OutBytesPerWarp;

template <int BN>
struct F8Cfg {
  static constexpr int kABytes = kF8BM * 128;
  static constexpr int kBBytes = BN * 128;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = (200 * 1024) / kStageBytes > 8 ? 8 : (200 * 1024) / kStageBytes;
  static constexpr int kBufs = 512 / BN;  // TMEM accumulators
  static constexpr int kCols = BN / 4;    // columns per epilogue warp
  static constexpr int kLd = 32;          // columns per TMEM load
  static constexpr uint32_t kIdesc = make_idesc(kFmtE4M3, kFmtE4M3, kF8BM, BN);
  static constexpr size_t kSmemBytes =
      size_t(kStages) * kStageBytes + kF8OutBytes + 1024 /*align*/ + 256 /*barriers*/;
  static_assert(kSmemBytes <= 232448, "shared memory per block");
  static_assert(BN == 128 || BN == 256, "N tile");
  static_assert(kCols % 32 == 0 && kCols % kLd == 0, "epilogue column split");
  static_assert((2 * kStages + 2 * kBufs + 1) * 8 + 16 <= 256, "barrier region");
};

struct F8Params {
  const float* a_scale;  // [M, G]
  const float* w_scale;  // [ceil(N/128), G]
  __nv_bfloat16* out;    // [M, N]
  int M, N, G;           // G = K / 128 (K groups = K blocks)
  int m_tiles, n_tiles;
  int splits;            // K splits per output tile (1 = none)
  float* part;           // splits > 1: [tiles * splits][kF8BM][BN] float32 partial tiles
  unsigned* counter;     // splits > 1: [tiles] arrival counters (left at zero)
  uint32_t wait_ns;            // bound of every wait (ns, below 2^32)
  int skip_it;                 // testing: CTA 0's producer skips this K-group iteration (-1: never)
  const uint8_t* wt;           // tiled weights (16 KiB tiles, see tile_weight_kernel), or null
};

__device__ __forceinline__ uint32_t f8_timer() {  // low word of %globaltimer (ns; wraps every 4.3 s)
  uint32_t t;
  asm volatile("mov.u32 %0, %%globaltimer_lo;" : "=r"(t));
  return t;
}
__device__ __forceinline__ uint32_t f8_ld_flag(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void f8_st_flag(uint32_t addr) {
  asm volatile("st.volatile.shared.u32 [%0], %1;" ::"r"(addr), "r"(1u) : "memory");
}

// try_wait that suspends the thread until the phase completes or hint_ns elapse: a
// waiting warp then takes no issue slots from the warps doing the work. The hint is kept
// short (1 us): measured on a B200, a 50 us hint left split-K calls 13-25 % slower (M = 96
// and 256 on 5120 x 6144) while the prefill shapes ran the same, so a suspended thread does
// not always resume as soon as the phase completes.
__device__ __forceinline__ bool f8_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}
constexpr uint32_t kF8SleepNs = 1000;

// Bounded wait with the limit of the launch (limit < 2^32 ns; differences of the low timer
// word are exact for intervals that short). Between checks of the abort flag and the
// clock the thread sleeps in try_wait for at most kF8SleepNs. On expiry it raises the
// CTA's abort flag (a shared-memory word) and the device status word; it also gives up
// once the flag is set.
__device__ __forceinline__ bool f8_wait(uint32_t bar, uint32_t parity, uint32_t abort_addr, uint32_t limit) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint32_t t0 = f8_timer();
  for (;;) {
    if (f8_try_wait_sleep(bar, parity, kF8SleepNs)) return true;
    if (f8_ld_flag(abort_addr)) return false;
    if (f8_timer() - t0 > limit) {
      f8_st_flag(abort_addr);
      atomicOr(&g_status, kStatusTimeout);
      return false;
    }
  }
}

// Drain wait: ignores the abort flag (waits for copies or MMAs already issued), bounded.
__device__ __forceinline__ void f8_drain(uint32_t bar, uint32_t parity, uint32_t limit) {
  const uint32_t t0 = f8_timer();
  while (!f8_try_wait_sleep(bar, parity, kF8SleepNs))
    if (f8_timer() - t0 > limit) {
      atomicOr(&g_status, kStatusTimeout);
      return;
    }
}

__device__ __forceinline__ void f8_epilogue_bar() { asm volatile("bar.sync 1, 512;" ::: "memory"); }

template <int kRegs>
__device__ __forceinline__ void f8_setmaxnreg_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegs)); }
template <int kRegs>
__device__ __forceinline__ void f8_setmaxnreg_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegs)); }

// acc[j], acc[j+1] += p0 * s, p1 * s: one packed instruction, each lane an IEEE fma (RN).
__device__ __forceinline__ void ffma2(float& a0, float& a1, uint32_t p0, uint32_t p1, float s) {
  unsigned long long acc, x, ss;
  asm("mov.b64 %0, {%1, %2};" : "=l"(acc) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "r"(p0), "r"(p1));
  asm("mov.b64 %0, {%1, %1};" : "=l"(ss) : "f"(s));
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(x), "l"(ss));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(acc));
}

__device__ __forceinline__ uint32_t f8_pack_bf16x2(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Output staging: each epilogue warp owns kF8OutBytesPerWarp of shared memory (32 rows x
// 32 bf16, the 64-byte-swizzled layout of a 32 x 32 TMA store box).

// Store this warp's 32 rows x kCols columns of bf16 output (rows row0.., columns col0..)
// through its staging buffer with TMA stores of 32 columns each: the tensor engine writes
// whole lines, where per-thread row stores would send 32 half-filled sectors per
// instruction. Before the buffer is rewritten, the previous store must have read it.
// The TMA store drops the parts of a box outside the output (M and N tails).
template <int kCols>
__device__ __forceinline__ void f8_store_tile_tma(const CUtensorMap* tm_out, uint32_t stage, int row0, int col0,
                                                  const float* acc) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int hh = 0; hh < kCols / 32; ++hh) {
    if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float* v = acc + 32 * hh + 8 * j;
      // 64-byte swizzle: 16-byte chunk j of row r sits at chunk j ^ ((r / 2) % 4) of its 64 bytes
      const uint32_t addr = stage + uint32_t(lane * 64 + 16 * (j ^ ((lane >> 1) & 3)));
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(f8_pack_bf16x2(v[0], v[1])),
                   "r"(f8_pack_bf16x2(v[2], v[3])), "r"(f8_pack_bf16x2(v[4], v[5])), "r"(f8_pack_bf16x2(v[6], v[7]))
                   : "memory");
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // visible to the tensor engine
    __syncwarp();
    if (lane == 0) {
      asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                       reinterpret_cast<uint64_t>(tm_out)),
                   "r"(col0 + 32 * hh), "r"(row0), "r"(stage)
                   : "memory");
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    }
  }
}

// Split K: store this split's partial tile, then finish the tile (splitk.cuh: the
// distributed sum when every CTA holds one item, else the last split to arrive sums it).
// Every epilogue thread calls this for every item (also after an abort), so the epilogue
// barriers always see all 512 threads.
template <int BN, int kCols>
__device__ __forceinline__ void f8_splitk(const F8Params& p, int item, int tile, int row_in_tile, int row, int col0,
                                          int cq, const float* acc, bool have, volatile int* flag,
                                          volatile int* abort_flag, int items) {
  if (have && row < p.M) {
    float* part_item = p.part + int64_t(item) * kF8BM * BN;
#pragma unroll
    for (int j = 0; j < kCols; j += 4)
      __stcg(reinterpret_cast<float4*>(splitk_quad(part_item, kF8BM, row_in_tile, cq * kCols + j)),
             make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]));
  }
  const int tm = tile % p.m_tiles, tn = tile / p.m_tiles;
  const int row0 = tm * kF8BM, tcol0 = tn * BN;
  SplitTile t;
  t.part = p.part + int64_t(tile) * p.splits * kF8BM * BN;
  t.split_elems = kF8BM * BN;
  t.bm = kF8BM;
  t.rows = min(kF8BM, p.M - row0);
  t.qpr = min(BN, p.N - tcol0) / 4;
  __nv_bfloat16* const out_t = p.out + int64_t(row0) * p.N + tcol0;
  const int ldo = p.N;
  auto store = [out_t, ldo](int r, int c, float4 s) {
    *reinterpret_cast<uint2*>(out_t + int64_t(r) * ldo + c) =
        make_uint2(f8_pack_bf16x2(s.x, s.y), f8_pack_bf16x2(s.z, s.w));
  };
  // after a timed-out wait nothing is published (the status word reports it; the caller
  // re-zeroes the workspace before reusing it)
  splitk_finish(p.counter + tile, t, p.splits, item - tile * p.splits, have && !*abort_flag, items,
                int(threadIdx.x) - 128, kF8EpiThreads, flag, p.wait_ns, &g_status, f8_epilogue_bar, store);
}

template <int BN, bool kSplitK>
__global__ void __launch_bounds__(kF8Threads, 1)
    gemm_fp8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmOut, const F8Params p) {
  using C = F8Cfg<BN>;
  constexpr int S = C::kStages;
  constexpr int NBUF = C::kBufs;
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // [S stages][output staging, 16 x 2 KiB][barriers]
  uint8_t* out_stage = smem + size_t(S) * C::kStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(out_stage + kF8OutBytes);
  // bars: full[S], empty[S], tfull[NBUF], tempty[NBUF], drain
  uint32_t* misc = reinterpret_cast<uint32_t*>(bars + 2 * S + 2 * NBUF + 1);
  uint32_t* tmem_slot = misc;
  const uint32_t abort_addr = smem_u32(misc + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  volatile int* split_flag = reinterpret_cast<volatile int*>(misc + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + S + s); };
  auto tfull_bar = [&](int b) { return smem_u32(bars + 2 * S + b); };
  auto tempty_bar = [&](int b) { return smem_u32(bars + 2 * S + NBUF + b); };
  const uint32_t drain_bar = smem_u32(bars + 2 * S + 2 * NBUF);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < NBUF; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), kF8EpiWarps);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // launch-time values before the grid-dependency wait (they do not depend on the
  // previous kernel), so their first parameter reads overlap it
  const uint32_t tmem_base = *tmem_slot;
  const int splits = kSplitK ? p.splits : 1;
  const int items = p.m_tiles * p.n_tiles * splits;
  const int KB = p.G;
  const uint32_t lim = p.wait_ns;
  pdl_wait();  // the previous kernel's results are visible from here

  if (warp < 4) {
    f8_setmaxnreg_dec<kF8ProducerRegs>();
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------------ TMA producer
      const int skip = blockIdx.x == 0 ? p.skip_it : -1;
      int it = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < items && ok; item += gridDim.x) {
        const int tile = item / splits, sp = item - tile * splits;
        const int kb0 = KB * sp / splits, kb1 = KB * (sp + 1) / splits;
        const int tm = tile % p.m_tiles, tn = tile / p.m_tiles;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % S;
          if (!f8_wait(empty_bar(s), ((it / S) & 1) ^ 1, abort_addr, lim)) {
            ok = false;
            break;
          }
          if (it == skip) continue;  // testing: this stage is never filled
          const uint32_t a_dst = smem_u32(smem + size_t(s) * C::kStageBytes);
          mbar_arrive_expect_tx(full_bar(s), C::kStageBytes);
          tma_load_2d(a_dst, &tmA, full_bar(s), kb * 128, tm * kF8BM);
          if (p.wt) {  // tiled weights: the BN / 128 tiles of this K group, each one contiguous copy
#pragma unroll
            for (int h = 0; h < BN / 128; ++h)
              bulk_load(a_dst + C::kABytes + 16384 * h,
                        p.wt + ((int64_t(tn) * (BN / 128) + h) * p.G + kb) * 16384, 16384, full_bar(s));
          } else {
            tma_load_2d(a_dst + C::kABytes, &tmB, full_bar(s), kb * 128, tn * BN);
          }
        }
      }
      // drain (bounded, regardless of abort): the last issue of every stage has landed.
      // Iterations 0 .. it-1 were issued (except a skipped one, whose stage still holds
      // the previous fill, consumed before the skip's empty wait passed).
      for (int j = it > S ? it - S : 0; j < it; ++j)
        if (j != skip) f8_drain(full_bar(j % S), (j / S) & 1, lim);
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      int it = 0, acc_it = 0;
      bool ok = true, issued = false;
      for (int item = blockIdx.x; item < items && ok; item += gridDim.x) {
        const int sp = item % splits;
        const int kb0 = KB * sp / splits, kb1 = KB * (sp + 1) / splits;
        for (int kb = kb0; kb < kb1; ++kb, ++it, ++acc_it) {
          const int s = it % S;
          const int b = acc_it % NBUF;
          if (!f8_wait(full_bar(s), (it / S) & 1, abort_addr, lim) ||
              !f8_wait(tempty_bar(b), ((acc_it / NBUF) & 1) ^ 1, abort_addr, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + size_t(s) * C::kStageBytes);
          const uint64_t adesc = sw128_kmajor_desc(a_addr);
          const uint64_t bdesc = sw128_kmajor_desc(a_addr + C::kABytes);
          const uint32_t d_tmem = tmem_base + uint32_t(b * BN);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) umma_f8f6f4(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, C::kIdesc, kk > 0);
          issued = true;
          umma_commit(empty_bar(s));  // the stage is free once these MMAs have read it
          umma_commit(tfull_bar(b));  // the group's partial is in TMEM
        }
      }
      if (issued) {  // every MMA issued by this thread has completed once drain_bar flips
        umma_commit(drain_bar);
        f8_drain(drain_bar, 0, lim);
      }
    }
  } else {
    f8_setmaxnreg_inc<kF8EpilogueRegs>();
    // ------------------------------------------------------------ epilogue warps 4..19
    constexpr int kCols = C::kCols;
    constexpr int kLd = C::kLd;
    const int q = warp & 3;                // TMEM lane quarter this warp may access
    const int cq = (warp - 4) >> 2;        // column quarter of the tile
    const int row_in_tile = 32 * q + lane;
    const uint32_t lane_addr = tmem_base + (uint32_t(32 * q) << 16) + uint32_t(cq * kCols);
    int acc_it = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < items && (kSplitK || ok); item += gridDim.x) {
      const int tile = item / splits, sp = item - tile * splits;
      const int kb0 = KB * sp / splits, kb1 = KB * (sp + 1) / splits;
      const int tm = tile % p.m_tiles, tn = tile / p.m_tiles;
      const int row = tm * kF8BM + row_in_tile;
      const int col0 = tn * BN + cq * kCols;
      float acc[kCols];
#pragma unroll
      for (int j = 0; j < kCols; ++j) acc[j] = 0.f;
      // Scales one group ahead (a_scale rows are L1 hits after the first touch). The loads
      // for group kb+1 are issued only after group kb's buffer release: the release of
      // mbarrier.arrive waits for this thread's outstanding loads, so a load issued before
      // it would put its latency on the hand-off to the MMA issuer.
      const int a_idx = (row < p.M ? row : 0) * KB;
      const int w_idx = (col0 < p.N ? (col0 >> 7) : 0) * KB;
      float sa_next = __ldg(p.a_scale + a_idx + kb0);
      float sw_next = __ldg(p.w_scale + w_idx + kb0);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (kSplitK && !ok) continue;
        const int b = acc_it % NBUF;
        if (!__all_sync(0xffffffffu, f8_wait(tfull_bar(b), (acc_it / NBUF) & 1, abort_addr, lim))) {
          ok = false;
          if (kSplitK) continue;
          break;
        }
        tc_fence_after();
        const uint32_t t_addr = lane_addr + uint32_t(b * BN);
        float sc = 0.f;
#pragma unroll
        for (int h = 0; h < kCols / kLd; ++h) {
          uint32_t r[kLd];
          tmem_ld_32x32b_x32(t_addr + uint32_t(kLd * h), r);
          tmem_ld_wait();
          if (h == 0) sc = sa_next * sw_next;
          if (h == kCols / kLd - 1) {  // the buffer's last columns are in registers: free it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty_bar(b));
            if (kb + 1 < kb1) {
              sa_next = __ldg(p.a_scale + a_idx + kb + 1);
              sw_next = __ldg(p.w_scale + w_idx + kb + 1);
            }
          }
#pragma unroll
          for (int j = 0; j < kLd; j += 2) ffma2(acc[kLd * h + j], acc[kLd * h + j + 1], r[j], r[j + 1], sc);
        }
        ++acc_it;
      }
      if constexpr (!kSplitK) {
        if (!ok) break;
        f8_store_tile_tma<kCols>(&tmOut, smem_u32(out_stage + (warp - 4) * kF8OutBytesPerWarp), tm * kF8BM + 32 * q,
                                 col0, acc);
      } else {
        f8_splitk<BN, kCols>(p, item, tile, row_in_tile, row, col0, cq, acc, ok, split_flag, abort_flag, items);
      }
    }
  }

  if (warp >= 4 && (threadIdx.x & 31) == 0)
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");  // this warp's output stores are complete
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ---------------------------------------------------------------- CTA-pair kernel
// The same promotion on pairs of SMs (a cluster of two CTAs, tcgen05 cta_group::2): the
// pair computes a 256 x 256 output tile with M = 256 MMAs issued by the leader CTA; each
// CTA stages its own 128 rows of A and its own 128 rows (output columns) of W, so per SM
// a K group moves 32 KiB into shared memory instead of 48 KiB for a 128 x 256 tile, and
// the tensor core reads 8 KiB of operands per MMA instead of 12 KiB. Each CTA's TMEM holds
// the fp32 partials of its 128 rows x 256 columns; its sixteen epilogue warps promote them
// exactly as in the single-CTA kernel.
//
// Protocol (both CTAs run the same roles; rank 0 issues the MMAs):
//   full[s]   each CTA: its own TMA bytes of stage s
//   full2[s]  leader: the peer's relay thread arrives once the peer's full[s] completed
//   empty[s]  each CTA: the leader's MMA commit (multicast to both) frees stage s
//   tfull[b]  each CTA: the leader's MMA commit (multicast) -- buffer b holds a partial
//   tempty[b] leader: 32 arrivals, one per epilogue warp of either CTA
// Every CTA drains its own TMA loads on its own barriers; a CTA whose wait gives up stops
// its own roles (the peer's waits then run out on their own); both CTAs meet at a cluster
// barrier before the TMEM is freed and before either exits, so no remote arrival or MMA
// can reach a finished CTA.
__device__ __forceinline__ uint32_t f8p_cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t f8p_mapa(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void f8p_cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrive on a barrier of another CTA of the cluster, with the default semantics of an
// arrive (release at CTA scope): a release at cluster scope would wait for every earlier
// global store of the thread (the output tiles) to become visible first. What the waiter
// needs ordered is already complete when this thread arrives: TMEM reads finished with
// tcgen05.wait::ld and fenced with tcgen05.fence::before_thread_sync, or TMA bytes that
// completed this CTA's own barrier.
__device__ __forceinline__ void f8p_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void f8p_tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void f8p_tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void f8p_tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void f8p_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on the barrier at this offset in every CTA of cta_mask once the MMAs issued so far
// have completed.
__device__ __forceinline__ void f8p_commit_mc(uint32_t bar, uint16_t cta_mask) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::
                   "r"(bar), "h"(cta_mask)
               : "memory");
}

constexpr int kF8PStages = 6;
constexpr int kF8PStageBytes = 2 * 128 * 128;  // own A box + own W box
constexpr size_t kF8PSmemBytes = size_t(kF8PStages) * kF8PStageBytes + kF8OutBytes + 1024 + 256;
static_assert(kF8PSmemBytes <= 232448, "shared memory per block");
static_assert((3 * kF8PStages + 4 + 4 + 1) * 8 + 16 <= 256, "barrier region");

// kHalves = 1: one M = 256, N = 256 MMA per K step into one of two 256-column TMEM
// buffers. kHalves = 2: two M = 256, N = 128 MMAs per K step, each into its own 128-column
// slot of a four-slot ring, so the tensor core can run one and a half K groups ahead of
// the promotion instead of one (the A operand is read twice per K step). In an N = 128
// MMA each CTA supplies 64 of its W rows: slot columns 0..63 are the leader's rows
// 64h .. 64h+63 of the pair tile, columns 64..127 the peer's rows 128+64h .. 128+64h+63.
template <int kHalves>
__global__ void __launch_bounds__(kF8Threads, 1)
    gemm_fp8_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                         const __grid_constant__ CUtensorMap tmOut, const F8Params p) {
  constexpr int S = kF8PStages;
  constexpr int BN = 256;
  constexpr int kCols = BN / 4;
  constexpr int kSlots = 2 * kHalves;          // TMEM accumulators
  constexpr int kSlotCols = 512 / kSlots;      // 256 or 128
  constexpr uint32_t kIdesc = make_idesc(kFmtE4M3, kFmtE4M3, 256, kSlotCols);
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* out_stage = smem + size_t(S) * kF8PStageBytes;  // 16 x 2 KiB output staging
  uint64_t* bars = reinterpret_cast<uint64_t*>(out_stage + kF8OutBytes);
  // bars: full[S], full2[S], empty[S], tfull[kSlots], tempty[kSlots], drain
  uint32_t* misc = reinterpret_cast<uint32_t*>(bars + 3 * S + 2 * kSlots + 1);
  uint32_t* tmem_slot = misc;
  const uint32_t abort_addr = smem_u32(misc + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = f8p_cluster_rank();
  const bool leader = rank == 0;
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto full2_bar = [&](int s) { return smem_u32(bars + S + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + 2 * S + s); };
  auto tfull_bar = [&](int b) { return smem_u32(bars + 3 * S + b); };
  auto tempty_bar = [&](int b) { return smem_u32(bars + 3 * S + kSlots + b); };
  const uint32_t drain_bar = smem_u32(bars + 3 * S + 2 * kSlots);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(full2_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < kSlots; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 2 * kF8EpiWarps / kHalves);  // the warps reading the slot, both CTAs
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  if (warp == 1) {
    f8p_tmem_alloc(smem_u32(tmem_slot), 512);
    f8p_tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  f8p_cluster_sync();  // both CTAs' barriers are initialised and their TMEM allocated
  tc_fence_after();
  pdl_wait();  // the previous kernel's results are visible from here
  const uint32_t tmem_base = *tmem_slot;

  const int clusters = int(gridDim.x >> 1);
  const int cid = int(blockIdx.x >> 1);
  const int items = p.m_tiles * p.n_tiles;
  const int KB = p.G;
  const uint32_t lim = p.wait_ns;

  if (warp < 4) {
    f8_setmaxnreg_dec<kF8ProducerRegs>();
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------------ TMA producer (both CTAs)
      const int skip = (cid == 0 && leader) ? p.skip_it : -1;
      int it = 0;
      bool ok = true;
      for (int item = cid; item < items && ok; item += clusters) {
        const int tm = item % p.m_tiles, tn = item / p.m_tiles;
        const int arow = tm * 256 + int(rank) * 128, brow = tn * 256 + int(rank) * 128;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % S;
          if (!f8_wait(empty_bar(s), ((it / S) & 1) ^ 1, abort_addr, lim)) {
            ok = false;
            break;
          }
          if (it == skip) continue;  // testing: this stage is never filled
          const uint32_t a_dst = smem_u32(smem + size_t(s) * kF8PStageBytes);
          mbar_arrive_expect_tx(full_bar(s), kF8PStageBytes);
          tma_load_2d(a_dst, &tmA, full_bar(s), kb * 128, arow);
          tma_load_2d(a_dst + 128 * 128, &tmB, full_bar(s), kb * 128, brow);
        }
      }
      for (int j = it > S ? it - S : 0; j < it; ++j)  // drain this CTA's own loads
        if (j != skip) f8_drain(full_bar(j % S), (j / S) & 1, lim);
    } else if (warp == 1 && lane == 0 && !leader) {
      // ------------------------------------------------------------ relay (peer)
      // tells the leader's MMA issuer that this CTA's half of stage s has landed
      const int n_its = (cid < items ? (items - cid + clusters - 1) / clusters : 0) * KB;
      for (int it = 0; it < n_its; ++it) {
        const int s = it % S;
        if (!f8_wait(full_bar(s), (it / S) & 1, abort_addr, lim)) break;
        f8p_arrive_remote(f8p_mapa(full2_bar(s), 0));
      }
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------------------ MMA issuer (leader)
      // one K group per iteration; accumulator slot u = kHalves * it + h cycles the ring
      const int n_its = (cid < items ? (items - cid + clusters - 1) / clusters : 0) * KB;
      bool issued = false, ok = true;
      for (int it = 0; it < n_its && ok; ++it) {
        const int s = it % S;
        if (!f8_wait(full_bar(s), (it / S) & 1, abort_addr, lim) ||
            !f8_wait(full2_bar(s), (it / S) & 1, abort_addr, lim))
          break;
        const uint32_t a_addr = smem_u32(smem + size_t(s) * kF8PStageBytes);
        const uint64_t adesc = sw128_kmajor_desc(a_addr);
#pragma unroll
        for (int h = 0; h < kHalves; ++h) {
          const int u = kHalves * it + h;
          const int b = u % kSlots;
          if (!f8_wait(tempty_bar(b), ((u / kSlots) & 1) ^ 1, abort_addr, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t bdesc = sw128_kmajor_desc(a_addr + 128 * 128 + h * 64 * 128);
          const uint32_t d_tmem = tmem_base + uint32_t(b * kSlotCols);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) f8p_mma(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, kIdesc, kk > 0);
          issued = true;
          f8p_commit_mc(tfull_bar(b), 0x3);  // both CTAs' slot b holds this part of the group's partial
        }
        if (!ok) break;
        f8p_commit_mc(empty_bar(s), 0x3);  // both CTAs' stage s is free once these MMAs have read it
      }
      if (issued) {  // every MMA issued by this thread has completed once drain_bar flips
        f8p_commit_mc(drain_bar, 0x1);
        f8_drain(drain_bar, 0, lim);
      }
    }
  } else {
    f8_setmaxnreg_inc<kF8EpilogueRegs>();
    // ------------------------------------------------------------ epilogue warps 4..19
    // warp (q, cq): TMEM lanes 32q..32q+31 (this CTA's rows) and 64 output columns. With
    // kHalves = 1 they are columns 64cq.. of the single slot; with kHalves = 2 the warp
    // reads slot half h = cq / 2, slot columns 64 (cq % 2).., which hold output columns
    // 128 (cq % 2) + 64 h.. of the pair tile.
    const int q = warp & 3;
    const int cq = (warp - 4) >> 2;
    const int h = kHalves == 2 ? (cq >> 1) : 0;
    const int slot_col = kHalves == 2 ? (cq & 1) * 64 : cq * 64;
    const int out_col = kHalves == 2 ? (cq & 1) * 128 + h * 64 : cq * 64;
    const int row_in_tile = 32 * q + lane;
    const uint32_t lane_addr = tmem_base + (uint32_t(32 * q) << 16) + uint32_t(slot_col);
    // the leader's tempty[0]; the others follow it (a CTA's shared window is contiguous)
    const uint32_t tempty_lead = f8p_mapa(tempty_bar(0), 0);
    int acc_it = 0;
    bool ok = true;
    for (int item = int(blockIdx.x >> 1); item < items && ok; item += int(gridDim.x >> 1)) {
      const int tm = item % p.m_tiles, tn = item / p.m_tiles;
      const int row = tm * 256 + int(blockIdx.x & 1u) * 128 + row_in_tile;  // cluster rank = blockIdx.x % 2
      const int col0 = tn * BN + out_col;
      float acc[kCols];
#pragma unroll
      for (int j = 0; j < kCols; ++j) acc[j] = 0.f;
      const int a_idx = (row < p.M ? row : 0) * KB;
      const int w_idx = (col0 < p.N ? (col0 >> 7) : 0) * KB;
      // scales one group ahead, requested after the release (see the single-CTA kernel)
      float sa_next = __ldg(p.a_scale + a_idx);
      float sw_next = __ldg(p.w_scale + w_idx);
      for (int kb = 0; kb < KB; ++kb) {
        const int u = kHalves * acc_it + h;
        const int b = u % kSlots;
        if (!__all_sync(0xffffffffu, f8_wait(tfull_bar(b), (u / kSlots) & 1, abort_addr, lim))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t t_addr = lane_addr + uint32_t(b * kSlotCols);
        float sc = 0.f;
#pragma unroll
        for (int c = 0; c < kCols / 32; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(t_addr + uint32_t(32 * c), r);
          tmem_ld_wait();
          if (c == 0) sc = sa_next * sw_next;
          if (c == kCols / 32 - 1) {  // this warp's columns are in registers: release its part
            tc_fence_before();
            __syncwarp();
            if (lane == 0) f8p_arrive_remote(tempty_lead + 8u * uint32_t(b));
            if (kb + 1 < KB) {
              sa_next = __ldg(p.a_scale + a_idx + kb + 1);
              sw_next = __ldg(p.w_scale + w_idx + kb + 1);
            }
          }
#pragma unroll
          for (int j = 0; j < 32; j += 2) ffma2(acc[32 * c + j], acc[32 * c + j + 1], r[j], r[j + 1], sc);
        }
        ++acc_it;
      }
      if (!ok) break;
      f8_store_tile_tma<kCols>(&tmOut, smem_u32(out_stage + (warp - 4) * kF8OutBytesPerWarp), row - lane, col0, acc);
    }
    if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");  // output stores complete
  }

  tc_fence_before();
  __syncthreads();
  f8p_cluster_sync();  // neither CTA frees TMEM or exits while the other may still reach it
  if (warp == 1) {
    tc_fence_after();
    f8p_tmem_dealloc(tmem_base, 512);
  }
}

// ---------------------------------------------------------------- host side
// Test hook: the wait bound and the skipped iteration of the next launches.
static std::atomic<uint32_t> g_f8_wait_ns{uint32_t(kWaitLimitNs)};
static std::atomic<int> g_f8_skip_it{-1};

void fp8_tc_set_test_fault(unsigned long long wait_ns, int skip_it) {
  // the kernel compares 32-bit timer differences: keep the bound below 2^31 ns
  g_f8_wait_ns.store(uint32_t(wait_ns == 0 ? kWaitLimitNs : std::min<unsigned long long>(wait_ns, 2000000000ull)));
  g_f8_skip_it.store(skip_it);
}

template <int BN, bool kSplitK>
static int launch_f8(const void* A, const void* W, const F8Params& prm, void* stream) {
  using C = F8Cfg<BN>;
  if (const int e = set_max_dynamic_smem(reinterpret_cast<const void*>(gemm_fp8_kernel<BN, kSplitK>),
                                         int(C::kSmemBytes)))
    return e;
  CUtensorMap ma, mb, mo;
  if (!make_tma_2d_kmajor(&ma, A, true, prm.M, int64_t(prm.G) * 128, kF8BM) ||
      !make_tma_2d_bf16_store(&mo, prm.out, prm.M, prm.N))
    return int(cudaErrorInvalidValue);
  if (prm.wt)
    mb = ma;  // (unused: the weight tiles are plain copies)
  else if (!make_tma_2d_kmajor(&mb, W, true, prm.N, int64_t(prm.G) * 128, BN))
    return int(cudaErrorInvalidValue);
  const int items = prm.m_tiles * prm.n_tiles * prm.splits;
  const int grid = std::min(items, device_sm_count());
  return launch_kernel(gemm_fp8_kernel<BN, kSplitK>, dim3(grid), dim3(kF8Threads), C::kSmemBytes, stream, ma, mb, mo,
                       prm);
}

// K splits: the configuration's split_k if set, else automatic -- split only when the
// output tiles leave most SMs idle, into enough splits to fill about one wave, at most 8
// and at least two K groups per split.
static int f8_splits(const KernelConfig& cfg, int64_t M, int64_t N, int64_t K) {
  const int64_t kb = K / 128;
  const int64_t tiles = ((M + kF8BM - 1) / kF8BM) * ((N + cfg.bn - 1) / cfg.bn);
  int64_t sp = cfg.split_k;
  if (sp <= 0) {
    const int64_t sms = device_sm_count();
    // one wave: tiles x splits <= SMs (a second, partial wave would double the time)
    sp = 2 * tiles >= sms ? 1 : std::min<int64_t>({sms / tiles, kb / 2, 8});
  }
  sp = std::max<int64_t>(1, std::min(sp, kb));
  if (sp > 1 && tiles > kMaxCounters) sp = 1;
  return int(sp);
}

// Clusters of two that can be resident at once (per device), for the persistent grid
// (both instantiations have the same resources).
static int f8p_max_clusters() {
  static int counts[64];
  static std::once_flag once[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::call_once(once[dev], [] {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 148);
    cfg.blockDim = dim3(kF8Threads);
    cfg.dynamicSmemBytes = kF8PSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_fp8_pair_kernel<1>, &cfg) != cudaSuccess) n = 0;
    int d = 0;
    cudaGetDevice(&d);
    counts[d] = n;
  });
  return counts[dev];
}

int fp8_pair_clusters() {
  if (set_max_dynamic_smem(reinterpret_cast<const void*>(gemm_fp8_pair_kernel<1>), int(kF8PSmemBytes)) ||
      set_max_dynamic_smem(reinterpret_cast<const void*>(gemm_fp8_pair_kernel<2>), int(kF8PSmemBytes)))
    return 0;
  return f8p_max_clusters();
}

int launch_fp8_pair(int halves, const void* A, const float* a_scale, const void* W, const float* w_scale, void* out,
                    int64_t M, int64_t N, int64_t K, void* stream) {
  if (M * (K / 128) >= (int64_t(1) << 31) || ((N + 127) / 128) * (K / 128) >= (int64_t(1) << 31))
    return int(cudaErrorInvalidValue);
  const int max_clusters = fp8_pair_clusters();
  if (max_clusters <= 0) return int(cudaErrorInvalidConfiguration);
  CUtensorMap ma, mb, mo;
  if (!make_tma_2d_kmajor(&ma, A, true, M, K, 128) || !make_tma_2d_kmajor(&mb, W, true, N, K, 128) ||
      !make_tma_2d_bf16_store(&mo, out, M, N))
    return int(cudaErrorInvalidValue);
  F8Params p{};
  p.a_scale = a_scale;
  p.w_scale = w_scale;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.M = int(M);
  p.N = int(N);
  p.G = int(K / 128);
  p.m_tiles = int((M + 255) / 256);
  p.n_tiles = int((N + 255) / 256);
  p.splits = 1;
  p.wait_ns = g_f8_wait_ns.load();
  p.skip_it = g_f8_skip_it.load();
  const int clusters = std::min(p.m_tiles * p.n_tiles, max_clusters);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(kF8Threads);
  cfg.dynamicSmemBytes = kF8PSmemBytes;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  return halves == 2 ? int(cudaLaunchKernelEx(&cfg, gemm_fp8_pair_kernel<2>, ma, mb, mo, p))
                     : int(cudaLaunchKernelEx(&cfg, gemm_fp8_pair_kernel<1>, ma, mb, mo, p));
}

size_t fp8_tc_workspace_bytes(int64_t M, int64_t N, int64_t K, const KernelConfig& cfg) {
  const int sp = f8_splits(cfg, M, N, K);
  if (sp == 1) return 0;
  const int64_t tiles = ((M + kF8BM - 1) / kF8BM) * ((N + cfg.bn - 1) / cfg.bn);
  return kCounterBytes + size_t(tiles) * sp * kF8BM * cfg.bn * sizeof(float);
}

int launch_fp8_tc(const KernelConfig& cfg, const void* A, const float* a_scale, const void* W, const float* w_scale,
                  void* out, int64_t M, int64_t N, int64_t K, void* ws, void* stream, bool tiled_w) {
  // the kernel indexes the scale matrices with 32-bit integers
  if (M * (K / 128) >= (int64_t(1) << 31) || ((N + 127) / 128) * (K / 128) >= (int64_t(1) << 31))
    return int(cudaErrorInvalidValue);
  F8Params p{};
  p.a_scale = a_scale;
  p.w_scale = w_scale;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.M = int(M);
  p.N = int(N);
  p.G = int(K / 128);
  p.m_tiles = int((M + kF8BM - 1) / kF8BM);
  p.n_tiles = int((N + cfg.bn - 1) / cfg.bn);
  p.splits = f8_splits(cfg, M, N, K);
  p.wait_ns = g_f8_wait_ns.load();
  p.skip_it = g_f8_skip_it.load();
  p.wt = tiled_w ? static_cast<const uint8_t*>(W) : nullptr;
  if (p.splits > 1) {
    if (!ws) return int(cudaErrorInvalidValue);
    p.counter = static_cast<unsigned*>(ws);
    p.part = reinterpret_cast<float*>(static_cast<char*>(ws) + kCounterBytes);
  }
  const bool split = p.splits > 1;
  switch (cfg.bn) {
    case 128: return split ? launch_f8<128, true>(A, W, p, stream) : launch_f8<128, false>(A, W, p, stream);
    case 256: return split ? launch_f8<256, true>(A, W, p, stream) : launch_f8<256, false>(A, W, p, stream);
    default: return int(cudaErrorInvalidValue);
  }
}

}  // namespace fp8bs
