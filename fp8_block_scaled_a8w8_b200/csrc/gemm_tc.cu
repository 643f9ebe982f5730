// Tensor-core GEMM for prefill-sized M: tcgen05.mma with TMEM accumulators, operands
// staged in shared memory by TMA (128-byte swizzle), persistent and warp-specialised.
//
//   warp 0        TMA producer: one 128-row A box and one BN-row W box per K block
//   warp 1        TMEM allocator and MMA issuer (one elected thread)
//   warps 4..11   epilogue: TMEM -> registers -> bf16/f32 -> global
//
// a8w8 block scale: a 128-wide K group is one K block. Each group's four
// tcgen05.mma (K = 32 each) write a fresh float32 partial P_g into one of two TMEM
// buffers; while the tensor core fills the other buffer with group g+1, the epilogue
// warps read P_g and add a_scale[row,g] * w_scale[col/128,g] * P_g into float32
// register accumulators -- the block-scale definition, group by group
// ([cookbook#8]: 128x128 weight blocks; 1x128 activation groups), with the
// scale promotion overlapped with the next group's MMAs.
// bf16: the K blocks (64 columns) accumulate in TMEM; the two buffers alternate
// between output tiles so the epilogue of one tile overlaps the next tile's MMAs.
//
// Every wait is bounded (kWaitLimitNs); a timed-out wait raises the CTA's abort flag
// and the device status word, the roles leave their loops, in-flight TMA loads and
// MMAs are drained (bounded) and TMEM is freed before the CTA exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"
#include "splitk.cuh"

namespace fp8bs {

FP8BS_DEFINE_STATUS(tc)

// 12 warps = 3 warpgroups. Warpgroup 0: warp 0 TMA producer, warp 1 TMEM allocator and MMA
// issuer, warps 2-3 idle. Warpgroups 1-2 (warps 4-11): epilogue. Registers are moved from
// warpgroup 0 to the epilogue with setmaxnreg: the launch gives every thread kLaunchRegs
// (checked by the build), 128 threads drop to kProducerRegs and 256 rise to kEpilogueRegs,
// which sums to exactly the launch's 384 * kLaunchRegs.
constexpr int kTcThreads = 384;
constexpr int kLaunchRegs = 168;
constexpr int kProducerRegs = 56;
constexpr int kEpilogueRegs = 224;
static_assert(128 * kProducerRegs + 256 * kEpilogueRegs <= kTcThreads * kLaunchRegs, "register split");
constexpr int kBM = 128;
constexpr int kKBlockBytes = 128;

template <bool kFp8, int BN>
struct TcCfg {
  static constexpr int kABytes = kBM * kKBlockBytes;
  static constexpr int kBBytes = BN * kKBlockBytes;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = (200 * 1024) / kStageBytes > 8 ? 8 : (200 * 1024) / kStageBytes;
  static constexpr int kTmemCols = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128 : (2 * BN <= 256) ? 256 : 512;
  static constexpr int kHalfCols = BN / 2;  // columns per epilogue warp
  static constexpr int kChunk = kHalfCols >= 32 ? 32 : kHalfCols;
  static constexpr int kChunks = kHalfCols / kChunk;
  static constexpr uint32_t kIdesc = make_idesc(kFp8 ? kFmtE4M3 : kFmtBF16, kFp8 ? kFmtE4M3 : kFmtBF16, kBM, BN);
  static constexpr size_t kSmemBytes = size_t(kStages) * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;
  static_assert(kHalfCols % kChunk == 0, "chunking");
  static_assert(BN % 16 == 0 && BN >= 32 && BN <= 256, "N tile");
};

struct TcParams {
  const float* a_scale;  // [M, G] (a8w8)
  const float* w_scale;  // [ceil(N/128), G] (a8w8)
  void* out;             // [M, N]
  int M, N, K;
  int kblocks;           // K blocks of 128 bytes
  int m_tiles, n_tiles;
  int out_fp32;
  int splits;            // K splits per output tile (1 = none)
  float* part;           // splits > 1: [tiles * splits][kBM][BN] float32 partial tiles
  unsigned* counter;     // splits > 1: [tiles] arrival counters (left at zero)
};

__device__ __forceinline__ void tc_epilogue_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld_chunk16(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

template <int kRegs>
__device__ __forceinline__ void setmaxnreg_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegs)); }
template <int kRegs>
__device__ __forceinline__ void setmaxnreg_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegs)); }

template <int kChunk>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&r)[32]) {
  if constexpr (kChunk == 32)
    tmem_ld_32x32b_x32(taddr, r);
  else
    tmem_ld_chunk16(taddr, r);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Store kChunk consecutive columns of one row (bf16 or f32), masked at N.
template <int kChunk>
__device__ __forceinline__ void store_row_chunk(const TcParams& p, int row, int col, const float* v) {
  if (row >= p.M) return;
  if (p.out_fp32) {
    float* dst = static_cast<float*>(p.out) + int64_t(row) * p.N + col;
#pragma unroll
    for (int j = 0; j < kChunk; j += 4)
      if (col + j < p.N) *reinterpret_cast<float4*>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
  } else {
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + int64_t(row) * p.N + col;
#pragma unroll
    for (int j = 0; j < kChunk; j += 8)
      if (col + j < p.N)
        *reinterpret_cast<uint4*>(dst + j) =
            make_uint4(pack_bf16x2(v[j], v[j + 1]), pack_bf16x2(v[j + 2], v[j + 3]), pack_bf16x2(v[j + 4], v[j + 5]),
                       pack_bf16x2(v[j + 6], v[j + 7]));
  }
}

// Split K: every split stores its float32 partial tile, then the tile is finished as
// splitk.cuh describes (the distributed sum when every CTA holds one item, else the last
// split to arrive sums it): the partials in split order, rounded once.
template <int BN, int kChunk>
__device__ __forceinline__ void tc_store_partial(const TcParams& p, int item, int row_in_tile, int col, int row,
                                                 const float* v) {
  if (row >= p.M) return;
  float* part_item = p.part + int64_t(item) * kBM * BN;
#pragma unroll
  for (int j = 0; j < kChunk; j += 4)
    __stcg(reinterpret_cast<float4*>(splitk_quad(part_item, kBM, row_in_tile, col + j)),
           make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]));
}

template <int BN>
__device__ __forceinline__ void tc_splitk_finish(const TcParams& p, int item, int tile, volatile int* flag,
                                                 volatile int* abort_flag, int items) {
  const int tm = tile % p.m_tiles, tn = tile / p.m_tiles;
  const int row0 = tm * kBM, tcol0 = tn * BN;
  SplitTile t;
  t.part = p.part + int64_t(tile) * p.splits * kBM * BN;
  t.split_elems = kBM * BN;
  t.bm = kBM;
  t.rows = min(kBM, p.M - row0);
  t.qpr = min(BN, p.N - tcol0) / 4;
  auto store = [&](int r, int c, float4 s) {
    const int64_t o = int64_t(row0 + r) * p.N + tcol0 + c;
    if (p.out_fp32)
      *reinterpret_cast<float4*>(static_cast<float*>(p.out) + o) = s;
    else
      *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.out) + o) =
          make_uint2(pack_bf16x2(s.x, s.y), pack_bf16x2(s.z, s.w));
  };
  // after a timed-out wait nothing is published (the status word reports it; the caller
  // re-zeroes the workspace before reusing it)
  splitk_finish(p.counter + tile, t, p.splits, item - tile * p.splits, !*abort_flag, items, int(threadIdx.x) - 128,
                256, flag, kWaitLimitNs, &g_status, tc_epilogue_bar, store);
}

// kSplitK: instantiated with split-K support; without it the kernel is exactly the
// one-split kernel (no split bookkeeping in the register budget of the hot loop).
template <bool kFp8, int BN, bool kSplitK>
__global__ void __launch_bounds__(kTcThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const TcParams p) {
  using C = TcCfg<kFp8, BN>;
  constexpr int S = C::kStages;
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tiles = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + size_t(S) * C::kStageBytes);
  // bars: full[S], empty[S], tmem_full[2], tmem_empty[2], drain
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* split_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);  // split-K finish

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + S + s); };
  auto tfull_bar = [&](int b) { return smem_u32(bars + 2 * S + b); };
  auto tempty_bar = [&](int b) { return smem_u32(bars + 2 * S + 2 + b); };
  const uint32_t drain_bar = smem_u32(bars + 2 * S + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 8);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // launch-time values before the grid-dependency wait (they do not depend on the
  // previous kernel), so their first parameter reads overlap it
  const uint32_t tmem_base = *tmem_slot;
  // work items: (output tile, K split); item -> tile = item / splits, K blocks [kb0, kb1)
  const int splits = kSplitK ? p.splits : 1;
  const int items = p.m_tiles * p.n_tiles * splits;
  const int KB = p.kblocks;
  const int G = p.K / 128;  // scale groups (a8w8)
  pdl_wait();  // the previous kernel's results are visible from here

  if (warp < 4) {
   setmaxnreg_dec<kProducerRegs>();  // warpgroup 0 hands registers to the epilogue
   if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int it = 0;
      int last_it[8];
      for (int s = 0; s < S; ++s) last_it[s] = -1;
      bool ok = true;
      for (int item = blockIdx.x; item < items && ok; item += gridDim.x) {
        const int tile = item / splits, sp = item - tile * splits;
        const int kb0 = KB * sp / splits, kb1 = KB * (sp + 1) / splits;
        const int tm = tile % p.m_tiles, tn = tile / p.m_tiles;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % S;
          if (!mbar_wait_bounded(empty_bar(s), ((it / S) & 1) ^ 1, abort_flag, &g_status)) {
            ok = false;
            break;
          }
          const uint32_t a_dst = smem_u32(tiles + size_t(s) * C::kStageBytes);
          const uint32_t b_dst = a_dst + C::kABytes;
          mbar_arrive_expect_tx(full_bar(s), C::kStageBytes);
          const int kx = kFp8 ? kb * 128 : kb * 64;
          tma_load_2d(a_dst, &tmA, full_bar(s), kx, tm * kBM);
          tma_load_2d(b_dst, &tmB, full_bar(s), kx, tn * BN);
          last_it[s] = it;
        }
      }
      // drain: wait (bounded, regardless of abort) for every issued load to land
      for (int s = 0; s < S; ++s) {
        if (last_it[s] < 0) continue;
        const uint32_t par = (last_it[s] / S) & 1;
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(full_bar(s), par))
          if (globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicOr(&g_status, kStatusTimeout);
            break;
          }
      }
    }
   } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int it = 0, acc_it = 0, tile_it = 0;
      bool ok = true;
      bool issued = false;
      for (int item = blockIdx.x; item < items && ok; item += gridDim.x, ++tile_it) {
        const int sp = item % splits;
        const int kb0 = KB * sp / splits, kb1 = KB * (sp + 1) / splits;
        uint32_t d_tmem = 0;
        int tb = tile_it & 1;
        if (!kFp8) {
          if (!mbar_wait_bounded(tempty_bar(tb), ((tile_it >> 1) & 1) ^ 1, abort_flag, &g_status)) break;
          tc_fence_after();
          d_tmem = tmem_base + uint32_t(tb * BN);
        }
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % S;
          if (!mbar_wait_bounded(full_bar(s), (it / S) & 1, abort_flag, &g_status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          int b = 0;
          if (kFp8) {
            b = acc_it & 1;
            if (!mbar_wait_bounded(tempty_bar(b), ((acc_it >> 1) & 1) ^ 1, abort_flag, &g_status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            d_tmem = tmem_base + uint32_t(b * BN);
          }
          const uint32_t a_addr = smem_u32(tiles + size_t(s) * C::kStageBytes);
          const uint64_t adesc = sw128_kmajor_desc(a_addr);
          const uint64_t bdesc = sw128_kmajor_desc(a_addr + C::kABytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t acc = kFp8 ? (kk > 0) : (kb > kb0 || kk > 0);
            if (kFp8)
              umma_f8f6f4(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, C::kIdesc, acc);
            else
              umma_f16(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, C::kIdesc, acc);
          }
          issued = true;
          umma_commit(empty_bar(s));
          if (kFp8) {
            umma_commit(tfull_bar(b));
            ++acc_it;
          }
        }
        if (!kFp8 && ok) umma_commit(tfull_bar(tb));
      }
      // drain: every MMA issued by this thread has completed once drain_bar flips
      if (issued) {
        umma_commit(drain_bar);
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(drain_bar, 0))
          if (globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicOr(&g_status, kStatusTimeout);
            break;
          }
      }
    }
   }
  } else {
    setmaxnreg_inc<kEpilogueRegs>();
    // ------------------------------------------------------------ epilogue warps 4..11
    const int q = warp & 3;          // TMEM lane quarter this warp may access
    const int h = (warp - 4) >> 2;   // column half
    const int row_in_tile = 32 * q + lane;
    const uint32_t lane_addr = tmem_base + (uint32_t(32 * q) << 16);
    int acc_it = 0, tile_it = 0;
    bool ok = true;
    // With split K every epilogue warp goes through every item, also after a timed-out wait
    // (then without touching TMEM or memory), so the epilogue barriers of the split-K
    // finish always see all eight warps.
    for (int item = blockIdx.x; item < items && (kSplitK || ok); item += gridDim.x, ++tile_it) {
      const int tile = item / splits, sp = item - tile * splits;
      const int kb0 = KB * sp / splits, kb1 = KB * (sp + 1) / splits;
      const int tm = tile % p.m_tiles, tn = tile / p.m_tiles;
      const int row = tm * kBM + row_in_tile;
      const int col0 = tn * BN + h * C::kHalfCols;
      if constexpr (kFp8) {
        float acc[C::kHalfCols];
#pragma unroll
        for (int j = 0; j < C::kHalfCols; ++j) acc[j] = 0.f;
        const int nbw = col0 >> 7;  // W scale block of this warp's columns
        const bool nb_ok = col0 < p.N;
        const float* asrow = p.a_scale + int64_t(row < p.M ? row : 0) * G;
        const bool row_ok = row < p.M;
        // a_scale of this row, four groups ahead (L1 hits after the first touch of the row)
        float sa0 = row_ok ? __ldg(asrow + kb0) : 0.f;
        float sa1 = (row_ok && kb0 + 1 < kb1) ? __ldg(asrow + kb0 + 1) : 0.f;
        float sa2 = (row_ok && kb0 + 2 < kb1) ? __ldg(asrow + kb0 + 2) : 0.f;
        float sa3 = (row_ok && kb0 + 3 < kb1) ? __ldg(asrow + kb0 + 3) : 0.f;
        float sw0 = nb_ok ? __ldg(p.w_scale + int64_t(nbw) * G + kb0) : 0.f;
        for (int kb = kb0; kb < kb1; ++kb) {
          const float sc = sa0 * sw0;
          sa0 = sa1;
          sa1 = sa2;
          sa2 = sa3;
          sa3 = (row_ok && kb + 4 < kb1) ? __ldg(asrow + kb + 4) : 0.f;
          sw0 = (nb_ok && kb + 1 < kb1) ? __ldg(p.w_scale + int64_t(nbw) * G + kb + 1) : 0.f;
          const int b = acc_it & 1;
          if (kSplitK && !ok) continue;
          if (!__all_sync(0xffffffffu, mbar_wait_bounded(tfull_bar(b), (acc_it >> 1) & 1, abort_flag, &g_status))) {
            ok = false;
            if (kSplitK) continue;
            break;
          }
          tc_fence_after();
          const uint32_t t_addr = lane_addr + uint32_t(b * BN + h * C::kHalfCols);
          // TMEM reads double-buffered: chunk c+1 is in flight while chunk c is scaled and
          // accumulated; the buffer is released as soon as its last chunk has landed
          uint32_t r0[32], r1[32];
          tmem_ld<C::kChunk>(t_addr, r0);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c) {
            uint32_t(&cur)[32] = (c & 1) ? r1 : r0;
            uint32_t(&nxt)[32] = (c & 1) ? r0 : r1;
            if (c + 1 < C::kChunks) tmem_ld<C::kChunk>(t_addr + (c + 1) * C::kChunk, nxt);
#pragma unroll
            for (int j = 0; j < C::kChunk; ++j)
              acc[c * C::kChunk + j] = fmaf(__uint_as_float(cur[j]), sc, acc[c * C::kChunk + j]);
            if (c + 1 < C::kChunks) {
              tmem_ld_wait();
              if (c + 2 == C::kChunks) {  // the last chunk is in registers: free the buffer
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(tempty_bar(b));
              }
            }
          }
          if (C::kChunks == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty_bar(b));
          }
          ++acc_it;
        }
        if (!kSplitK) {
          if (!ok) break;
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c) store_row_chunk<C::kChunk>(p, row, col0 + c * C::kChunk, acc + c * C::kChunk);
        } else {
          if (ok) {
#pragma unroll
            for (int c = 0; c < C::kChunks; ++c)
              tc_store_partial<BN, C::kChunk>(p, item, row_in_tile, h * C::kHalfCols + c * C::kChunk, row,
                                              acc + c * C::kChunk);
          }
          tc_splitk_finish<BN>(p, item, tile, split_flag, abort_flag, items);
        }
      } else {
        const int b = tile_it & 1;
        if (ok && !__all_sync(0xffffffffu, mbar_wait_bounded(tfull_bar(b), (tile_it >> 1) & 1, abort_flag, &g_status)))
          ok = false;
        if (!ok && !kSplitK) break;
        if (ok) {
          tc_fence_after();
          const uint32_t t_addr = lane_addr + uint32_t(b * BN + h * C::kHalfCols);
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c) {
            uint32_t r[32];
            tmem_ld<C::kChunk>(t_addr + c * C::kChunk, r);
            tmem_ld_wait();
            float v[C::kChunk];
#pragma unroll
            for (int j = 0; j < C::kChunk; ++j) v[j] = __uint_as_float(r[j]);
            if (!kSplitK)
              store_row_chunk<C::kChunk>(p, row, col0 + c * C::kChunk, v);
            else
              tc_store_partial<BN, C::kChunk>(p, item, row_in_tile, h * C::kHalfCols + c * C::kChunk, row, v);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tempty_bar(b));
        }
        if (kSplitK) tc_splitk_finish<BN>(p, item, tile, split_flag, abort_flag, items);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ---------------------------------------------------------------- host side
template <bool kFp8, int BN, bool kSplitK>
static int launch_tc_split(const void* A, const void* W, const TcParams& prm, void* stream) {
  using C = TcCfg<kFp8, BN>;
  if (const int attr = set_max_dynamic_smem(reinterpret_cast<const void*>(gemm_tc_kernel<kFp8, BN, kSplitK>),
                                            int(C::kSmemBytes)))
    return attr;
  CUtensorMap ma, mb;
  if (!make_tma_2d_kmajor(&ma, A, kFp8, prm.M, prm.K, kBM) || !make_tma_2d_kmajor(&mb, W, kFp8, prm.N, prm.K, BN))
    return int(cudaErrorInvalidValue);
  const int tiles = prm.m_tiles * prm.n_tiles * prm.splits;
  const int grid = std::min(tiles, device_sm_count());
  return launch_kernel(gemm_tc_kernel<kFp8, BN, kSplitK>, dim3(grid), dim3(kTcThreads), C::kSmemBytes, stream, ma, mb,
                       prm);
}

template <bool kFp8, int BN>
static int launch_tc_t(const void* A, const void* W, const TcParams& prm, void* stream) {
  return prm.splits > 1 ? launch_tc_split<kFp8, BN, true>(A, W, prm, stream)
                        : launch_tc_split<kFp8, BN, false>(A, W, prm, stream);
}

// K splits for a shape: the configuration's split_k if set, else automatic -- split only
// when the output tiles leave most SMs idle, into enough splits to fill about one wave, at
// most 8 and at least two K blocks per split (the partial tiles cost 8 bytes of traffic per
// output element per split).
static int tc_splits(const KernelConfig& cfg, int64_t M, int64_t N, int64_t K, bool fp8) {
  const int64_t kb = fp8 ? K / 128 : K / 64;
  const int64_t tiles = ((M + kBM - 1) / kBM) * ((N + cfg.bn - 1) / cfg.bn);
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

size_t tc_workspace_bytes(int op, int64_t M, int64_t N, int64_t K, const KernelConfig& cfg) {
  const bool fp8 = op == FP8BS_OP_A8W8_BLOCKSCALE;
  const int sp = tc_splits(cfg, M, N, K, fp8);
  if (sp == 1) return 0;
  const int64_t tiles = ((M + kBM - 1) / kBM) * ((N + cfg.bn - 1) / cfg.bn);
  return kCounterBytes + size_t(tiles) * sp * kBM * cfg.bn * sizeof(float);
}

static TcParams make_params(const float* a_scale, const float* w_scale, void* out, int64_t M, int64_t N, int64_t K,
                            int bn, bool fp8, int out_fp32) {
  TcParams p{};
  p.a_scale = a_scale;
  p.w_scale = w_scale;
  p.out = out;
  p.M = int(M);
  p.N = int(N);
  p.K = int(K);
  p.kblocks = int(fp8 ? K / 128 : K / 64);
  p.m_tiles = int((M + kBM - 1) / kBM);
  p.n_tiles = int((N + bn - 1) / bn);
  p.out_fp32 = out_fp32;
  p.splits = 1;
  return p;
}

static int set_splits(TcParams& p, const KernelConfig& cfg, bool fp8, void* ws) {
  p.splits = tc_splits(cfg, p.M, p.N, p.K, fp8);
  if (p.splits > 1) {
    if (!ws) return int(cudaErrorInvalidValue);
    p.counter = static_cast<unsigned*>(ws);
    p.part = reinterpret_cast<float*>(static_cast<char*>(ws) + kCounterBytes);
  }
  return 0;
}

int launch_tc_a8w8(const KernelConfig& cfg, const void* A, const float* a_scale, const void* W,
                   const float* w_scale, void* out, int64_t M, int64_t N, int64_t K, void* ws, void* stream) {
  TcParams p = make_params(a_scale, w_scale, out, M, N, K, cfg.bn, true, 0);
  if (const int e = set_splits(p, cfg, true, ws)) return e;
  switch (cfg.bn) {
    case 128: return launch_tc_t<true, 128>(A, W, p, stream);
    case 256: return launch_tc_t<true, 256>(A, W, p, stream);
    default: return int(cudaErrorInvalidValue);
  }
}

int launch_tc_bf16(const KernelConfig& cfg, const void* A, const void* W, void* out, int out_fp32, int64_t M,
                   int64_t N, int64_t K, void* ws, void* stream) {
  TcParams p = make_params(nullptr, nullptr, out, M, N, K, cfg.bn, false, out_fp32);
  if (const int e = set_splits(p, cfg, false, ws)) return e;
  switch (cfg.bn) {
    case 32: return launch_tc_t<false, 32>(A, W, p, stream);
    case 64: return launch_tc_t<false, 64>(A, W, p, stream);
    case 128: return launch_tc_t<false, 128>(A, W, p, stream);
    case 192: return launch_tc_t<false, 192>(A, W, p, stream);
    case 256: return launch_tc_t<false, 256>(A, W, p, stream);
    default: return int(cudaErrorInvalidValue);
  }
}

}  // namespace fp8bs
