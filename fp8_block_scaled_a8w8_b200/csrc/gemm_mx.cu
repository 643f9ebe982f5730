// MX32 variant of the a8w8 GEMM on the tensor core's own block scaling: tcgen05.mma
// kind::mxf8f6f4.block_scale with E8M0 scale factors in TMEM.
//
//   out[b,m,n] = sum_g 2^(ea[b,m,g] + ew[b,n/32,g] - 254) * sum_{k in g} A[b,m,k] W[b,n,k]
//
// with 32-wide K groups g, 1x32 activation scales and 32x32 weight-block scales
// ([aiter#7247] "Motivation": MX32, w_scale_block 32x32; "Technical Details": the dense
// shapes and the batched b = 8, N = 1024, K = 4096 GEMM). Because the scales are powers of
// two the hardware applies them inside the MMA, so the fp32 accumulator stays in TMEM
// over the whole K range -- no per-group promotion by the epilogue, unlike the fp32-scale
// 128-block kernels.
//
// Tiles of 128 rows x 192 columns, persistent CTAs, K staged 128 at a time (four K = 32
// MMAs, each selecting its scale byte with the instruction's scale-factor ids).
//   warp 0        TMA producer: A box 128 rows x 128 bytes, W box 192 rows x 128 bytes
//   warp 1        TMEM allocator and MMA issuer
//   warps 4..7    scale-factor writers: per stage, tcgen05.st of the tile's scale bytes
//                 into a TMEM slot -- row m at lane m % 32 of every 32-lane subpartition,
//                 column m / 32, one byte per K group (measured layout of the block-scaled
//                 MMA's scale-factor operands)
//   warps 8..15   epilogue: TMEM -> bf16 -> shared memory -> TMA store (two TMEM
//                 accumulators alternate between tiles)
// Small tile counts split K: each split stores the rows < M of its fp32 tile and the tile
// is finished as splitk.cuh describes (partials summed in split order, rounded once).
// Every wait is bounded; on expiry the CTA raises its abort flag and the status word,
// drains what it issued and frees TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>

#include "internal.h"
#include "ptx.cuh"
#include "splitk.cuh"

namespace fp8bs {

FP8BS_DEFINE_STATUS(mx)

constexpr int kMxThreads = 512;
constexpr int kMxBM = 128;
constexpr int kMxStages = 4;
constexpr int kMxABytes = kMxBM * 128;
constexpr int kMxEpiWarps = 8;
constexpr int kMxOutBytes = kMxEpiWarps * 2048;  // one 32 x 32 bf16 staging box per epilogue warp
// scale-byte prefetch ring of each scale-factor writer warp: 128 activation-row words +
// 8 weight-block words per stage, kMxSfAhead stages in flight
constexpr int kMxSfSlotBytes = 512 + 32;
constexpr int kMxSfRing = 8, kMxSfAhead = 6;
constexpr int kMxSfBytes = kMxSfRing * kMxSfSlotBytes;
// Tile width BN: 192 with two TMEM accumulators alternating between tiles, or 256 with
// one (for launches whose tiles fit one wave, where no CTA has a next tile to overlap).
template <int BN>
struct MxCfg {
  static constexpr int kBBytes = BN * 128;
  static constexpr int kStageBytes = kMxABytes + kBBytes;
  static constexpr int kBufs = (2 * BN + 32 * kMxStages <= 512) ? 2 : 1;
  static constexpr uint32_t kSfBase = uint32_t(kBufs * BN);  // TMEM: [accumulators][scale-factor slots, 32 columns]
  static constexpr size_t kSmemBytes = size_t(kMxStages) * kStageBytes + kMxOutBytes + kMxSfBytes + 1024 + 256;
  static_assert(BN == 192 || BN == 256, "tile width");
  static_assert(kSfBase + 32 * kMxStages <= 512, "TMEM budget");
  static_assert(kStageBytes % 1024 == 0, "stage alignment");
  static_assert(kSmemBytes <= 232448, "shared memory per block");
  static_assert(BN / 32 <= 8, "weight-block scale words per stage");
};

struct MxParams {
  const uint8_t* a_e;   // [batch][M][K/32] E8M0
  const uint8_t* w_e;   // [batch][ceil(N/32)][K/32] E8M0
  __nv_bfloat16* out;   // [batch][M][N]
  int M, N, K32, KB, NB32, batch;
  int m_tiles, n_tiles, splits;
  float* part;          // splits > 1: [items][kMxBM][BN] float32 partial tiles
  unsigned* counter;    // splits > 1: [tiles]
  uint32_t wait_ns;
};

// Block-scaled instruction descriptor: E4M3 x E4M3, both K-major, E8M0 scale factors
// (bit 23), B scale-factor id at bits 4-5, A's at bits 29-30, N >> 3 at 17-22, M >> 4 at 24-28.
__host__ __device__ constexpr uint32_t mx_idesc(uint32_t m, uint32_t n, uint32_t sf_id) {
  return (sf_id << 4) | ((n >> 3) << 17) | (1u << 23) | ((m >> 4) << 24) | (sf_id << 29);
}

__device__ __forceinline__ void mx_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                       uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(sfa), "r"(sfb), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void mx_tmem_st_x4(uint32_t taddr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}
__device__ __forceinline__ void mx_tmem_st_x8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}
__device__ __forceinline__ void mx_tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void mx_tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y,
                                               int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}

__device__ __forceinline__ uint32_t mx_timer() {
  uint32_t t;
  asm volatile("mov.u32 %0, %%globaltimer_lo;" : "=r"(t));
  return t;
}
// Bounded wait (sleeping in try_wait, at most 1 us at a time, between checks of the abort
// flag and the clock; a longer suspend hint delays some resumes, as in the a8w8 kernels).
__device__ __forceinline__ bool mx_wait(uint32_t bar, uint32_t parity, volatile int* abort, uint32_t limit) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint32_t t0 = mx_timer();
  for (;;) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(1000u)
        : "memory");
    if (ok) return true;
    if (*abort) return false;
    if (mx_timer() - t0 > limit) {
      *abort = 1;
      atomicOr(&g_status, kStatusTimeout);
      return false;
    }
  }
}
__device__ __forceinline__ void mx_drain(uint32_t bar, uint32_t parity, uint32_t limit) {
  const uint32_t t0 = mx_timer();
  while (!mbar_try_wait(bar, parity))
    if (mx_timer() - t0 > limit) {
      atomicOr(&g_status, kStatusTimeout);
      return;
    }
}

__device__ __forceinline__ uint32_t mx_pack_bf16x2(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ void mx_epi_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
// Barrier of the four scale-factor writer warps that also ANDs a flag over their threads,
// so that all four leave their loop together (a warp that left alone would strand the
// others at the next barrier).
__device__ __forceinline__ bool mx_sf_bar_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 3, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(uint32_t(v))
      : "memory");
  return r != 0;
}

// item -> (split, tile); tile -> (tm fastest, tn, batch)
struct MxItem {
  int sp, tile, tm, tn, bt, kb0, kb1;
};
__device__ __forceinline__ MxItem mx_item(const MxParams& p, int item) {
  MxItem r;
  r.tile = item / p.splits;
  r.sp = item - r.tile * p.splits;
  r.tm = r.tile % p.m_tiles;
  const int rest = r.tile / p.m_tiles;
  r.tn = rest % p.n_tiles;
  r.bt = rest / p.n_tiles;
  r.kb0 = p.KB * r.sp / p.splits;
  r.kb1 = p.KB * (r.sp + 1) / p.splits;
  return r;
}

// Walks this CTA's stages (item, K block) in order.
struct MxStageIter {
  MxItem w;
  int item, kb;
  bool valid;
  __device__ MxStageIter(const MxParams& p, int items) : item(blockIdx.x) {
    valid = item < items;
    if (valid) {
      w = mx_item(p, item);
      kb = w.kb0;
    }
  }
  __device__ void advance(const MxParams& p, int items) {
    if (++kb < w.kb1) return;
    item += gridDim.x;
    valid = item < items;
    if (valid) {
      w = mx_item(p, item);
      kb = w.kb0;
    }
  }
};

template <bool kSplitK, int BN>
__global__ void __launch_bounds__(kMxThreads, 1)
    gemm_mx_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmOut, const MxParams p) {
  using C = MxCfg<BN>;
  constexpr int S = kMxStages;
  constexpr int NB = C::kBufs;
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* out_stage = smem + size_t(S) * C::kStageBytes;
  uint8_t* sf_ring = out_stage + kMxOutBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sf_ring + kMxSfBytes);
  // bars: full[S], empty[S], sf_full[S], tfull[2], tempty[2], drain
  uint32_t* misc = reinterpret_cast<uint32_t*>(bars + 3 * S + 5);
  uint32_t* tmem_slot = misc;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  volatile int* split_flag = reinterpret_cast<volatile int*>(misc + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + S + s); };
  auto sf_full_bar = [&](int s) { return smem_u32(bars + 2 * S + s); };
  auto tfull_bar = [&](int b) { return smem_u32(bars + 3 * S + b); };
  auto tempty_bar = [&](int b) { return smem_u32(bars + 3 * S + 2 + b); };
  const uint32_t drain_bar = smem_u32(bars + 3 * S + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
      mbar_init(sf_full_bar(s), 4);  // the four scale-factor writer warps
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), kMxEpiWarps);
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
  const int items = p.batch * p.m_tiles * p.n_tiles * splits;
  const uint32_t lim = p.wait_ns;
  pdl_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < items && ok; item += gridDim.x) {
        const MxItem w = mx_item(p, item);
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
          const int s = it % S;
          if (!mx_wait(empty_bar(s), ((it / S) & 1) ^ 1, abort_flag, lim)) {
            ok = false;
            break;
          }
          const uint32_t dst = smem_u32(smem + size_t(s) * C::kStageBytes);
          mbar_arrive_expect_tx(full_bar(s), C::kStageBytes);
          mx_tma_load_3d(dst, &tmA, full_bar(s), kb * 128, w.tm * kMxBM, w.bt);
          mx_tma_load_3d(dst + kMxABytes, &tmB, full_bar(s), kb * 128, w.tn * BN, w.bt);
        }
      }
      for (int j = it > S ? it - S : 0; j < it; ++j) mx_drain(full_bar(j % S), (j / S) & 1, lim);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int it = 0, tile_it = 0;
      bool ok = true, issued = false;
      for (int item = blockIdx.x; item < items && ok; item += gridDim.x, ++tile_it) {
        const MxItem w = mx_item(p, item);
        const int b = tile_it % NB;
        if (!mx_wait(tempty_bar(b), ((tile_it / NB) & 1) ^ 1, abort_flag, lim)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + uint32_t(b * BN);
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
          const int s = it % S;
          if (!mx_wait(full_bar(s), (it / S) & 1, abort_flag, lim) ||
              !mx_wait(sf_full_bar(s), (it / S) & 1, abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + size_t(s) * C::kStageBytes);
          const uint64_t adesc = sw128_kmajor_desc(a_addr), bdesc = sw128_kmajor_desc(a_addr + kMxABytes);
          const uint32_t sfa = tmem_base + C::kSfBase + uint32_t(32 * s), sfb = sfa + 16;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mx_mma(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, mx_idesc(kMxBM, BN, kk), sfa, sfb,
                   (kb > w.kb0 || kk > 0) ? 1u : 0u);
          issued = true;
          umma_commit(empty_bar(s));  // the stage and its scale-factor slot are free
        }
        if (ok) umma_commit(tfull_bar(b));
      }
      if (issued) {
        umma_commit(drain_bar);
        mx_drain(drain_bar, 0, lim);
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ scale-factor writers
    // Warp q writes TMEM lanes 32q..32q+31 (every subpartition holds the same copy). The
    // scale bytes come from global memory (L2) with a latency of several stages, so the
    // four warps copy them kMxSfAhead stages ahead with cp.async into one shared-memory
    // ring: per stage warp q fetches activation rows 32q .. 32q+31 (4 bytes = 4 K groups
    // each) and warp 4 the tile's 6 weight blocks, one commit group per stage; a barrier of
    // the four warps then makes every row visible to all of them.
    const int q = warp & 3;
    const uint32_t lane_addr = tmem_base + (uint32_t(32 * q) << 16);
    const uint32_t ring = smem_u32(sf_ring);
    MxStageIter use_it(p, items), fetch_it(p, items);
    auto fetch = [&](int slot) {
      if (fetch_it.valid) {
        const MxItem& w = fetch_it.w;
        const uint8_t* arow = p.a_e + (int64_t(w.bt) * p.M) * p.K32 + 4 * fetch_it.kb;
        const uint8_t* wrow = p.w_e + (int64_t(w.bt) * p.NB32) * p.K32 + 4 * fetch_it.kb;
        const uint32_t base = ring + slot * kMxSfSlotBytes;
        const int r = min(w.tm * kMxBM + 32 * q + lane, p.M - 1);  // rows past M: any valid row
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(base + 4 * (32 * q + lane)),
                     "l"(arow + int64_t(r) * p.K32)
                     : "memory");
        if (q == 0 && lane < BN / 32) {
          const int nb = min(w.tn * (BN / 32) + lane, p.NB32 - 1);
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(base + 512 + 4 * lane),
                       "l"(wrow + int64_t(nb) * p.K32)
                       : "memory");
        }
        fetch_it.advance(p, items);
      }
      asm volatile("cp.async.commit_group;" ::: "memory");  // one group per stage, empty past the end
    };
#pragma unroll 1
    for (int d = 0; d < kMxSfAhead; ++d) fetch(d % kMxSfRing);
    int it = 0;
    for (; use_it.valid; ++it) {
      fetch((it + kMxSfAhead) % kMxSfRing);
      asm volatile("cp.async.wait_group %0;" ::"n"(kMxSfAhead) : "memory");  // this warp's bytes of stage it
      const int s = it % S;
      const bool ok = __all_sync(0xffffffffu, mx_wait(empty_bar(s), ((it / S) & 1) ^ 1, abort_flag, lim));
      if (!mx_sf_bar_and(ok)) break;  // the other three warps' bytes too (the ring slot is complete)
      const uint32_t base = ring + (it % kMxSfRing) * kMxSfSlotBytes;
      uint32_t sa[4], sb[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) asm volatile("ld.shared.u32 %0, [%1];" : "=r"(sa[j]) : "r"(base + 4 * (32 * j + lane)));
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        sb[j] = 0x7F7F7F7Fu;
        if (j < BN / 32) asm volatile("ld.shared.u32 %0, [%1];" : "=r"(sb[j]) : "r"(base + 512 + 4 * j));
      }
      tc_fence_after();
      const uint32_t slot = lane_addr + C::kSfBase + uint32_t(32 * s);
      mx_tmem_st_x4(slot, sa[0], sa[1], sa[2], sa[3]);  // column j: rows 32j + lane
      mx_tmem_st_x8(slot + 16, sb);                      // column j: output columns 32j .. 32j + 31
      mx_tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sf_full_bar(s));
      use_it.advance(p, items);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // nothing in flight into the ring at exit
  } else if (warp >= 8) {
    // ------------------------------------------------------------ epilogue warps 8..15
    const int e = warp - 8, q = warp & 3, h = e >> 2;  // lane quarter, 96-column half
    const uint32_t lane_addr = tmem_base + (uint32_t(32 * q) << 16);
    const uint32_t stage = smem_u32(out_stage + e * 2048);
    int tile_it = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < items && (kSplitK || ok); item += gridDim.x, ++tile_it) {
      const MxItem w = mx_item(p, item);
      const int b = tile_it % NB;
      const int row0 = w.tm * kMxBM + 32 * q;
      const int col_base = w.tn * BN + h * (BN / 2);
      if (ok && !__all_sync(0xffffffffu, mx_wait(tfull_bar(b), (tile_it / NB) & 1, abort_flag, lim))) ok = false;
      if (ok) {
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < BN / 64; ++c) {  // chunks of 32 columns
          uint32_t r[32];
          tmem_ld_32x32b_x32(lane_addr + uint32_t(b * BN + h * (BN / 2) + 32 * c), r);
          tmem_ld_wait();
          if (c == BN / 64 - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty_bar(b));
          }
          const int col0 = col_base + 32 * c;
          if constexpr (!kSplitK) {
            if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t addr = stage + uint32_t(lane * 64 + 16 * (j ^ ((lane >> 1) & 3)));
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                           "r"(mx_pack_bf16x2(__uint_as_float(r[8 * j]), __uint_as_float(r[8 * j + 1]))),
                           "r"(mx_pack_bf16x2(__uint_as_float(r[8 * j + 2]), __uint_as_float(r[8 * j + 3]))),
                           "r"(mx_pack_bf16x2(__uint_as_float(r[8 * j + 4]), __uint_as_float(r[8 * j + 5]))),
                           "r"(mx_pack_bf16x2(__uint_as_float(r[8 * j + 6]), __uint_as_float(r[8 * j + 7])))
                           : "memory");
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) {
              asm volatile(
                  "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
                      reinterpret_cast<uint64_t>(&tmOut)),
                  "r"(col0), "r"(row0), "r"(w.bt), "r"(stage)
                  : "memory");
              asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            }
          } else {
            const int row = row0 + lane;
            if (row < p.M) {
              float* part_item = p.part + int64_t(item) * kMxBM * BN;
#pragma unroll
              for (int j = 0; j < 32; j += 4)
                __stcg(reinterpret_cast<float4*>(splitk_quad(part_item, kMxBM, 32 * q + lane, h * (BN / 2) + 32 * c + j)),
                       make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]), __uint_as_float(r[j + 2]),
                                   __uint_as_float(r[j + 3])));
            }
          }
        }
      }
      if constexpr (kSplitK) {
        // publish this split and finish the tile (splitk.cuh): the partials in split order
        const int trow0 = w.tm * kMxBM, tcol0 = w.tn * BN;
        SplitTile t;
        t.part = p.part + int64_t(w.tile) * p.splits * kMxBM * BN;
        t.split_elems = kMxBM * BN;
        t.bm = kMxBM;
        t.rows = min(kMxBM, p.M - trow0);
        t.qpr = min(BN, p.N - tcol0) / 4;
        __nv_bfloat16* out_t = p.out + (int64_t(w.bt) * p.M + trow0) * p.N + tcol0;
        auto store = [&](int r, int c, float4 s) {
          *reinterpret_cast<uint2*>(out_t + int64_t(r) * p.N + c) =
              make_uint2(mx_pack_bf16x2(s.x, s.y), mx_pack_bf16x2(s.z, s.w));
        };
        splitk_finish(p.counter + w.tile, t, p.splits, w.sp, ok && !*abort_flag, items,
                      int(threadIdx.x) - 256, 256, split_flag, lim, &g_status, mx_epi_bar, store);
      } else {
        if (!ok) break;
      }
    }
    if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ---------------------------------------------------------------- host side
static bool make_map_3d(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, int esz, int64_t inner, int64_t rows,
                        int64_t batch, int box_inner, int box_rows, CUtensorMapSwizzle sw) {
  static PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  if (!enc) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  cuuint64_t dims[3] = {cuuint64_t(inner), cuuint64_t(rows), cuuint64_t(batch)};
  cuuint64_t strides[2] = {cuuint64_t(inner * esz), cuuint64_t(inner * rows * esz)};
  cuuint32_t box[3] = {cuuint32_t(box_inner), cuuint32_t(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  std::memset(m, 0, sizeof(*m));
  return enc(m, dt, 3, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// K splits of a one-wave split launch: as many as keep tiles x splits within the SMs, at
// most 8 (the finish loads every split of an element at once), each at least 2 K blocks.
static int64_t mx_auto_splits(int64_t tiles, int64_t kb) {
  const int64_t sms = device_sm_count();
  int64_t sp = 2 * tiles >= sms ? 1 : std::min<int64_t>({sms / tiles, kb / 2, 8});
  sp = std::max<int64_t>(1, std::min(sp, kb));
  if (sp > 1 && tiles > kMaxCounters) sp = 1;
  return sp;
}

// Tile width: 192 (two accumulators, tiles overlap on a persistent grid), unless 192-wide
// tiles would spill into a partial second wave that 256-wide tiles avoid (e.g. M = 768,
// N = 5120: 162 tiles of 192 on 148 SMs, 120 of 256); then 256 with one accumulator. A
// single GEMM whose 192-wide tiles split K also takes 256-wide tiles when their split
// leaves each CTA fewer K stages, a 256-wide stage counted as 1.15 of a 192-wide one
// (measured on a B200: M = 768, N = 1792, K = 5120 20.3 -> 18.6 us; M = 48, N = 4608 12.4
// -> 11.9 us; batched calls ran 2-4 % slower, so they keep 192).
static int mx_bn(int64_t batch, int64_t M, int64_t N, int64_t K) {
  const int64_t sms = device_sm_count();
  const int64_t mt = batch * ((M + kMxBM - 1) / kMxBM);
  const int64_t t192 = mt * ((N + 191) / 192), t256 = mt * ((N + 255) / 256);
  if (t192 > sms && t256 <= sms) return 256;
  if (batch == 1 && 2 * t192 < sms) {
    const int64_t kb = K / 128;
    const int64_t s192 = mx_auto_splits(t192, kb), s256 = mx_auto_splits(t256, kb);
    if (115 * ((kb + s256 - 1) / s256) < 100 * ((kb + s192 - 1) / s192)) return 256;
  }
  return 192;
}

static int mx_splits(int64_t batch, int64_t M, int64_t N, int64_t K) {
  const int bn = mx_bn(batch, M, N, K);
  return int(mx_auto_splits(batch * ((M + kMxBM - 1) / kMxBM) * ((N + bn - 1) / bn), K / 128));
}

size_t mx_workspace_bytes(int64_t batch, int64_t M, int64_t N, int64_t K) {
  const int sp = mx_splits(batch, M, N, K);
  if (sp == 1) return 0;
  const int bn = mx_bn(batch, M, N, K);
  const int64_t tiles = batch * ((M + kMxBM - 1) / kMxBM) * ((N + bn - 1) / bn);
  return kCounterBytes + size_t(tiles) * sp * kMxBM * bn * sizeof(float);
}

int launch_gemm_mx32(const void* A, const uint8_t* a_e, const void* W, const uint8_t* w_e, void* out, int64_t batch,
                     int64_t M, int64_t N, int64_t K, void* ws, void* stream, unsigned wait_ns) {
  MxParams p{};
  p.a_e = a_e;
  p.w_e = w_e;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.M = int(M);
  p.N = int(N);
  p.K32 = int(K / 32);
  p.KB = int(K / 128);
  p.NB32 = int((N + 31) / 32);
  p.batch = int(batch);
  p.m_tiles = int((M + kMxBM - 1) / kMxBM);
  const int bn = mx_bn(batch, M, N, K);
  p.n_tiles = int((N + bn - 1) / bn);
  p.splits = mx_splits(batch, M, N, K);
  p.wait_ns = wait_ns;
  if (p.splits > 1) {
    if (!ws) return int(cudaErrorInvalidValue);
    p.counter = static_cast<unsigned*>(ws);
    p.part = reinterpret_cast<float*>(static_cast<char*>(ws) + kCounterBytes);
  }
  CUtensorMap ma, mb, mo;
  if (!make_map_3d(&ma, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, M, batch, 128, kMxBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_3d(&mb, W, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, N, batch, 128, bn, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_3d(&mo, out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, M, batch, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
    return int(cudaErrorInvalidValue);
  const int items = p.batch * p.m_tiles * p.n_tiles * p.splits;
  const int grid = std::min(items, device_sm_count());
  auto go = [&](auto kernel, size_t smem) {
    if (const int e = set_max_dynamic_smem(reinterpret_cast<const void*>(kernel), int(smem))) return e;
    return launch_kernel(kernel, dim3(grid), dim3(kMxThreads), smem, stream, ma, mb, mo, p);
  };
  if (bn == 256)
    return p.splits > 1 ? go(gemm_mx_kernel<true, 256>, MxCfg<256>::kSmemBytes)
                        : go(gemm_mx_kernel<false, 256>, MxCfg<256>::kSmemBytes);
  return p.splits > 1 ? go(gemm_mx_kernel<true, 192>, MxCfg<192>::kSmemBytes)
                      : go(gemm_mx_kernel<false, 192>, MxCfg<192>::kSmemBytes);
}

}  // namespace fp8bs
