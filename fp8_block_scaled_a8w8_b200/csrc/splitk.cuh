// Split-K reduction of one output tile, shared by the tensor-core GEMM kernels.
//
// A work item is (tile, split k): the split computes the float32 partial product of the
// tile over its own K range and stores it at part_tile + k * split_elems. Inside a split
// the tile is stored quad-major: columns 4c .. 4c+3 of tile row r are the float4 at index
// c * BM + r (BM rows per tile), so that one warp storing one column quad of its 32
// consecutive rows writes one contiguous 512-byte span, and the finish reads consecutive
// rows with consecutive threads. An output element is the sum of the tile's partials in
// split order (k = 0, 1, ..., starting from 0.0f): a fixed order, so the result is
// bit-identical whichever CTA adds it and however the work is divided.
//
// Two ways to the sum, chosen per launch:
//   distributed  (every CTA holds exactly one item, so the splits of a tile are resident
//                together): each split publishes its partial with a release add on the
//                tile's counter, polls (acquire, bounded) until all splits have arrived,
//                counts itself out and sums its own 1/S share of the tile's elements. The
//                split that counts out last (the counter reaching 2S) resets the counter.
//   last arrival (persistent grids with several items per CTA): each split counts in with
//                an acq_rel add; the split that arrives last resets the counter and sums
//                the whole tile.
// Either way all of an element's split loads are issued before its first add, and the
// elements are spread over every thread of the epilogue, so the finish costs one L2 round
// trip per batch of elements rather than one per split and column chunk.
//
// Ordering: the epilogue threads' partial stores (st.global.cg) precede a barrier of the
// epilogue group, after which one thread's release add publishes them at gpu scope (the
// barrier orders the other threads' stores before that release); a thread whose acquire
// load observes every arrival, followed by a barrier of the group, orders all the group's
// partial loads (ld.global.cg) after the other CTAs' stores. Plain weak polling would not
// do: it is not guaranteed to observe a store made on the other die's L2 partition.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"

namespace fp8bs {

constexpr int kMaxSplits = 8;  // K splits per tile (the host policies stay within it)

// Where a split's partial keeps columns col .. col+3 of tile row r (col % 4 == 0).
__device__ __forceinline__ float* splitk_quad(float* part_item, int bm, int r, int col) {
  return part_item + (int64_t(col >> 2) * bm + r) * 4;
}

// The valid region of one tile's partials.
struct SplitTile {
  const float* part;    // split 0 of the tile
  int split_elems;      // floats from one split's partial to the next
  int bm;               // rows of the tile (the quad-major row count)
  int rows;             // valid rows (the rest of the tile lies past M)
  int qpr;              // valid 4-column quads per row (valid columns / 4; N % 4 == 0)
};

// Sums quads [u0, u1) of the tile (quad u: column quad u / rows, row u % rows), thread tid
// of nthr taking every nthr-th quad, kQ quads per pass with the loads of up to kS splits
// each in flight (kQ * kS float4 loads at once).
template <int kQ, int kS, class Store>
__device__ __forceinline__ void splitk_sum(const SplitTile& t, int splits, int u0, int u1, int tid, int nthr,
                                           Store& store) {
#pragma unroll 1
  for (int u = u0 + tid; u < u1; u += kQ * nthr) {
    int r[kQ], c[kQ];
    bool in[kQ];
    float4 s[kQ];
#pragma unroll
    for (int i = 0; i < kQ; ++i) {
      const int ui = u + i * nthr;
      in[i] = ui < u1;
      c[i] = in[i] ? ui / t.rows : 0;
      r[i] = in[i] ? ui - c[i] * t.rows : 0;
      s[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll 1
    for (int k0 = 0; k0 < splits; k0 += kS) {
      float4 v[kQ][kS];
#pragma unroll
      for (int i = 0; i < kQ; ++i)
#pragma unroll
        for (int k = 0; k < kS; ++k)
          v[i][k] = (in[i] && k0 + k < splits)
                        ? __ldcg(reinterpret_cast<const float4*>(t.part + (k0 + k) * t.split_elems) +
                                 (c[i] * t.bm + r[i]))
                        : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int i = 0; i < kQ; ++i)
#pragma unroll
        for (int k = 0; k < kS; ++k)
          if (k0 + k < splits) {
            s[i].x += v[i][k].x;
            s[i].y += v[i][k].y;
            s[i].z += v[i][k].z;
            s[i].w += v[i][k].w;
          }
    }
#pragma unroll
    for (int i = 0; i < kQ; ++i)
      if (in[i]) store(r[i], 4 * c[i], s[i]);
  }
}

// The finish of one item, called by every thread of the epilogue group (tid 0..nthr-1,
// whose barrier is bar) after the thread's own stores of the item's partial.
//   have   this CTA completed its partial (false after a timed-out wait: it publishes
//          nothing; the other splits' waits then run out and the status word reports it)
//   items  work items of the launch: the distributed way when every CTA of the grid holds
//          exactly one (items <= CTAs)
//   flag   a shared-memory word of the CTA
// store(r, c, sum) writes the 4 output columns c .. c+3 of tile row r.
template <class Bar, class Store>
__device__ __forceinline__ void splitk_finish(unsigned* counter, const SplitTile& t, int splits, int sp, bool have,
                                              int items, int tid, int nthr, volatile int* flag,
                                              unsigned long long limit_ns, unsigned int* status, Bar&& bar,
                                              Store&& store) {
  bar();  // every epilogue thread's partial stores precede the release below
  if (tid == 0) {
    int v = 0;
    if (have) {
      if (items <= int(gridDim.x)) {
        red_add_release_gpu(counter, 1u);
        v = 1;
        const unsigned long long t0 = globaltimer_ns();
        while (ld_acquire_gpu(counter) < unsigned(splits)) {
          if (globaltimer_ns() - t0 > limit_ns) {
            atomicOr(status, kStatusTimeout);
            v = 0;
            break;
          }
        }
      } else {
        // the last arrival resets the counter at once: every split has counted in
        v = atom_add_acq_rel_gpu(counter, 1u) == unsigned(splits - 1) ? 2 : 0;
        if (v) *counter = 0u;
      }
    }
    *flag = v;
  }
  bar();
  const int v = *flag;
  if (v == 0) return;
  // count out (this CTA's poll is over); the round trip overlaps the sum's loads. Once the
  // counter reaches 2S no split is still polling it, so the last one out resets it.
  unsigned out_old = 0;
  if (v == 1 && tid == 0) out_old = atomicAdd(counter, 1u);
  const int q = t.rows * t.qpr;
  const int u0 = v == 1 ? int(int64_t(q) * sp / splits) : 0;
  const int u1 = v == 1 ? int(int64_t(q) * (sp + 1) / splits) : q;
  if (splits <= 2)
    splitk_sum<8, 2>(t, splits, u0, u1, tid, nthr, store);
  else if (splits <= 4)
    splitk_sum<4, 4>(t, splits, u0, u1, tid, nthr, store);
  else
    splitk_sum<2, kMaxSplits>(t, splits, u0, u1, tid, nthr, store);
  if (v == 1 && tid == 0 && out_old == unsigned(2 * splits - 1)) *counter = 0u;
}

}  // namespace fp8bs
