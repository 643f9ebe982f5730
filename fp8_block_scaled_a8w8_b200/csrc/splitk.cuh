// Split-K reduction of one output tile, shared by the tensor-core GEMM kernels.
//
// A work item is (tile, split k): the split computes the float32 partial product of the
// tile over its own K range and stores it at part_tile + k * split_elems, row-major with a
// row stride of ld floats. An output element is the sum of the tile's partials in split
// order (k = 0, 1, ..., starting from 0.0f): a fixed order, so the result is bit-identical
// whichever CTA adds it and however the work is divided.
//
// Two ways to the sum, chosen per launch:
//   distributed  (every CTA holds exactly one item, so the splits of a tile are resident
//                together): each split publishes its partial with a release add on the
//                tile's counter, polls (acquire, bounded) until all splits have arrived,
//                counts itself out and sums its own 1/S share of the tile's elements. The
//                split that counts out last (the counter reaching 2S) resets the counter.
//   last arrival (persistent grids with several items per CTA): each split counts in with
//                an acq_rel add; the split that arrives last sums the whole tile and
//                resets the counter.
// Either way all of an element's split loads are issued before its first add, and the
// elements are spread over every thread of the epilogue, so the finish costs one L2 round
// trip per batch of elements rather than one per split and column chunk.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"

namespace fp8bs {

constexpr int kMaxSplits = 8;  // K splits per tile that the finish loads at once

// The valid region of one tile's partials.
struct SplitTile {
  const float* part;    // split 0 of the tile
  int split_elems;      // floats from one split's partial to the next
  int ld;               // row stride, floats
  int rows;             // valid rows (the rest of the tile lies past M)
  int qpr;              // valid 4-column quads per row (valid columns / 4; N % 4 == 0)
};

// Sums quads [u0, u1) of the tile, thread tid of nthr taking every nthr-th quad, with the
// loads of up to kS splits in flight at once (the quad's row and column are stepped rather
// than divided out in the loop).
template <int kS, class Store>
__device__ __forceinline__ void splitk_sum(const SplitTile& t, int splits, int u0, int u1, int tid, int nthr,
                                           Store& store) {
  int u = u0 + tid;
  if (u >= u1) return;
  int r = u / t.qpr, c = u - r * t.qpr;
  const int dr = nthr / t.qpr, dc = nthr - dr * t.qpr;
#pragma unroll 1
  for (; u < u1; u += nthr) {
    const float* src = t.part + r * t.ld + 4 * c;
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
    for (int k0 = 0; k0 < splits; k0 += kS) {
      float4 v[kS];
#pragma unroll
      for (int k = 0; k < kS; ++k)
        v[k] = k0 + k < splits ? __ldcg(reinterpret_cast<const float4*>(src + (k0 + k) * t.split_elems))
                               : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k = 0; k < kS; ++k)
        if (k0 + k < splits) {
          s.x += v[k].x;
          s.y += v[k].y;
          s.z += v[k].z;
          s.w += v[k].w;
        }
    }
    store(r, 4 * c, s);
    r += dr;
    c += dc;
    if (c >= t.qpr) {
      c -= t.qpr;
      ++r;
    }
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
        // count out: once the counter reaches 2S no split is still polling it
        if (v && atomicAdd(counter, 1u) == unsigned(2 * splits - 1)) *counter = 0u;
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
  const int q = t.rows * t.qpr;
  const int u0 = v == 1 ? int(int64_t(q) * sp / splits) : 0;
  const int u1 = v == 1 ? int(int64_t(q) * (sp + 1) / splits) : q;
  splitk_sum<kMaxSplits>(t, splits, u0, u1, tid, nthr, store);
}

}  // namespace fp8bs
