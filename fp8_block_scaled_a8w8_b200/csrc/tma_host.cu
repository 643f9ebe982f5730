// Host-side TMA tensor-map creation shared by the kernels that stage operands with TMA.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "internal.h"

namespace fp8bs {

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// 2-D K-major map over a row-major [rows, cols] matrix (1-byte e4m3 or 2-byte bf16):
// box = 128 bytes of K x box_rows rows, 128-byte swizzle, out-of-range rows read as zero.
bool make_tma_2d_kmajor(CUtensorMap* m, const void* ptr, bool one_byte, int64_t rows, int64_t cols, int box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const int esz = one_byte ? 1 : 2;
  cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(cols * esz)};
  cuuint32_t box[2] = {cuuint32_t(128 / esz), cuuint32_t(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  std::memset(m, 0, sizeof(*m));
  CUresult r = enc(m, one_byte ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D map over a row-major bf16 [rows, cols] output for TMA stores: box = 32 columns (64
// bytes) x 32 rows, 64-byte swizzle (the layout the epilogue stages in shared memory);
// elements outside [rows, cols] are not written.
bool make_tma_2d_bf16_store(CUtensorMap* m, void* ptr, int64_t rows, int64_t cols) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(cols * 2)};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  std::memset(m, 0, sizeof(*m));
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace fp8bs
