// Host-side internals shared by the C ABI (api.cu), the dispatch table
// (dispatch.cpp) and the kernel launchers (*.cu).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda.h>
#include <cuda_runtime.h>

#include <utility>

#include "fp8bs.h"

namespace fp8bs {

enum Path : int {
  kPathGemv = 0,  // weight-streaming split-K kernel (mma.sync, small M)
  kPathTc = 1,    // tcgen05/TMEM tensor-core kernel fed by TMA
  kPathGemvTma = 2,  // weight-streaming split-K kernel fed by TMA (mma.sync, small M)
  kPathGemvUmma = 3,  // weight-streaming split-K kernel fed by TMA, tcgen05 products (small M)
  kPathTcWide = 4,    // tcgen05/TMEM a8w8 kernel with the sixteen-warp promotion epilogue
  kPathTcPair = 5,    // the same on CTA pairs (cta_group::2, 256 x 256 tiles)
};

// One kernel configuration a dispatch-table row can name.
struct KernelConfig {
  const char* name;
  int op;           // FP8BS_OP_*
  int path;         // Path
  int bn;           // tensor-core path: N tile (columns of W per CTA)
  int split_k;      // tensor-core path: K splits (0 = automatic from the tile count, 1 = none)
  int gemv_depth;   // weight-streaming path: units in flight per warp; CTA-pair path: MMAs per K step
};

// Registry of every configuration (static storage).
const KernelConfig* find_config(int op, const char* name);
const KernelConfig* const* list_configs(int op, int* count);
// Heuristic configuration for a shape with no table row.
const KernelConfig* default_config(int op, int64_t M, int64_t N, int64_t K);
// Table lookup with the padded-M walk; record != 0 counts it in the census.
const KernelConfig* dispatch(int op, int64_t M, int64_t N, int64_t K, bool record, int64_t* padded_M, bool* hit);

// Workspace layout shared by the split-K kernels: a fixed region of arrival counters
// (one per output block, at most kMaxCounters) followed by the partial sums. The counter
// region does not depend on the shape, so one call's counters never land on another
// call's partial sums; every call leaves its counters at zero.
constexpr int64_t kMaxCounters = 65536;
constexpr size_t kCounterBytes = size_t(kMaxCounters) * 4;

// Largest M the weight-streaming path handles (8 tokens per mma.sync N block, 4 blocks).
constexpr int64_t kGemvMaxM = 32;

// Read and clear the device-side status words of the translation units whose kernels
// wait (~0u on a CUDA error).
unsigned int take_status_tc();
unsigned int take_status_gemv_tma();
unsigned int take_status_gemv_umma();
unsigned int take_status_fp8();
unsigned int take_status_mx();

// Device properties, cached per device.
int device_sm_count();
// cudaFuncAttributeMaxDynamicSharedMemorySize for a kernel, set once per (kernel, device)
// in the context of the current device. Returns a cudaError_t value as int.
int set_max_dynamic_smem(const void* kernel, int bytes);

// ---- launchers (return a cudaError_t value as int; 0 = success) ----
int launch_quant_act(const void* x, int64_t M, int64_t K, int64_t ld_x, void* q, float* scale, void* stream);
int launch_quant_weight(const float* w, int64_t N, int64_t K, void* q, float* scale, void* stream);
int launch_quant_act_mx32(const void* x, int64_t M, int64_t K, int64_t ld_x, void* q, void* ecode, void* stream);
int launch_quant_weight_mx32(const float* w, int64_t N, int64_t K, void* q, void* ecode, void* stream);
int launch_add_rmsnorm_quant(const void* x, const void* residual, const void* gamma, float eps, void* residual_out,
                             void* q, float* scale, int64_t M, int64_t K, void* stream);

size_t gemv_workspace_bytes(int op, int64_t M, int64_t N, int64_t K, const KernelConfig& cfg);
int launch_gemv_a8w8(const KernelConfig& cfg, const void* A, const float* a_scale, const void* W,
                     const float* w_scale, void* out, int64_t M, int64_t N, int64_t K, void* ws, void* stream);
int launch_gemv_bf16(const KernelConfig& cfg, const void* A, const void* W, void* out, int out_fp32, int64_t M,
                     int64_t N, int64_t K, void* ws, void* stream);

size_t gemv_tma_workspace_bytes(int64_t M, int64_t N, int64_t K);
int launch_gemv_tma_a8w8(const void* A, const float* a_scale, const void* W, const float* w_scale, void* out,
                         int64_t M, int64_t N, int64_t K, void* ws, int static_w, void* stream);

size_t gemv_umma_workspace_bytes(int64_t M, int64_t N, int64_t K);
int launch_gemv_umma_a8w8(const void* A, const float* a_scale, const void* W, const float* w_scale, void* out,
                          int64_t M, int64_t N, int64_t K, void* ws, int static_w, void* stream, bool tiled_w = false);
// The decode kernel can read this shape's weights in the tiled layout (its scales fit the
// staging region; otherwise the shape goes to the mma.sync kernel, which cannot).
bool gemv_umma_reads_tiles(int64_t M, int64_t N, int64_t K);
// Tiled weight layout: bytes of the tiles of an [N, K] e4m3 weight, and the tiling launch.
size_t tiled_weight_bytes(int64_t N, int64_t K);
int launch_tile_weight(const void* w, int64_t N, int64_t K, void* wt, void* stream);
size_t gemv_umma_bf16_workspace_bytes(int64_t M, int64_t N, int64_t K);
int launch_gemv_umma_bf16(const void* A, const void* W, void* out, int out_fp32, int64_t M, int64_t N, int64_t K,
                          void* ws, void* stream);

// Launch a kernel on a stream with programmatic stream serialisation (PDL) unless the
// environment sets FP8BS_PDL=0. Returns the cudaError_t of the launch as int.
bool pdl_enabled();

// Allocation-free variant of the weight-streaming kernel: its scratch is a fixed array in
// the library image. *too_big = 1 when the shape needs more scratch than the array holds.
int launch_gemv_tma_noalloc(const void* A, const float* a_scale, const void* W, const float* w_scale, void* out,
                            int64_t M, int64_t N, int64_t K, void* stream, int* too_big);

// 2-D K-major TMA map, 128-byte swizzle, box = 128 bytes x box_rows.
bool make_tma_2d_kmajor(CUtensorMap* m, const void* ptr, bool one_byte, int64_t rows, int64_t cols, int box_rows);
// 2-D bf16 [rows, cols] map for TMA stores: box 32 x 32, 64-byte swizzle.
bool make_tma_2d_bf16_store(CUtensorMap* m, void* ptr, int64_t rows, int64_t cols);

size_t fp8_tc_workspace_bytes(int64_t M, int64_t N, int64_t K, const KernelConfig& cfg);
int launch_fp8_tc(const KernelConfig& cfg, const void* A, const float* a_scale, const void* W, const float* w_scale,
                  void* out, int64_t M, int64_t N, int64_t K, void* ws, void* stream,
                  bool tiled_w = false);
// MX32 GEMM (E8M0 scales on 32-wide K groups, hardware block scaling), batch >= 1.
size_t mx_workspace_bytes(int64_t batch, int64_t M, int64_t N, int64_t K);
int launch_gemm_mx32(const void* A, const uint8_t* a_e, const void* W, const uint8_t* w_e, void* out, int64_t batch,
                     int64_t M, int64_t N, int64_t K, void* ws, void* stream, unsigned wait_ns);

// CTA-pair kernel (no split K, no workspace) and the clusters of two that fit at once.
int launch_fp8_pair(int halves, const void* A, const float* a_scale, const void* W, const float* w_scale, void* out,
                    int64_t M, int64_t N, int64_t K, void* stream);
int fp8_pair_clusters();
// Testing: bound of every wait (0 = the default 1 s) and an iteration whose loads CTA 0's
// producer skips (-1 = none) for the next launches of the wide-epilogue kernel.
void fp8_tc_set_test_fault(unsigned long long wait_ns, int skip_it);

size_t tc_workspace_bytes(int op, int64_t M, int64_t N, int64_t K, const KernelConfig& cfg);
int launch_tc_a8w8(const KernelConfig& cfg, const void* A, const float* a_scale, const void* W,
                   const float* w_scale, void* out, int64_t M, int64_t N, int64_t K, void* ws, void* stream);
int launch_tc_bf16(const KernelConfig& cfg, const void* A, const void* W, void* out, int out_fp32, int64_t M,
                   int64_t N, int64_t K, void* ws, void* stream);

#ifdef __CUDACC__
template <typename... KArgs, typename... Args>
int launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, void* stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return int(cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...));
}
#endif

}  // namespace fp8bs
