// The C ABI declared in include/fp8bs.h: argument validation, dispatch, launch.
// Nothing here allocates device memory or synchronises (except
// fp8bs_get_device_status, which is documented to).
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdlib>
#include <mutex>
#include <set>
#include <utility>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

#define FP8BS_API extern "C" __attribute__((visibility("default")))

namespace fp8bs {

int device_sm_count() {
  static int counts[64];
  static std::once_flag once[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::call_once(once[dev], [dev] {
    int c = 0;
    if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0) c = 148;
    counts[dev] = c;
  });
  return counts[dev];
}

int set_max_dynamic_smem(const void* kernel, int bytes) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  int dev = 0;
  if (const cudaError_t e = cudaGetDevice(&dev)) return int(e);
  std::lock_guard<std::mutex> lk(mu);
  if (done.count({kernel, dev})) return 0;
  if (const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes))
    return int(e);
  done.insert({kernel, dev});
  return 0;
}

bool pdl_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("FP8BS_PDL");
    return !(e && e[0] == '0');
  }();
  return on;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// sm_100 family only; checked once per device.
static fp8bs_status check_device() {
  static int ok[64];
  static std::once_flag once[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FP8BS_ERR_CUDA;
  if (dev < 0 || dev >= 64) return FP8BS_ERR_UNSUPPORTED;
  std::call_once(once[dev], [dev] {
    int major = 0;
    ok[dev] = (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess && major == 10)
                  ? 1
                  : 0;
  });
  return ok[dev] ? FP8BS_OK : FP8BS_ERR_UNSUPPORTED;
}

static fp8bs_status from_cuda(int e) { return e == 0 ? FP8BS_OK : FP8BS_ERR_CUDA; }

static size_t op_workspace(int op, int64_t M, int64_t N, int64_t K, const KernelConfig& cfg) {
  switch (cfg.path) {
    case kPathGemv: return gemv_workspace_bytes(op, M, N, K, cfg);
    case kPathGemvTma: return gemv_tma_workspace_bytes(M, N, K);
    case kPathGemvUmma:
      return op == FP8BS_OP_BF16 ? gemv_umma_bf16_workspace_bytes(M, N, K) : gemv_umma_workspace_bytes(M, N, K);
    case kPathTcWide: return fp8_tc_workspace_bytes(M, N, K, cfg);
    case kPathTcPair: return 0;
    default: return tc_workspace_bytes(op, M, N, K, cfg);
  }
}

}  // namespace fp8bs

using namespace fp8bs;

FP8BS_API const char* fp8bs_status_string(fp8bs_status s) {
  switch (s) {
    case FP8BS_OK: return "ok";
    case FP8BS_ERR_INVALID_ARG: return "invalid argument";
    case FP8BS_ERR_UNSUPPORTED: return "unsupported shape or device";
    case FP8BS_ERR_ALIGNMENT: return "pointer or leading dimension not 16-byte aligned";
    case FP8BS_ERR_WORKSPACE: return "workspace missing or too small";
    case FP8BS_ERR_CUDA: return "CUDA runtime error";
    case FP8BS_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

FP8BS_API const char* fp8bs_version(void) { return "fp8bs 0.1.0 (sm_100a)"; }

FP8BS_API fp8bs_status fp8bs_quant_act_per_token_group(const void* x_bf16, int64_t M, int64_t K, int64_t ld_x,
                                                       void* q_e4m3, float* a_scale, int group,
                                                       fp8bs_stream_t stream) {
  if (!x_bf16 || !q_e4m3 || !a_scale || M <= 0 || K <= 0 || group != 128 || K % 128 != 0 || ld_x < K)
    return FP8BS_ERR_INVALID_ARG;
  if (M > (int64_t(1) << 31) / (K / 128)) return FP8BS_ERR_UNSUPPORTED;
  if (!aligned16(x_bf16) || !aligned16(q_e4m3) || !aligned16(a_scale) || ld_x % 8 != 0) return FP8BS_ERR_ALIGNMENT;
  fp8bs_status st = check_device();
  if (st != FP8BS_OK) return st;
  return from_cuda(launch_quant_act(x_bf16, M, K, ld_x, q_e4m3, a_scale, stream));
}

FP8BS_API fp8bs_status fp8bs_add_rmsnorm_quant(const void* x_bf16, const void* residual_bf16,
                                                const void* gamma_bf16, float eps, int64_t M, int64_t K,
                                                void* residual_out_bf16, void* q_e4m3, float* a_scale,
                                                fp8bs_stream_t stream) {
  if (!x_bf16 || !residual_bf16 || !gamma_bf16 || !residual_out_bf16 || !q_e4m3 || !a_scale || M <= 0 || K <= 0 ||
      K % 128 != 0 || !(eps >= 0.f))
    return FP8BS_ERR_INVALID_ARG;
  if (M >= (int64_t(1) << 31) / (K / 128) || K > 32768) return FP8BS_ERR_UNSUPPORTED;
  if (!aligned16(x_bf16) || !aligned16(residual_bf16) || !aligned16(gamma_bf16) || !aligned16(residual_out_bf16) ||
      !aligned16(q_e4m3) || !aligned16(a_scale))
    return FP8BS_ERR_ALIGNMENT;
  fp8bs_status st = check_device();
  if (st != FP8BS_OK) return st;
  return from_cuda(
      launch_add_rmsnorm_quant(x_bf16, residual_bf16, gamma_bf16, eps, residual_out_bf16, q_e4m3, a_scale, M, K, stream));
}

FP8BS_API fp8bs_status fp8bs_quant_act_mx32(const void* x_bf16, int64_t M, int64_t K, int64_t ld_x, void* q_e4m3,
                                             uint8_t* a_e8m0, fp8bs_stream_t stream) {
  if (!x_bf16 || !q_e4m3 || !a_e8m0 || M <= 0 || K <= 0 || K % 32 != 0 || ld_x < K) return FP8BS_ERR_INVALID_ARG;
  if (M > (int64_t(1) << 31) / (K / 32)) return FP8BS_ERR_UNSUPPORTED;
  if (!aligned16(x_bf16) || !aligned16(q_e4m3) || ld_x % 8 != 0) return FP8BS_ERR_ALIGNMENT;
  fp8bs_status st = check_device();
  if (st != FP8BS_OK) return st;
  return from_cuda(launch_quant_act_mx32(x_bf16, M, K, ld_x, q_e4m3, a_e8m0, stream));
}

FP8BS_API fp8bs_status fp8bs_quant_weight_mx32(const float* w_f32, int64_t N, int64_t K, void* q_e4m3,
                                               uint8_t* w_e8m0, fp8bs_stream_t stream) {
  if (!w_f32 || !q_e4m3 || !w_e8m0 || N <= 0 || K <= 0 || K % 32 != 0) return FP8BS_ERR_INVALID_ARG;
  if (((N + 31) / 32) * (K / 32) > (int64_t(1) << 31) / 32) return FP8BS_ERR_UNSUPPORTED;
  if (!aligned16(w_f32) || !aligned16(q_e4m3)) return FP8BS_ERR_ALIGNMENT;
  fp8bs_status st = check_device();
  if (st != FP8BS_OK) return st;
  return from_cuda(launch_quant_weight_mx32(w_f32, N, K, q_e4m3, w_e8m0, stream));
}

FP8BS_API size_t fp8bs_mx32_workspace_bytes(int64_t batch, int64_t M, int64_t N, int64_t K) {
  if (batch <= 0 || M <= 0 || N <= 0 || K <= 0 || K % 128 != 0) return 0;
  return mx_workspace_bytes(batch, M, N, K);
}

FP8BS_API fp8bs_status fp8bs_quant_weight_block128(const float* w_f32, int64_t N, int64_t K, void* q_e4m3,
                                                   float* w_scale, fp8bs_stream_t stream) {
  if (!w_f32 || !q_e4m3 || !w_scale || N <= 0 || K <= 0 || K % 128 != 0) return FP8BS_ERR_INVALID_ARG;
  if ((N + 127) / 128 > 65535 || K / 128 > (int64_t(1) << 31)) return FP8BS_ERR_UNSUPPORTED;
  if (!aligned16(w_f32) || !aligned16(q_e4m3) || !aligned16(w_scale)) return FP8BS_ERR_ALIGNMENT;
  fp8bs_status st = check_device();
  if (st != FP8BS_OK) return st;
  return from_cuda(launch_quant_weight(w_f32, N, K, q_e4m3, w_scale, stream));
}

FP8BS_API size_t fp8bs_workspace_bytes(int op, int64_t M, int64_t N, int64_t K) {
  if (op < 0 || op >= FP8BS_NUM_OPS || M <= 0 || N <= 0 || K <= 0) return 0;
  int64_t pm = 0;
  bool hit = false;
  const KernelConfig* cfg = dispatch(op, M, N, K, false, &pm, &hit);
  if (!cfg) return 0;
  // also enough for the shape's default configuration, which a tiled-weight call runs when
  // the row names a kernel that does not read weight tiles
  return std::max(op_workspace(op, M, N, K, *cfg), op_workspace(op, M, N, K, *default_config(op, M, N, K)));
}

static fp8bs_status check_gemm_shape(int64_t M, int64_t N, int64_t K, int64_t kdiv) {
  if (M <= 0 || N <= 0 || K <= 0 || K % kdiv != 0 || N % 16 != 0) return FP8BS_ERR_INVALID_ARG;
  if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31)) return FP8BS_ERR_UNSUPPORTED;
  return FP8BS_OK;
}

FP8BS_API fp8bs_status fp8bs_gemm_a8w8_blockscale_ex(const void* A_e4m3, const float* a_scale, const void* W_e4m3,
                                                     const float* w_scale, void* out_bf16, int64_t M, int64_t N,
                                                     int64_t K, void* workspace, size_t workspace_bytes, uint32_t flags,
                                                     fp8bs_stream_t stream) {
  if (flags & ~uint32_t(FP8BS_FLAG_STATIC_WEIGHTS | FP8BS_FLAG_TILED_WEIGHTS)) return FP8BS_ERR_INVALID_ARG;
  if (!A_e4m3 || !a_scale || !W_e4m3 || !w_scale || !out_bf16) return FP8BS_ERR_INVALID_ARG;
  fp8bs_status st = check_gemm_shape(M, N, K, 128);
  if (st != FP8BS_OK) return st;
  if (!aligned16(A_e4m3) || !aligned16(W_e4m3) || !aligned16(out_bf16) || !aligned16(a_scale) || !aligned16(w_scale))
    return FP8BS_ERR_ALIGNMENT;
  st = check_device();
  if (st != FP8BS_OK) return st;
  int64_t pm = 0;
  bool hit = false;
  const KernelConfig* cfg = dispatch(FP8BS_OP_A8W8_BLOCKSCALE, M, N, K, true, &pm, &hit);
  if (!cfg) return FP8BS_ERR_UNSUPPORTED;
  const bool tiled = (flags & FP8BS_FLAG_TILED_WEIGHTS) != 0;
  if (tiled) {
    // only the tcgen05 weight-streaming and wide-epilogue kernels read weight tiles: a row
    // naming another configuration runs the shape's default instead
    if (cfg->path != kPathGemvUmma && cfg->path != kPathTcWide) cfg = default_config(FP8BS_OP_A8W8_BLOCKSCALE, M, N, K);
    if (cfg->path == kPathGemvUmma && !gemv_umma_reads_tiles(M, N, K)) return FP8BS_ERR_UNSUPPORTED;
  }
  const size_t need = op_workspace(FP8BS_OP_A8W8_BLOCKSCALE, M, N, K, *cfg);
  if (need && (!workspace || workspace_bytes < need)) return FP8BS_ERR_WORKSPACE;
  if (need && !aligned16(workspace)) return FP8BS_ERR_ALIGNMENT;
  int e;
  if (cfg->path == kPathGemv)
    e = launch_gemv_a8w8(*cfg, A_e4m3, a_scale, W_e4m3, w_scale, out_bf16, M, N, K, workspace, stream);
  else if (cfg->path == kPathGemvTma)
    e = launch_gemv_tma_a8w8(A_e4m3, a_scale, W_e4m3, w_scale, out_bf16, M, N, K, workspace,
                             (flags & FP8BS_FLAG_STATIC_WEIGHTS) ? 1 : 0, stream);
  else if (cfg->path == kPathGemvUmma)
    e = launch_gemv_umma_a8w8(A_e4m3, a_scale, W_e4m3, w_scale, out_bf16, M, N, K, workspace,
                              (flags & FP8BS_FLAG_STATIC_WEIGHTS) ? 1 : 0, stream, tiled);
  else if (cfg->path == kPathTcWide)
    e = launch_fp8_tc(*cfg, A_e4m3, a_scale, W_e4m3, w_scale, out_bf16, M, N, K, workspace, stream, tiled);
  else if (cfg->path == kPathTcPair)
    e = launch_fp8_pair(cfg->gemv_depth, A_e4m3, a_scale, W_e4m3, w_scale, out_bf16, M, N, K, stream);
  else
    e = launch_tc_a8w8(*cfg, A_e4m3, a_scale, W_e4m3, w_scale, out_bf16, M, N, K, workspace, stream);
  return from_cuda(e);
}

FP8BS_API size_t fp8bs_tiled_weight_bytes(int64_t N, int64_t K) {
  if (N <= 0 || K <= 0 || K % 128 != 0) return 0;
  return tiled_weight_bytes(N, K);
}

FP8BS_API fp8bs_status fp8bs_tile_weight_e4m3(const void* W_e4m3, int64_t N, int64_t K, void* W_tiled,
                                              fp8bs_stream_t stream) {
  if (!W_e4m3 || !W_tiled || N <= 0 || K <= 0 || K % 128 != 0) return FP8BS_ERR_INVALID_ARG;
  if (!aligned16(W_e4m3) || !aligned16(W_tiled)) return FP8BS_ERR_ALIGNMENT;
  fp8bs_status st = check_device();
  if (st != FP8BS_OK) return st;
  return from_cuda(launch_tile_weight(W_e4m3, N, K, W_tiled, stream));
}

FP8BS_API fp8bs_status fp8bs_gemm_a8w8_blockscale(const void* A_e4m3, const float* a_scale, const void* W_e4m3,
                                                  const float* w_scale, void* out_bf16, int64_t M, int64_t N,
                                                  int64_t K, void* workspace, size_t workspace_bytes,
                                                  fp8bs_stream_t stream) {
  return fp8bs_gemm_a8w8_blockscale_ex(A_e4m3, a_scale, W_e4m3, w_scale, out_bf16, M, N, K, workspace,
                                       workspace_bytes, 0u, stream);
}

FP8BS_API fp8bs_status fp8bs_gemm_a8w8_blockscale_noalloc(const void* A_e4m3, const float* a_scale,
                                                          const void* W_e4m3, const float* w_scale, void* out_bf16,
                                                          int64_t M, int64_t N, int64_t K, fp8bs_stream_t stream) {
  if (!A_e4m3 || !a_scale || !W_e4m3 || !w_scale || !out_bf16) return FP8BS_ERR_INVALID_ARG;
  fp8bs_status st = check_gemm_shape(M, N, K, 128);
  if (st != FP8BS_OK) return st;
  if (!aligned16(A_e4m3) || !aligned16(W_e4m3) || !aligned16(out_bf16) || !aligned16(a_scale) || !aligned16(w_scale))
    return FP8BS_ERR_ALIGNMENT;
  st = check_device();
  if (st != FP8BS_OK) return st;
  int too_big = 0;
  const int e = launch_gemv_tma_noalloc(A_e4m3, a_scale, W_e4m3, w_scale, out_bf16, M, N, K, stream, &too_big);
  if (too_big) return FP8BS_ERR_UNSUPPORTED;
  return from_cuda(e);
}

FP8BS_API fp8bs_status fp8bs_gemm_bf16(const void* A_bf16, const void* W_bf16, void* out, int out_is_fp32, int64_t M,
                                       int64_t N, int64_t K, void* workspace, size_t workspace_bytes,
                                       fp8bs_stream_t stream) {
  if (!A_bf16 || !W_bf16 || !out) return FP8BS_ERR_INVALID_ARG;
  fp8bs_status st = check_gemm_shape(M, N, K, 64);
  if (st != FP8BS_OK) return st;
  if (!aligned16(A_bf16) || !aligned16(W_bf16) || !aligned16(out)) return FP8BS_ERR_ALIGNMENT;
  st = check_device();
  if (st != FP8BS_OK) return st;
  int64_t pm = 0;
  bool hit = false;
  const KernelConfig* cfg = dispatch(FP8BS_OP_BF16, M, N, K, true, &pm, &hit);
  if (!cfg) return FP8BS_ERR_UNSUPPORTED;
  const size_t need = op_workspace(FP8BS_OP_BF16, M, N, K, *cfg);
  if (need && (!workspace || workspace_bytes < need)) return FP8BS_ERR_WORKSPACE;
  if (need && !aligned16(workspace)) return FP8BS_ERR_ALIGNMENT;
  int e;
  if (cfg->path == kPathGemv)
    e = launch_gemv_bf16(*cfg, A_bf16, W_bf16, out, out_is_fp32, M, N, K, workspace, stream);
  else if (cfg->path == kPathGemvUmma)
    e = launch_gemv_umma_bf16(A_bf16, W_bf16, out, out_is_fp32, M, N, K, workspace, stream);
  else
    e = launch_tc_bf16(*cfg, A_bf16, W_bf16, out, out_is_fp32, M, N, K, workspace, stream);
  return from_cuda(e);
}

FP8BS_API fp8bs_status fp8bs_gemm_a8w8_mx32(const void* A_e4m3, const uint8_t* a_e8m0, const void* W_e4m3,
                                            const uint8_t* w_e8m0, void* out_bf16, int64_t batch, int64_t M,
                                            int64_t N, int64_t K, void* workspace, size_t workspace_bytes,
                                            fp8bs_stream_t stream) {
  if (!A_e4m3 || !a_e8m0 || !W_e4m3 || !w_e8m0 || !out_bf16 || batch <= 0) return FP8BS_ERR_INVALID_ARG;
  fp8bs_status st = check_gemm_shape(M, N, K, 128);
  if (st != FP8BS_OK) return st;
  if (batch > 65535 || batch * M >= (int64_t(1) << 31) / (K / 32) || batch * ((N + 31) / 32) * (K / 32) >= (int64_t(1) << 31))
    return FP8BS_ERR_UNSUPPORTED;
  if (!aligned16(A_e4m3) || !aligned16(W_e4m3) || !aligned16(out_bf16) || !aligned16(a_e8m0) || !aligned16(w_e8m0))
    return FP8BS_ERR_ALIGNMENT;
  st = check_device();
  if (st != FP8BS_OK) return st;
  const size_t need = mx_workspace_bytes(batch, M, N, K);
  if (need && (!workspace || workspace_bytes < need)) return FP8BS_ERR_WORKSPACE;
  if (need && !aligned16(workspace)) return FP8BS_ERR_ALIGNMENT;
  return from_cuda(launch_gemm_mx32(A_e4m3, a_e8m0, W_e4m3, w_e8m0, out_bf16, batch, M, N, K, workspace, stream,
                                    unsigned(kWaitLimitNs)));
}

FP8BS_API fp8bs_status fp8bs_get_device_status(fp8bs_stream_t stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FP8BS_ERR_CUDA;
  const unsigned int a = take_status_tc(), b = take_status_gemv_tma(), c = take_status_gemv_umma(),
                     d = take_status_fp8(), e = take_status_mx();
  if (a == ~0u || b == ~0u || c == ~0u || d == ~0u || e == ~0u) return FP8BS_ERR_CUDA;
  const unsigned int v = a | b | c | d | e;
  return (v & kStatusTimeout) ? FP8BS_ERR_TIMEOUT : FP8BS_OK;
}

FP8BS_API fp8bs_status fp8bs_test_set_wait_fault(uint64_t wait_limit_ns, int64_t skip_iteration) {
  if (skip_iteration < -1 || skip_iteration > INT32_MAX) return FP8BS_ERR_INVALID_ARG;
  fp8_tc_set_test_fault(wait_limit_ns, int(skip_iteration));
  return FP8BS_OK;
}
