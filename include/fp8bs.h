/*
 * fp8bs -- a8w8 block-scaled FP8 GEMM for NVIDIA B200 (sm_100a): C ABI.
 *
 * Operation (the GEMM behind gemm_a8w8_blockscale in the pages
 * [cookbook#8] "Why aiter#5069's measured -25% kernel win moved serving
 * throughput by 0.0%" -- GLM-5.2-FP8 is block quantised with
 * weight_block_size [128,128] and so takes gemm_a8w8_blockscale -- and
 * [aiter#7752] "[Perf] Retune gfx942 Qwen3.8-27B a8w8 blockscale decode rows
 * for cold weights", section "Kernel"):
 *
 *   out[m,n] = sum_g a_scale[m,g] * w_scale[n/128,g]
 *                    * sum_{k = 128g .. 128g+127} A[m,k] * W[n,k]
 *
 * A and W hold OCP e4m3 ("e4m3fn") codes, one byte per element; A is
 * quantised per token per 1x128 group of K, W per 128x128 block; scales are
 * float32 (scale = amax / 448); accumulation is float32; out is bfloat16,
 * rounded once (round to nearest even).
 *
 * Conventions shared by every entry point:
 *  - All matrices are row-major with the reduction dimension K contiguous
 *    ("NT"): A [M,K], W [N,K], out [M,N], a_scale [M, K/128],
 *    w_scale [ceil(N/128), K/128]. Leading dimensions equal the row length
 *    unless an ld argument says otherwise.
 *  - Every pointer to matrix data is a DEVICE pointer, owned by the caller.
 *    The library calls no allocator: it never allocates, frees or retains
 *    device memory (its only device storage is a few status words and the
 *    fixed scratch array of fp8bs_gemm_a8w8_blockscale_noalloc, both part of
 *    the library image). Device pointers must be 16-byte aligned
 *    (FP8BS_ERR_ALIGNMENT otherwise).
 *  - Every compute call is asynchronous on the given CUDA stream (a
 *    cudaStream_t; NULL is the legacy default stream), performs no host
 *    synchronisation and no allocation, and may be captured in a CUDA graph.
 *  - Arguments are validated before anything is launched: an invalid call
 *    returns a status other than FP8BS_OK and launches nothing. A launch
 *    failure reported by the CUDA runtime returns FP8BS_ERR_CUDA.
 *  - There is no CPU fallback: without a usable sm_100 device the compute
 *    calls return FP8BS_ERR_CUDA or FP8BS_ERR_UNSUPPORTED.
 *  - No C++ exception crosses this interface. All functions are thread-safe;
 *    the dispatch table's counters are process-global atomics.
 *  - Calls run on the device that is current on the calling thread. Kernel
 *    attributes such as the dynamic shared-memory size are set once per kernel
 *    and device, at the kernel's first launch on that device.
 */
#ifndef FP8BS_H
#define FP8BS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, without pulling in the CUDA headers. */
typedef struct CUstream_st* fp8bs_stream_t;

typedef enum {
  FP8BS_OK = 0,
  FP8BS_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, K % 128 != 0, N % 16 != 0, ... */
  FP8BS_ERR_UNSUPPORTED = 2, /* shape or device the library has no kernel for */
  FP8BS_ERR_ALIGNMENT = 3,   /* a device pointer or leading dimension is not 16-byte aligned */
  FP8BS_ERR_WORKSPACE = 4,   /* workspace missing or smaller than fp8bs_workspace_bytes() */
  FP8BS_ERR_CUDA = 5,        /* the CUDA runtime reported an error at launch */
  FP8BS_ERR_TIMEOUT = 6      /* a kernel gave up a bounded device-side wait (see fp8bs_get_device_status) */
} fp8bs_status;

/* Operation ids for the dispatch table and workspace sizing. */
enum { FP8BS_OP_A8W8_BLOCKSCALE = 0, FP8BS_OP_BF16 = 1, FP8BS_NUM_OPS = 2 };

/*
 * Activation quantisation, per token per 1x128 group.
 * For every row m and group g (K/128 groups):
 *   amax = max |x[m, 128g .. 128g+127]|,  a_scale[m,g] = amax / 448 (IEEE fp32 division),
 *   q[m,k] = e4m3_rn_satfinite(x[m,k] / a_scale[m,g])  (IEEE fp32 division, one rounding);
 * a group with amax == 0 gets a_scale 0 and codes +-0 (0x00 / 0x80, the sign of x).
 * x_bf16 : device, bf16 [M, ld_x] (row stride ld_x elements, ld_x >= K, ld_x % 8 == 0)
 * q_e4m3 : device, e4m3 codes [M, K] (row stride K), written
 * a_scale: device, float32 [M, K/128] (row stride K/128), written
 * group  : must be 128.
 * Result bit-identical to the CPU oracle (codes and scales).
 */
fp8bs_status fp8bs_quant_act_per_token_group(const void* x_bf16, int64_t M, int64_t K, int64_t ld_x,
                                             void* q_e4m3, float* a_scale, int group,
                                             fp8bs_stream_t stream);

/*
 * Fused residual add + RMSNorm + activation quantisation: the step that produces the
 * a8w8 GEMM's input (add_rmsnorm_quant in the decode kernel table of [mi210 docs/43]
 * "43-ck-int8-gemm-gfx90a.md", Rounds 40-41). For every token row m:
 *   h[m,k]  = bf16(float(x[m,k]) + float(residual[m,k]))   written to residual_out
 *   r[m]    = 1 / sqrt(sum_k h[m,k]^2 / K + eps)             float32
 *   y[m,k]  = (h[m,k] * r[m]) * gamma[k]                     float32, never rounded to bf16
 *   q, a_scale = the per-token 1x128 quantisation of y (as fp8bs_quant_act_per_token_group)
 * x_bf16, residual_bf16: device, bf16 [M, K]; gamma_bf16: device, bf16 [K];
 * residual_out_bf16: device, bf16 [M, K], written (it may be residual_bf16 itself);
 * q_e4m3: device, e4m3 [M, K], written; a_scale: device, float32 [M, K/128], written.
 * Requires K % 128 == 0, eps >= 0 (FP8BS_ERR_INVALID_ARG otherwise) and K <= 32768
 * (FP8BS_ERR_UNSUPPORTED otherwise: one CTA holds a row in registers). residual_out is
 * bit-identical to the oracle's; the mean square is a float32 sum, so a code may differ
 * from the float64 oracle's by one step where y / a_scale is within float32 error of a
 * rounding midpoint.
 */
fp8bs_status fp8bs_add_rmsnorm_quant(const void* x_bf16, const void* residual_bf16, const void* gamma_bf16,
                                     float eps, int64_t M, int64_t K, void* residual_out_bf16, void* q_e4m3,
                                     float* a_scale, fp8bs_stream_t stream);

/*
 * Weight quantisation, per 128x128 block ([cookbook#8]: weight_block_size [128,128]).
 * For every block (nb, g): amax over rows 128nb .. min(N,128nb+128)-1 and columns
 * 128g .. 128g+127; w_scale[nb,g] = amax / 448; codes as for activations.
 * w_f32  : device, float32 [N, K]; q_e4m3: device, e4m3 [N, K]; w_scale: device, float32
 * [ceil(N/128), K/128]. A set-up step (not on the per-call path).
 */
fp8bs_status fp8bs_quant_weight_block128(const float* w_f32, int64_t N, int64_t K, void* q_e4m3,
                                         float* w_scale, fp8bs_stream_t stream);

/*
 * The a8w8 block-scaled GEMM (formula at the top of this file).
 * A_e4m3 [M,K], a_scale [M,K/128], W_e4m3 [N,K], w_scale [ceil(N/128),K/128],
 * out_bf16 [M,N]: device pointers. Requires M,N,K > 0, K % 128 == 0, N % 16 == 0.
 * workspace: device scratch of at least fp8bs_workspace_bytes(FP8BS_OP_A8W8_BLOCKSCALE, M, N, K)
 * bytes (may be NULL when that is 0). It must be zero-filled once before its first
 * use. It holds split-K arrival counters, which every call leaves at zero, and partial
 * sums, whose contents between calls are unspecified; so one workspace serves any
 * number of calls of any shapes issued in order on one stream. Calls that may run
 * concurrently need separate workspaces. After a call reported FP8BS_ERR_TIMEOUT
 * (fp8bs_get_device_status) the workspace must be zero-filled again.
 * The kernel is picked by the dispatch table (fp8bs_dispatch_lookup): for M <= 32 a
 * weight-streaming split-K kernel (tcgen05 products, TMA-fed, stream-K over 128-row x
 * 128-column units), otherwise a tiled tcgen05/TMEM kernel fed by TMA whose sixteen
 * epilogue warps apply the block scales group by group and store the output through
 * shared memory with TMA; it also splits K when its output tiles would leave most SMs
 * idle (then the call needs workspace too). A table row may instead name the CTA-pair
 * variant (tcgen05 cta_group::2, 256 x 256 tiles, configurations a8w8_tc2*).
 * Results are deterministic (split-K partial sums are reduced in a fixed order) and
 * within the float32-accumulation bound of the float64 oracle rounded once to bf16.
 */
fp8bs_status fp8bs_gemm_a8w8_blockscale(const void* A_e4m3, const float* a_scale, const void* W_e4m3,
                                        const float* w_scale, void* out_bf16, int64_t M, int64_t N,
                                        int64_t K, void* workspace, size_t workspace_bytes,
                                        fp8bs_stream_t stream);

/* Flags for fp8bs_gemm_a8w8_blockscale_ex. */
enum {
  /* W_e4m3 and w_scale are not written by any kernel that can still be running when this
   * call's kernel starts (true of inference weights loaded once). The weight-streaming
   * kernel then starts fetching W before the preceding kernel in the stream has finished
   * (programmatic dependent launch), overlapping its weight stream with that kernel's
   * tail; activations, scales and the workspace are still read only after it finished. */
  FP8BS_FLAG_STATIC_WEIGHTS = 1u,
  /* W_e4m3 points to the tiled layout written by fp8bs_tile_weight_e4m3 (not [N, K]).
   * The call then runs the tcgen05 weight-streaming kernel (M <= 32) or the wide-epilogue
   * tensor-core kernel (M > 32), whatever a table row names; a decode shape whose scales
   * do not fit that kernel's staging area returns FP8BS_ERR_UNSUPPORTED. */
  FP8BS_FLAG_TILED_WEIGHTS = 2u
};

/* fp8bs_gemm_a8w8_blockscale with flags (a bitwise OR of FP8BS_FLAG_*; unknown bits give
 * FP8BS_ERR_INVALID_ARG). fp8bs_gemm_a8w8_blockscale is this call with flags = 0. */
fp8bs_status fp8bs_gemm_a8w8_blockscale_ex(const void* A_e4m3, const float* a_scale, const void* W_e4m3,
                                           const float* w_scale, void* out_bf16, int64_t M, int64_t N,
                                           int64_t K, void* workspace, size_t workspace_bytes, uint32_t flags,
                                           fp8bs_stream_t stream);

/*
 * Tiled weight layout (the role of the pages' pre-shuffled B, "bpreshuffle" [aiter#7247],
 * for this hardware): W_e4m3 [N, K] rearranged into 16 KiB tiles, one per 128-row block b
 * and 128-wide K group g, tile (b, g) at byte offset (b * K/128 + g) * 16384; within a tile,
 * row r's 128 bytes in the order of the tensor core's 128-byte-swizzled K-major operand
 * (16-byte chunk c stored at position c ^ (r % 8)). The block count is rounded up to an even
 * number; rows past N are zero. Each tile is one contiguous copy into shared memory, which
 * streams from HBM faster than the 128-byte row pieces of the [N, K] layout.
 * fp8bs_tiled_weight_bytes: size of the tiled copy (0 for invalid sizes). Host only.
 * fp8bs_tile_weight_e4m3: writes it (device pointers, both 16-byte aligned; K % 128 == 0);
 * w_scale is unchanged. Pass the result with FP8BS_FLAG_TILED_WEIGHTS.
 */
size_t fp8bs_tiled_weight_bytes(int64_t N, int64_t K);
fp8bs_status fp8bs_tile_weight_e4m3(const void* W_e4m3, int64_t N, int64_t K, void* W_tiled, fp8bs_stream_t stream);

/*
 * The a8w8 block-scaled GEMM for decode-sized M without any caller-provided memory.
 * (No counterpart in the pages: an addition for callers that cannot allocate.)
 * Some callers cannot allocate device memory where they issue a GEMM -- their memory pool
 * is fixed or owned by a host framework, or an allocation there would synchronise -- so
 * they cannot supply the workspace fp8bs_gemm_a8w8_blockscale needs. This entry point
 * runs a weight-streaming split-K kernel (the TMA-fed mma.sync variant, not the tcgen05
 * one the dispatch table picks by default) with its scratch taken from one fixed
 * 8 MiB array that is part of the library image (every GPU that loads the library holds
 * it until the process exits); it calls no allocator of any kind.
 * Arguments and result as fp8bs_gemm_a8w8_blockscale, without the workspace.
 * Limits: M <= 32 and shapes whose split-K scratch fits the array (on a 148-SM B200 every
 * N up to 65536 * 128 rows qualifies); other shapes return FP8BS_ERR_UNSUPPORTED and
 * launch nothing.
 * The first call on a device looks up the array's device address (once per device, with
 * that device current); make that first call before any CUDA stream capture.
 * Every call uses the same array and it keeps the last call's contents: each call clears
 * the arrival counters it uses (an asynchronous memset on the stream) before its kernel.
 * Calls that can overlap on the GPU (different streams, or concurrent host threads) race
 * on the array and give wrong results; issue them in order on one stream.
 */
fp8bs_status fp8bs_gemm_a8w8_blockscale_noalloc(const void* A_e4m3, const float* a_scale, const void* W_e4m3,
                                                const float* w_scale, void* out_bf16, int64_t M, int64_t N,
                                                int64_t K, fp8bs_stream_t stream);

/*
 * MX32 variant ([aiter#7247] ROCm/aiter PR #7247, "Motivation": the 32x32 MXFP8 GEMMs,
 * w_scale_block 32x32, dense and batched): e4m3 operands with E8M0 scales (one byte, value
 * 2^(code - 127)) on 32-wide K groups -- per token for activations, per 32x32 block for
 * weights -- and float32 accumulation:
 *   out[b,m,n] = sum_g 2^(a_e8m0[b,m,g] - 127) * 2^(w_e8m0[b,n/32,g] - 127)
 *                      * sum_{k = 32g .. 32g+31} A[b,m,k] * W[b,n,k]
 * Quantisation: code = clamp(ceil(log2(float32(amax) / 448)) + 127, 0, 254) (0 when amax is
 * 0; the exponent read exactly from the float32 quotient), q = e4m3_rn_satfinite(x * 2^-e).
 * The tensor core applies the scales itself (tcgen05.mma kind::mxf8f6f4.block_scale).
 *
 * fp8bs_quant_act_mx32: x_bf16 [M, ld_x] (ld_x >= K, ld_x % 8 == 0), K % 32 == 0 ->
 *   q_e4m3 [M, K], a_e8m0 [M, K/32] (device). Bit-identical to the CPU oracle.
 * fp8bs_quant_weight_mx32: w_f32 [N, K], K % 32 == 0 -> q_e4m3 [N, K],
 *   w_e8m0 [ceil(N/32), K/32] (device); a partial last block is quantised over its rows.
 * fp8bs_gemm_a8w8_mx32: batch >= 1 independent GEMMs on contiguous stacks A_e4m3
 *   [batch, M, K], a_e8m0 [batch, M, K/32], W_e4m3 [batch, N, K], w_e8m0 [batch,
 *   ceil(N/32), K/32], out_bf16 [batch, M, N] (batch = 1 is the dense GEMM). Requires
 *   K % 128 == 0, N % 16 == 0, 16-byte aligned pointers. workspace: at least
 *   fp8bs_mx32_workspace_bytes(batch, M, N, K) bytes, zero-filled once, as for
 *   fp8bs_gemm_a8w8_blockscale (split-K arrival counters are left at zero). Results are
 *   deterministic and within the float32-accumulation bound of the float64 oracle rounded
 *   once to bf16.
 */
fp8bs_status fp8bs_quant_act_mx32(const void* x_bf16, int64_t M, int64_t K, int64_t ld_x, void* q_e4m3,
                                  uint8_t* a_e8m0, fp8bs_stream_t stream);
fp8bs_status fp8bs_quant_weight_mx32(const float* w_f32, int64_t N, int64_t K, void* q_e4m3, uint8_t* w_e8m0,
                                     fp8bs_stream_t stream);
size_t fp8bs_mx32_workspace_bytes(int64_t batch, int64_t M, int64_t N, int64_t K);
fp8bs_status fp8bs_gemm_a8w8_mx32(const void* A_e4m3, const uint8_t* a_e8m0, const void* W_e4m3,
                                  const uint8_t* w_e8m0, void* out_bf16, int64_t batch, int64_t M, int64_t N,
                                  int64_t K, void* workspace, size_t workspace_bytes, fp8bs_stream_t stream);

/*
 * Companion bf16 GEMM for the small-N router / indexer projections ([cookbook#8]:
 * the live BF16 lookups are the MoE router and the DSA indexer's weights_proj;
 * [aiter#7247] "Technical Details": N = 32..1024, some with fp32 output).
 * out[m,n] = sum_k A[m,k] * W[n,k], float32 accumulation, rounded once to bf16,
 * or stored as float32 when out_is_fp32 != 0.
 * A [M,K] bf16, W [N,K] bf16, out [M,N]: device. Requires K % 64 == 0, N % 16 == 0.
 * workspace as for fp8bs_gemm_a8w8_blockscale (op FP8BS_OP_BF16).
 */
fp8bs_status fp8bs_gemm_bf16(const void* A_bf16, const void* W_bf16, void* out, int out_is_fp32,
                             int64_t M, int64_t N, int64_t K, void* workspace, size_t workspace_bytes,
                             fp8bs_stream_t stream);

/* Bytes of workspace a call of op with this shape needs (0 if none): enough for the
 * configuration the dispatch table picks and for the shape's default configuration (which
 * a call with FP8BS_FLAG_TILED_WEIGHTS may run instead). Host only. */
size_t fp8bs_workspace_bytes(int op, int64_t M, int64_t N, int64_t K);

/*
 * Dispatch table ([aiter#7752] "PR-specific question": the lookup probes exact M,
 * then the next power of two below 16 or the next multiple of 16 up to 256, then
 * the next power of two; [mi210 docs/43] section 6: a miss runs the per-shape
 * default kernel). Rows are keyed (op, padded_M, N, K). Every lookup made by a GEMM
 * call is counted; fp8bs_dispatch_lookup with record=0 only inspects.
 * padded_M: the row's M on a hit, 0 on a miss. cfg: the kernel configuration name
 * that runs (NUL-terminated, truncated to cfg_len).
 */
fp8bs_status fp8bs_dispatch_lookup(int op, int64_t M, int64_t N, int64_t K, int record,
                                   int64_t* padded_M, int* hit, char* cfg, size_t cfg_len);

/* Add or replace a table row: kernel configuration cfg (a name returned by
 * fp8bs_dispatch_list_configs) for (op, M, N, K). */
fp8bs_status fp8bs_dispatch_set_row(int op, int64_t M, int64_t N, int64_t K, const char* cfg);

/* Remove all rows (keep_builtin = 0) or restore the built-in rows (keep_builtin = 1). */
fp8bs_status fp8bs_dispatch_reset_table(int keep_builtin);

/* Newline-separated list of the kernel configuration names a row may name for op. */
fp8bs_status fp8bs_dispatch_list_configs(int op, char* buf, size_t len);

/* Lookup counters for op since the last fp8bs_dispatch_reset_stats: all lookups
 * (hits, misses) and distinct keys (M, N, K, padded_M, cfg) among them. */
fp8bs_status fp8bs_dispatch_stats(int op, uint64_t* hits, uint64_t* misses, uint64_t* distinct_hits,
                                  uint64_t* distinct_misses);
fp8bs_status fp8bs_dispatch_reset_stats(void);

/* Census: one JSON object per distinct lookup key with its count, as a JSON array. */
fp8bs_status fp8bs_dispatch_dump_json(char* buf, size_t len);

/* The current table rows, one JSON object {"op","M","N","K","cfg","tuned"} per row, as a
 * JSON array ("tuned": the row's configuration was chosen by measurement, see the
 * package's tune.py; else it is the per-shape default). FP8BS_ERR_INVALID_ARG if len is
 * too small (buf then holds ""). */
fp8bs_status fp8bs_dispatch_dump_table_json(char* buf, size_t len);

/* 64-bit FNV-1a hash of the current table rows (identifies the table that ran). */
uint64_t fp8bs_dispatch_table_hash(void);

/* Synchronises the stream, then reports and clears the device-side status word:
 * FP8BS_ERR_TIMEOUT if any kernel abandoned a bounded wait since the last call. */
fp8bs_status fp8bs_get_device_status(fp8bs_stream_t stream);

const char* fp8bs_status_string(fp8bs_status status);

/*
 * Testing hook for the failure path of the bounded device-side waits (no counterpart in
 * the pages; it exercises the timeout reporting of fp8bs_get_device_status). Applies to
 * the launches that follow of the tensor-core a8w8 kernels with the wide promotion
 * epilogue (configurations a8w8_tcw_* and a8w8_tc2_*): every wait gives up after wait_limit_ns
 * nanoseconds (0 restores the default of one second), and if skip_iteration >= 0 the
 * producer of CTA 0 leaves the K-group iteration with that index (counted over the CTA's
 * work items) unfilled, so the MMA issuer's wait on it runs out (for CTA pairs, the
 * other waits of the pair then run out too). The kernel then abandons
 * its work, drains what it issued, frees its tensor memory and exits;
 * fp8bs_get_device_status reports FP8BS_ERR_TIMEOUT; part of the output is not written
 * and the workspace must be zero-filled before its next use. fp8bs_test_set_wait_fault(0,
 * -1) restores normal operation. Process-global; not for production use.
 * Returns FP8BS_ERR_INVALID_ARG for skip_iteration < -1 or > INT32_MAX.
 */
fp8bs_status fp8bs_test_set_wait_fault(uint64_t wait_limit_ns, int64_t skip_iteration);

/* Library version string. */
const char* fp8bs_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8BS_H */
