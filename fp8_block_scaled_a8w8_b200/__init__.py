"""fp8bs: a8w8 block-scaled FP8 GEMM for NVIDIA B200 (sm_100a).

Python binding over the C ABI of ``libfp8bs.so`` (declared in include/fp8bs.h).
The functions here only marshal arguments -- tensor pointers, sizes and the
current CUDA stream -- into the C entry points of the same names; every step of
the computation runs in the library's CUDA kernels. PyTorch provides device
memory and streams only. There is no CPU fallback: if the library is missing
or fails to load, every call raises.
"""

from __future__ import annotations

import ctypes
import json
import os

import torch

__all__ = [
    "lib", "Fp8bsError", "quant_act_per_token_group", "quant_weight_block128", "gemm_a8w8_blockscale",
    "gemm_bf16", "workspace_bytes", "Workspace", "dispatch_lookup", "dispatch_set_row", "dispatch_reset_table",
    "dispatch_list_configs", "dispatch_stats", "dispatch_reset_stats", "dispatch_dump_json", "dispatch_dump_table", "dispatch_table_hash",
    "get_device_status", "status_string", "version", "OP_A8W8_BLOCKSCALE", "OP_BF16", "LIB_PATH",
    "FLAG_STATIC_WEIGHTS", "FLAG_TILED_WEIGHTS", "tile_weight", "tiled_weight_bytes", "gemm_a8w8_blockscale_noalloc", "test_set_wait_fault", "add_rmsnorm_quant",
    "quant_act_mx32", "quant_weight_mx32", "gemm_a8w8_mx32", "mx32_workspace_bytes",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfp8bs.so")
OP_A8W8_BLOCKSCALE = 0
OP_BF16 = 1

STATUS_NAMES = {0: "FP8BS_OK", 1: "FP8BS_ERR_INVALID_ARG", 2: "FP8BS_ERR_UNSUPPORTED", 3: "FP8BS_ERR_ALIGNMENT",
                4: "FP8BS_ERR_WORKSPACE", 5: "FP8BS_ERR_CUDA", 6: "FP8BS_ERR_TIMEOUT"}


class Fp8bsError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)} ({status_string(status)})")


_lib = None

_c_void_p, _i64, _int, _sz, _u64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint64
_PROTOS = {
    "fp8bs_quant_act_per_token_group": (_int, [_c_void_p, _i64, _i64, _i64, _c_void_p, _c_void_p, _int, _c_void_p]),
    "fp8bs_quant_weight_block128": (_int, [_c_void_p, _i64, _i64, _c_void_p, _c_void_p, _c_void_p]),
    "fp8bs_quant_act_mx32": (_int, [_c_void_p, _i64, _i64, _i64, _c_void_p, _c_void_p, _c_void_p]),
    "fp8bs_quant_weight_mx32": (_int, [_c_void_p, _i64, _i64, _c_void_p, _c_void_p, _c_void_p]),
    "fp8bs_mx32_workspace_bytes": (_sz, [_i64, _i64, _i64, _i64]),
    "fp8bs_gemm_a8w8_mx32": (_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _i64, _i64, _i64, _i64,
                                    _c_void_p, _sz, _c_void_p]),
    "fp8bs_add_rmsnorm_quant": (_int, [_c_void_p, _c_void_p, _c_void_p, ctypes.c_float, _i64, _i64, _c_void_p,
                                       _c_void_p, _c_void_p, _c_void_p]),
    "fp8bs_gemm_a8w8_blockscale": (_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _i64, _i64, _i64,
                                          _c_void_p, _sz, _c_void_p]),
    "fp8bs_gemm_a8w8_blockscale_ex": (_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _i64, _i64, _i64,
                                             _c_void_p, _sz, ctypes.c_uint32, _c_void_p]),
    "fp8bs_tiled_weight_bytes": (_sz, [_i64, _i64]),
    "fp8bs_tile_weight_e4m3": (_int, [_c_void_p, _i64, _i64, _c_void_p, _c_void_p]),
    "fp8bs_gemm_a8w8_blockscale_noalloc": (_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _i64, _i64,
                                                  _i64, _c_void_p]),
    "fp8bs_gemm_bf16": (_int, [_c_void_p, _c_void_p, _c_void_p, _int, _i64, _i64, _i64, _c_void_p, _sz, _c_void_p]),
    "fp8bs_workspace_bytes": (_sz, [_int, _i64, _i64, _i64]),
    "fp8bs_dispatch_lookup": (_int, [_int, _i64, _i64, _i64, _int, ctypes.POINTER(_i64), ctypes.POINTER(_int),
                                     ctypes.c_char_p, _sz]),
    "fp8bs_dispatch_set_row": (_int, [_int, _i64, _i64, _i64, ctypes.c_char_p]),
    "fp8bs_dispatch_reset_table": (_int, [_int]),
    "fp8bs_dispatch_list_configs": (_int, [_int, ctypes.c_char_p, _sz]),
    "fp8bs_dispatch_stats": (_int, [_int, ctypes.POINTER(_u64), ctypes.POINTER(_u64), ctypes.POINTER(_u64),
                                    ctypes.POINTER(_u64)]),
    "fp8bs_dispatch_reset_stats": (_int, []),
    "fp8bs_dispatch_dump_json": (_int, [ctypes.c_char_p, _sz]),
    "fp8bs_dispatch_dump_table_json": (_int, [ctypes.c_char_p, _sz]),
    "fp8bs_dispatch_table_hash": (_u64, []),
    "fp8bs_get_device_status": (_int, [_c_void_p]),
    "fp8bs_test_set_wait_fault": (_int, [_u64, _i64]),
    "fp8bs_status_string": (ctypes.c_char_p, [_int]),
    "fp8bs_version": (ctypes.c_char_p, []),
}


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is not built; run `python -m fp8_block_scaled_a8w8_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _PROTOS.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise Fp8bsError(fn, status)


def status_string(status: int) -> str:
    return lib().fp8bs_status_string(status).decode()


def version() -> str:
    return lib().fp8bs_version().decode()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: torch.Tensor) -> int:
    if not t.is_cuda:
        raise ValueError("fp8bs takes device tensors only (no CPU path)")
    return t.data_ptr()


def _is_byte(t: torch.Tensor) -> bool:
    return t.element_size() == 1


# ------------------------------------------------------------------ quantisers
def quant_act_per_token_group(x: torch.Tensor, q: torch.Tensor | None = None, scale: torch.Tensor | None = None,
                              group: int = 128, stream=None):
    """x: bf16 [M, K] (rows may be strided, unit stride along K). Returns (codes float8_e4m3fn [M, K],
    scale float32 [M, K/128])."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D bf16 tensor with unit stride along K")
    M, K = x.shape
    if q is None:
        q = torch.empty((M, K), dtype=torch.float8_e4m3fn, device=x.device)
    if scale is None:
        scale = torch.empty((M, K // group), dtype=torch.float32, device=x.device)
    _check("fp8bs_quant_act_per_token_group",
           lib().fp8bs_quant_act_per_token_group(_ptr(x), M, K, x.stride(0), _ptr(q), _ptr(scale), group,
                                                 _stream(stream)))
    return q, scale


def add_rmsnorm_quant(x: torch.Tensor, residual: torch.Tensor, gamma: torch.Tensor, eps: float = 1e-6,
                      residual_out: torch.Tensor | None = None, q: torch.Tensor | None = None,
                      scale: torch.Tensor | None = None, stream=None):
    """Fused residual add + RMSNorm + per-token 1x128 quantisation (fp8bs_add_rmsnorm_quant).
    x, residual: bf16 [M, K] contiguous; gamma: bf16 [K]. Returns (residual_out bf16 [M, K],
    codes float8_e4m3fn [M, K], scale float32 [M, K/128]); residual_out may be residual."""
    for t in (x, residual, gamma):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("x, residual and gamma must be contiguous bf16 tensors")
    M, K = x.shape
    if residual.shape != (M, K) or gamma.shape != (K,):
        raise ValueError("residual must be [M, K] and gamma [K]")
    if residual_out is None:
        residual_out = torch.empty_like(x)
    if q is None:
        q = torch.empty((M, K), dtype=torch.float8_e4m3fn, device=x.device)
    if scale is None:
        scale = torch.empty((M, K // 128), dtype=torch.float32, device=x.device)
    _check("fp8bs_add_rmsnorm_quant",
           lib().fp8bs_add_rmsnorm_quant(_ptr(x), _ptr(residual), _ptr(gamma), float(eps), M, K, _ptr(residual_out),
                                         _ptr(q), _ptr(scale), _stream(stream)))
    return residual_out, q, scale


def quant_act_mx32(x: torch.Tensor, q: torch.Tensor | None = None, e8m0: torch.Tensor | None = None, stream=None):
    """MX32 activation quantisation (fp8bs_quant_act_mx32): x bf16 [M, K] (unit stride along K).
    Returns (codes float8_e4m3fn [M, K], E8M0 exponents uint8 [M, K/32])."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D bf16 tensor with unit stride along K")
    M, K = x.shape
    if q is None:
        q = torch.empty((M, K), dtype=torch.float8_e4m3fn, device=x.device)
    if e8m0 is None:
        e8m0 = torch.empty((M, K // 32), dtype=torch.uint8, device=x.device)
    _check("fp8bs_quant_act_mx32",
           lib().fp8bs_quant_act_mx32(_ptr(x), M, K, x.stride(0), _ptr(q), _ptr(e8m0), _stream(stream)))
    return q, e8m0


def quant_weight_mx32(w: torch.Tensor, q: torch.Tensor | None = None, e8m0: torch.Tensor | None = None,
                      stream=None):
    """MX32 weight quantisation (32x32 blocks): w float32 [N, K] contiguous. Returns (codes
    float8_e4m3fn [N, K], E8M0 exponents uint8 [ceil(N/32), K/32])."""
    if w.dtype != torch.float32 or w.dim() != 2 or not w.is_contiguous():
        raise ValueError("w must be a contiguous 2-D float32 tensor")
    N, K = w.shape
    if q is None:
        q = torch.empty((N, K), dtype=torch.float8_e4m3fn, device=w.device)
    if e8m0 is None:
        e8m0 = torch.empty(((N + 31) // 32, K // 32), dtype=torch.uint8, device=w.device)
    _check("fp8bs_quant_weight_mx32", lib().fp8bs_quant_weight_mx32(_ptr(w), N, K, _ptr(q), _ptr(e8m0), _stream(stream)))
    return q, e8m0


def mx32_workspace_bytes(batch: int, M: int, N: int, K: int) -> int:
    return int(lib().fp8bs_mx32_workspace_bytes(batch, M, N, K))


def gemm_a8w8_mx32(A: torch.Tensor, a_e8m0: torch.Tensor, W: torch.Tensor, w_e8m0: torch.Tensor,
                   out: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None):
    """MX32 GEMM (fp8bs_gemm_a8w8_mx32). 2-D operands (A [M, K], W [N, K]) are one GEMM;
    3-D stacks (A [b, M, K], W [b, N, K]) are b independent GEMMs. Returns out bf16 [.., M, N]."""
    if not (_is_byte(A) and _is_byte(W)) or A.dim() != W.dim() or A.dim() not in (2, 3):
        raise ValueError("A and W must be 2-D or 3-D one-byte (e4m3 code) tensors of the same rank")
    batch = A.shape[0] if A.dim() == 3 else 1
    M, K = A.shape[-2:]
    N = W.shape[-2]
    for t in (A, a_e8m0, W, w_e8m0):
        if not t.is_contiguous():
            raise ValueError("operands must be contiguous")
    if out is None:
        out = torch.empty(((batch,) if A.dim() == 3 else ()) + (M, N), dtype=torch.bfloat16, device=A.device)
    need = mx32_workspace_bytes(batch, M, N, K)
    if workspace is None:
        workspace = _workspace_for(A.device, need)
    ws_ptr = _ptr(workspace) if workspace is not None else None
    ws_len = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("fp8bs_gemm_a8w8_mx32",
           lib().fp8bs_gemm_a8w8_mx32(_ptr(A), _ptr(a_e8m0), _ptr(W), _ptr(w_e8m0), _ptr(out), batch, M, N, K, ws_ptr,
                                      ws_len, _stream(stream)))
    return out


def quant_weight_block128(w: torch.Tensor, q: torch.Tensor | None = None, scale: torch.Tensor | None = None,
                          stream=None):
    """w: float32 [N, K] contiguous. Returns (codes float8_e4m3fn [N, K], scale float32 [ceil(N/128), K/128])."""
    if w.dtype != torch.float32 or w.dim() != 2 or not w.is_contiguous():
        raise ValueError("w must be a contiguous 2-D float32 tensor")
    N, K = w.shape
    if q is None:
        q = torch.empty((N, K), dtype=torch.float8_e4m3fn, device=w.device)
    if scale is None:
        scale = torch.empty(((N + 127) // 128, K // 128), dtype=torch.float32, device=w.device)
    _check("fp8bs_quant_weight_block128",
           lib().fp8bs_quant_weight_block128(_ptr(w), N, K, _ptr(q), _ptr(scale), _stream(stream)))
    return q, scale


# ------------------------------------------------------------------ workspace
def workspace_bytes(op: int, M: int, N: int, K: int) -> int:
    return int(lib().fp8bs_workspace_bytes(op, M, N, K))


class Workspace:
    """A device scratch buffer, zero-filled when allocated, that grows on demand (torch
    allocates it; the library only uses it). Every call leaves its split-K arrival counters
    at zero and overwrites partial sums before reading them, so one instance serves any
    number of calls issued in order on one stream.

    Growing replaces the buffer: the device is synchronised before (no kernel still uses the
    old one) and after the zero fill (every stream sees the zeros). Growing is refused
    during CUDA-graph capture: size the workspace with an eager call first, or pass one."""

    def __init__(self, device=None):
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.buf = None

    def get(self, nbytes: int) -> torch.Tensor | None:
        if nbytes == 0:
            return None
        if self.buf is None or self.buf.numel() < nbytes:
            if torch.cuda.is_current_stream_capturing():
                raise RuntimeError("the default workspace cannot grow during CUDA-graph capture: make one eager "
                                   "call of this shape first, or pass workspace=")
            torch.cuda.synchronize(self.device)
            self.buf = torch.zeros(((nbytes + 255) // 256) * 256, dtype=torch.uint8, device=self.device)
            torch.cuda.synchronize(self.device)
        return self.buf


_default_ws: dict = {}


def _workspace_for(device, nbytes: int):
    key = (device.index if device.index is not None else torch.cuda.current_device())
    ws = _default_ws.get(key)
    if ws is None:
        ws = _default_ws[key] = Workspace(torch.device("cuda", key))
    return ws.get(nbytes)


# ------------------------------------------------------------------ GEMMs
FLAG_STATIC_WEIGHTS = 1
FLAG_TILED_WEIGHTS = 2


_tiled_bytes = {}


def tiled_weight_bytes(N: int, K: int) -> int:
    v = _tiled_bytes.get((N, K))
    if v is None:
        v = _tiled_bytes[(N, K)] = int(lib().fp8bs_tiled_weight_bytes(N, K))
    return v


def tile_weight(W: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The tiled copy of e4m3 weight codes W [N, K] (fp8bs_tile_weight_e4m3): 16 KiB tiles,
    one per 128-row block and 128-wide K group, for gemm_a8w8_blockscale(tiled_weights=True)."""
    if not _is_byte(W) or W.dim() != 2 or not W.is_contiguous():
        raise ValueError("W must be a contiguous 2-D one-byte (e4m3 code) tensor")
    N, K = W.shape
    nbytes = tiled_weight_bytes(N, K)
    if out is None:
        out = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    _check("fp8bs_tile_weight_e4m3", lib().fp8bs_tile_weight_e4m3(_ptr(W), N, K, _ptr(out), _stream(stream)))
    return out


def gemm_a8w8_blockscale(A: torch.Tensor, a_scale: torch.Tensor, W: torch.Tensor, w_scale: torch.Tensor,
                         out: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None,
                         static_weights: bool = False, tiled_weights: bool = False, N: int | None = None):
    """out[M, N] bf16 = sum_g a_scale[m,g] w_scale[n/128,g] sum_{k in g} A[m,k] W[n,k] (see include/fp8bs.h).

    static_weights: promise that W / w_scale are not written by a kernel still running when
    this call starts (FP8BS_FLAG_STATIC_WEIGHTS); lets the weight stream start early.
    tiled_weights: W is the tiled copy from tile_weight() (FP8BS_FLAG_TILED_WEIGHTS); N must
    then be given."""
    if not (_is_byte(A) and _is_byte(W)) or A.dim() != 2 or (W.dim() != 2 and not tiled_weights):
        raise ValueError("A and W must be 2-D one-byte (e4m3 code) tensors")
    M, K = A.shape
    if tiled_weights:
        if N is None:
            raise ValueError("tiled_weights needs N")
        if W.numel() < tiled_weight_bytes(N, K):
            raise ValueError("W is smaller than the tiled layout of [N, K]")
    else:
        N = W.shape[0]
    for t in (A, W, a_scale, w_scale):
        if not t.is_contiguous():
            raise ValueError("operands must be contiguous")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    if workspace is None:  # a caller's workspace is size-checked by the C entry point
        workspace = _workspace_for(A.device, workspace_bytes(OP_A8W8_BLOCKSCALE, M, N, K))
    ws_ptr = _ptr(workspace) if workspace is not None else None
    ws_len = workspace.numel() * workspace.element_size() if workspace is not None else 0
    flags = (FLAG_STATIC_WEIGHTS if static_weights else 0) | (FLAG_TILED_WEIGHTS if tiled_weights else 0)
    if flags:
        _check("fp8bs_gemm_a8w8_blockscale_ex",
               lib().fp8bs_gemm_a8w8_blockscale_ex(_ptr(A), _ptr(a_scale), _ptr(W), _ptr(w_scale), _ptr(out), M, N, K,
                                                   ws_ptr, ws_len, flags, _stream(stream)))
    else:
        _check("fp8bs_gemm_a8w8_blockscale",
               lib().fp8bs_gemm_a8w8_blockscale(_ptr(A), _ptr(a_scale), _ptr(W), _ptr(w_scale), _ptr(out), M, N, K,
                                                ws_ptr, ws_len, _stream(stream)))
    return out


def gemm_a8w8_blockscale_noalloc(A: torch.Tensor, a_scale: torch.Tensor, W: torch.Tensor, w_scale: torch.Tensor,
                                 out: torch.Tensor | None = None, stream=None):
    """gemm_a8w8_blockscale for M <= 32 without a workspace: for callers that cannot allocate
    device memory when they issue the GEMM (see include/fp8bs.h). Its scratch is one array in
    the library image shared by all calls, so calls must not overlap on the GPU."""
    M, K = A.shape
    N = W.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    _check("fp8bs_gemm_a8w8_blockscale_noalloc",
           lib().fp8bs_gemm_a8w8_blockscale_noalloc(_ptr(A), _ptr(a_scale), _ptr(W), _ptr(w_scale), _ptr(out), M, N,
                                                    K, _stream(stream)))
    return out


def gemm_bf16(A: torch.Tensor, W: torch.Tensor, out_fp32: bool = False, out: torch.Tensor | None = None,
              workspace: torch.Tensor | None = None, stream=None):
    """out[M, N] = A @ W^T with float32 accumulation; bf16 output, or float32 if out_fp32."""
    if A.dtype != torch.bfloat16 or W.dtype != torch.bfloat16 or not A.is_contiguous() or not W.is_contiguous():
        raise ValueError("A and W must be contiguous bf16 tensors")
    M, K = A.shape
    N = W.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32 if out_fp32 else torch.bfloat16, device=A.device)
    if workspace is None:  # a caller's workspace is size-checked by the C entry point
        workspace = _workspace_for(A.device, workspace_bytes(OP_BF16, M, N, K))
    ws_ptr = _ptr(workspace) if workspace is not None else None
    ws_len = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("fp8bs_gemm_bf16",
           lib().fp8bs_gemm_bf16(_ptr(A), _ptr(W), _ptr(out), 1 if out_fp32 else 0, M, N, K, ws_ptr, ws_len,
                                 _stream(stream)))
    return out


# ------------------------------------------------------------------ dispatch table / census
def dispatch_lookup(op: int, M: int, N: int, K: int, record: bool = False):
    """Returns (padded_M or None on a miss, config name)."""
    pm = _i64(0)
    hit = _int(0)
    buf = ctypes.create_string_buffer(64)
    _check("fp8bs_dispatch_lookup",
           lib().fp8bs_dispatch_lookup(op, M, N, K, 1 if record else 0, ctypes.byref(pm), ctypes.byref(hit), buf, 64))
    return (int(pm.value) if hit.value else None), buf.value.decode()


def dispatch_set_row(op: int, M: int, N: int, K: int, cfg: str) -> None:
    _check("fp8bs_dispatch_set_row", lib().fp8bs_dispatch_set_row(op, M, N, K, cfg.encode()))


def dispatch_reset_table(keep_builtin: bool = True) -> None:
    _check("fp8bs_dispatch_reset_table", lib().fp8bs_dispatch_reset_table(1 if keep_builtin else 0))


def dispatch_list_configs(op: int) -> list:
    buf = ctypes.create_string_buffer(4096)
    _check("fp8bs_dispatch_list_configs", lib().fp8bs_dispatch_list_configs(op, buf, 4096))
    return [s for s in buf.value.decode().split("\n") if s]


def dispatch_stats(op: int) -> dict:
    v = [_u64(0) for _ in range(4)]
    _check("fp8bs_dispatch_stats", lib().fp8bs_dispatch_stats(op, *[ctypes.byref(x) for x in v]))
    return dict(zip(["hits", "misses", "distinct_hits", "distinct_misses"], [int(x.value) for x in v]))


def dispatch_reset_stats() -> None:
    _check("fp8bs_dispatch_reset_stats", lib().fp8bs_dispatch_reset_stats())


def dispatch_dump_json() -> list:
    size = 1 << 16
    while True:
        buf = ctypes.create_string_buffer(size)
        st = lib().fp8bs_dispatch_dump_json(buf, size)
        if st == 0:
            return json.loads(buf.value.decode())
        if size > (1 << 28):
            _check("fp8bs_dispatch_dump_json", st)
        size *= 4


def dispatch_dump_table() -> list:
    """The current table rows: dicts with op, M, N, K, cfg and tuned (chosen by measurement)."""
    size = 1 << 16
    while True:
        buf = ctypes.create_string_buffer(size)
        st = lib().fp8bs_dispatch_dump_table_json(buf, size)
        if st == 0:
            return json.loads(buf.value.decode())
        if size > (1 << 28):
            _check("fp8bs_dispatch_dump_table_json", st)
        size *= 4


def dispatch_table_hash() -> str:
    return f"{int(lib().fp8bs_dispatch_table_hash()):016x}"


def get_device_status(stream=None) -> int:
    """Synchronises the stream; returns 0 or the FP8BS_ERR_* code (6 = a device-side wait timed out)."""
    return int(lib().fp8bs_get_device_status(_stream(stream)))


def test_set_wait_fault(wait_limit_ns: int = 0, skip_iteration: int = -1) -> None:
    """Testing hook (fp8bs_test_set_wait_fault): bound every wait of the following
    a8w8_tcw_* / a8w8_tc2_* launches by wait_limit_ns (0 = the default one second) and make CTA 0's
    producer leave K-group iteration skip_iteration unfilled (-1 = none)."""
    st = lib().fp8bs_test_set_wait_fault(int(wait_limit_ns), int(skip_iteration))
    if st:
        raise Fp8bsError("fp8bs_test_set_wait_fault", st)
