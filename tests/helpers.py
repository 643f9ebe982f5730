"""Shared helpers for the GPU parity tests: seeded inputs, oracle comparisons."""

import numpy as np
import torch

from oracle import bf16 as obf16
from oracle import e4m3 as oe4m3
from oracle import gemm as ogemm
from oracle import metrics as ometrics

# Spec tolerance: relative L2 against the oracle <= 3e-3 (the pages report 1.7e-3
# as the bf16 output-rounding floor and 2.5e-3 with split-K bf16 atomics).
REL_L2_TOL = 3e-3


def cuda(t):
    return t.cuda() if isinstance(t, torch.Tensor) else torch.from_numpy(np.ascontiguousarray(t)).cuda()


def codes_to_device(codes: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(codes)).cuda().view(torch.float8_e4m3fn)


def codes_from_device(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.uint8).cpu().numpy()


def abs_sum_a8w8(A_q, a_s, W_q, w_s):
    """sum_g |a_s w_s| sum_k |A W|: the scale of every output's terms (float64)."""
    A = np.abs(oe4m3.decode(A_q))
    W = np.abs(oe4m3.decode(W_q))
    N = W.shape[0]
    out = np.zeros((A.shape[0], N))
    nb = np.arange(N) // 128
    for g in range(A.shape[1] // 128):
        ks = slice(g * 128, (g + 1) * 128)
        out += np.abs(a_s[:, g].astype(np.float64))[:, None] * np.abs(w_s[nb, g].astype(np.float64))[None, :] * (
            A[:, ks] @ W[:, ks].T)
    return out


def check_a8w8(y_bf16: torch.Tensor, A_q, a_s, W_q, w_s, rows=None):
    """Element-wise and relative-L2 parity of a GPU bf16 output against the oracle.

    Element-wise bound: |y - r| <= 2^-8 |r| + 2^-12 * abs_sum, i.e. one bf16 rounding
    (relative error <= 2^-9, doubled for the binade edge) plus an accumulation error of
    2^-12 of the terms' absolute sum -- a tensor core that accumulated each 128-wide
    group with only ~13 significant bits would still meet it; float32 accumulation
    meets it with a wide margin. Returns (rel_l2, max_violation_ratio)."""
    if rows is not None:
        A_q, a_s = A_q[rows], a_s[rows]
    ref, ref_bf16 = ogemm.gemm_a8w8_blockscale(A_q, a_s, W_q, w_s)
    y = y_bf16.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        y = y[rows]
    asum = abs_sum_a8w8(A_q, a_s, W_q, w_s)
    tol = 2.0 ** -8 * np.abs(ref) + 2.0 ** -12 * asum
    err = np.abs(y - ref)
    bad = err > tol
    assert not bad.any(), (f"{bad.sum()} of {bad.size} outputs outside the bound; worst "
                           f"{np.unravel_index(np.argmax(err - tol), err.shape)}")
    rl = ometrics.rel_l2(y, ref)
    assert rl <= REL_L2_TOL, rl
    return rl, ometrics.rel_l2(y, ref_bf16)


def check_mx32(y_bf16: torch.Tensor, A_q, a_e, W_q, w_e, rows=None):
    """Element-wise and relative-L2 parity of a GPU MX32 GEMM output against the MX oracle,
    with the same bound as the 128-block GEMM: one bf16 rounding plus 2^-12 of the terms'
    absolute sum (a float32-accumulating tensor core meets it with a wide margin)."""
    from oracle import mx as omx
    if rows is not None:
        A_q, a_e = A_q[rows], a_e[rows]
    ref, _ = omx.gemm_a8w8_mx32(A_q, a_e, W_q, w_e)
    y = y_bf16.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        y = y[rows]
    A = np.abs(oe4m3.decode(A_q))
    W = np.abs(oe4m3.decode(W_q))
    sa, sw = omx.e8m0_decode(a_e), omx.e8m0_decode(w_e)
    nb = np.arange(W.shape[0]) // 32
    asum = np.zeros_like(ref)
    for g in range(A.shape[1] // 32):
        ks = slice(32 * g, 32 * g + 32)
        asum += sa[:, g][:, None] * sw[nb, g][None, :] * (A[:, ks] @ W[:, ks].T)
    tol = 2.0 ** -8 * np.abs(ref) + 2.0 ** -12 * asum
    bad = np.abs(y - ref) > tol
    assert not bad.any(), f"{bad.sum()} of {bad.size} outputs outside the bound"
    rl = ometrics.rel_l2(y, ref)
    assert rl <= REL_L2_TOL, rl
    return rl


def check_bf16(y: torch.Tensor, A, W, out_fp32: bool, rows=None):
    A = np.asarray(A, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    if rows is not None:
        A = A[rows]
    ref, ref_out = ogemm.gemm_bf16(A, W, out_fp32=out_fp32)
    yy = y.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        yy = yy[rows]
    asum = np.abs(A) @ np.abs(W).T
    rel = 2.0 ** -22 if out_fp32 else 2.0 ** -8
    tol = rel * np.abs(ref) + 2.0 ** -16 * asum
    err = np.abs(yy - ref)
    bad = err > tol
    assert not bad.any(), f"{bad.sum()} of {bad.size} outputs outside the bound"
    rl = ometrics.rel_l2(yy, ref)
    assert rl <= (1e-5 if out_fp32 else REL_L2_TOL), rl
    return rl


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy()
