"""Quantiser kernels vs the oracle: bit-exact codes and scales."""

import numpy as np
import pytest
import torch

import fp8_block_scaled_a8w8_b200 as fb
from fp8_block_scaled_a8w8_b200 import inputs
from oracle import quant as oquant
from tests.helpers import codes_from_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,K,outliers", [(1, 128, False), (3, 6144, False), (37, 5120, True), (257, 1024, False),
                                          (1, 6144, False), (4096, 6144, True), (16384, 512, False)])
def test_act_quant_bit_exact(M, K, outliers):
    x = inputs.activation_bf16(M, K, seed=M * 7 + K, outliers=outliers)
    q, s = fb.quant_act_per_token_group(x.cuda())
    torch.cuda.synchronize()
    q_o, s_o = oquant.quant_act_per_token_group(x.float().numpy())
    assert np.array_equal(codes_from_device(q), q_o)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_o.view(np.uint32))


def test_act_quant_edge_groups():
    K = 768
    x = torch.zeros((5, K), dtype=torch.float32)
    x[1, :128] = -0.0                                     # all -0 group
    x[2, 5] = 3.0                                         # single nonzero
    x[3, :] = torch.linspace(-3e38, 3e38, K, dtype=torch.float64).float()  # huge finite values
    x[4, 128:256] = 2.0 ** -133                           # bf16 subnormals
    x[4, 300] = -(2.0 ** -130)
    x[0, 640:768] = torch.tensor([2.0 ** (i % 20 - 10) * (-1) ** i for i in range(128)])
    xb = x.to(torch.bfloat16)
    q, s = fb.quant_act_per_token_group(xb.cuda())
    torch.cuda.synchronize()
    q_o, s_o = oquant.quant_act_per_token_group(xb.float().numpy())
    assert np.array_equal(codes_from_device(q), q_o)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_o.view(np.uint32))
    assert s_o[0, 0] == 0 and np.all(q_o[1, :128] == 0x80)


def test_act_quant_strided_rows():
    M, K, ld = 9, 1024, 1536
    big = inputs.activation_bf16(M, ld, seed=5)
    xv = big.cuda()[:, :K]
    q, s = fb.quant_act_per_token_group(xv)
    torch.cuda.synchronize()
    q_o, s_o = oquant.quant_act_per_token_group(big[:, :K].float().numpy())
    assert np.array_equal(codes_from_device(q), q_o)
    assert np.array_equal(s.cpu().numpy(), s_o)


@pytest.mark.parametrize("N,K", [(300, 384), (5120, 6144), (16, 128)])
def test_weight_quant_bit_exact(N, K):
    w = inputs.weight_f32(N, K, seed=N + K)
    q, s = fb.quant_weight_block128(w.cuda())
    torch.cuda.synchronize()
    q_o, s_o = oquant.quant_weight_block128(w.numpy())
    assert np.array_equal(codes_from_device(q), q_o)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_o.view(np.uint32))


def _cvt_probe_values(n_random: int, seed: int) -> np.ndarray:
    """Every midpoint between adjacent positive e4m3 values, one float32 ulp either side,
    their negatives, the grid values themselves, and n_random uniform values in
    [-448, 448] (float32)."""
    from oracle import e4m3
    pos = e4m3.decode(np.arange(0x7F, dtype=np.uint8))
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    special = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(np.inf)),
                              pos.astype(np.float32)])
    special = np.concatenate([special, -special])
    rnd = np.random.default_rng(seed).uniform(-448.0, 448.0, n_random).astype(np.float32)
    return np.concatenate([special, rnd])


def test_hardware_cvt_matches_oracle_encoder():
    """The GPU's e4m3 conversion (cvt.rn.satfinite) against the oracle's encoder, through
    the weight quantiser with every 128x128 block's scale pinned to exactly 1 (each block
    holds one 448): then each code is the conversion of the value itself. All float32
    midpoints and their neighbours plus 10^7 random values."""
    from oracle import e4m3
    vals = _cvt_probe_values(10_000_000, seed=11)
    per_block = 128 * 128 - 1
    nblk = -(-vals.size // per_block)
    flat = np.zeros(nblk * per_block, dtype=np.float32)
    flat[:vals.size] = vals
    blocks = np.concatenate([np.full((nblk, 1), 448.0, dtype=np.float32), flat.reshape(nblk, per_block)], axis=1)
    # block i occupies rows 128 * (i // G) .. +128, columns 128 * (i % G) .. +128
    G = 16
    nb_rows = -(-nblk // G)
    w = np.zeros((nb_rows * 128, G * 128), dtype=np.float32)
    for i in range(nblk):
        r, c = 128 * (i // G), 128 * (i % G)
        w[r:r + 128, c:c + 128] = blocks[i].reshape(128, 128)
    for i in range(nblk, nb_rows * G):  # padding blocks: a 448 keeps their scale 1 too
        r, c = 128 * (i // G), 128 * (i % G)
        w[r, c] = 448.0
    q, s = fb.quant_weight_block128(torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    assert np.all(s.cpu().numpy() == np.float32(1.0))
    assert np.array_equal(codes_from_device(q), e4m3.encode_rn_sat(w))
