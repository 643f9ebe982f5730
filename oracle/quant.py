"""Block quantisers of the a8w8 block-scale scheme.

Activations: per token, per 1x128 group along K. Weights: per 128x128 block.
In both, scale = amax / 448 and code = e4m3_rn_sat(x / scale) ([cookbook#8]:
the checkpoint is block quantised with weight_block_size [128,128], so its
dense layers take gemm_a8w8_blockscale; the 1x128 activation group is the
per-token-group granularity that pairs with it).

Arithmetic is IEEE float32, the precision the GPU quantiser works in, so the
fp8 codes and the scales are comparable bit for bit:
  amax  = max |x| over the group (exact: a max of float32 values)
  scale = float32(amax) / float32(448)          (one correctly rounded division)
  code  = encode_rn_sat(float32(x) / scale)     (one correctly rounded division,
                                                 then one RN-sat rounding)
A group whose amax is 0 has scale 0 and codes encode(+-0) = 0x00 / 0x80; the
pages are silent on this case and this is the plainest reading (the group
contributes nothing to the GEMM either way).

Parity: pinned in tests/test_oracle_quant.py (hand-computed groups, the
max-element-encodes-to-448 property, half-ulp reconstruction bound, zero and
tail groups, and a plant-a-mistake check).
"""

import numpy as np

from .e4m3 import encode_rn_sat, E4M3_MAX

GROUP = 128


def quant_act_per_token_group(x, group: int = GROUP):
    """x: [M, K] float32 holding bf16 values. Returns (codes uint8 [M, K], scale float32 [M, K/group])."""
    x = np.asarray(x, dtype=np.float32)
    M, K = x.shape
    assert group == GROUP and K % group == 0
    G = K // group
    codes = np.empty((M, K), dtype=np.uint8)
    scales = np.empty((M, G), dtype=np.float32)
    for g in range(G):
        blk = x[:, g * group:(g + 1) * group]
        amax = np.max(np.abs(blk), axis=1)  # [M], float32
        s = (amax / np.float32(E4M3_MAX)).astype(np.float32)
        scales[:, g] = s
        safe = np.where(s == 0, np.float32(1), s).astype(np.float32)
        y = (blk / safe[:, None]).astype(np.float32)
        y = np.where((s == 0)[:, None], blk, y)  # amax 0: the group is all +-0
        codes[:, g * group:(g + 1) * group] = encode_rn_sat(y)
    return codes, scales


def quant_weight_block128(w, block: int = 128):
    """w: [N, K] float32. Returns (codes uint8 [N, K], scale float32 [ceil(N/128), K/128]).

    A partial last block of rows (N % 128 != 0) is quantised over the rows it has.
    """
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    assert K % block == 0
    NB = (N + block - 1) // block
    G = K // block
    codes = np.empty((N, K), dtype=np.uint8)
    scales = np.empty((NB, G), dtype=np.float32)
    for nb in range(NB):
        r0, r1 = nb * block, min(N, (nb + 1) * block)
        for g in range(G):
            blk = w[r0:r1, g * block:(g + 1) * block]
            amax = np.float32(np.max(np.abs(blk)))
            s = np.float32(amax / np.float32(E4M3_MAX))
            scales[nb, g] = s
            y = blk if s == 0 else (blk / s).astype(np.float32)
            codes[r0:r1, g * block:(g + 1) * block] = encode_rn_sat(y)
    return codes, scales
