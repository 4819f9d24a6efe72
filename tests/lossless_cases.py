"""Inputs on which quantisation is lossless, so that the quantised
attention must equal exact fp64 attention.

INT8/FP8 case:
* Q and K carry integers in {-1, 0, 1} on channels 0..6 (so the integer
  scores lie in [-7, 7]); every 128-token block of Q has one +-127 on
  channel 7 and every block of K one +-127 on channel 8, with the partner
  operand zero on those channels.  Both per-block scales are therefore
  exactly 127 / 127 = 1 and the codes equal the values.
* K is built as [X; -X] over tokens, so every channel mean is exactly 0 and
  smoothing leaves K unchanged.
* V holds E4M3-exact values with a 448 in every channel, so vscale = 1.
* With sm_scale = ln 2 the probabilities are 2**(S - m) with S - m an integer
  in [-14, 0], and 448 * 2**-k is an exact E4M3 value for k <= 14.

NVFP4 case: the same idea with 16-element vectors.  Every vector holds one
+-6 (scale factor exactly 1) on a channel whose partner is zero; Q blocks
and K are [X; -X] (means 0, qk_correction 0); keys repeat in groups of 16
so that P is constant inside each 16-key vector and quantises exactly.
"""
import math

import torch

import workloads as W

LN2 = math.log(2.0)
E4M3_SMALL = [-3.0, -2.0, -1.5, -1.0, -0.5, 0.0, 0.5, 1.0, 1.5, 2.0, 3.0]
E2M1_VALUES = [-6.0, -4.0, -3.0, -2.0, -1.5, -1.0, -0.5, 0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _choice(values, shape, seed):
    idx = W.random_integer_tensor(shape, 0, len(values) - 1, seed).long()
    return torch.tensor(values, dtype=torch.float64)[idx]


def i8f8_case(B=1, Hq=2, Hkv=2, N=256, D=64, seed=0):
    """(q, k, v) bf16 tensors for the lossless INT8/FP8 case (N even)."""
    assert N % 2 == 0 and D >= 16
    half = N // 2
    q = torch.zeros(B, Hq, N, D, dtype=torch.float64)
    q[..., :7] = W.random_integer_tensor((B, Hq, N, 7), -1, 1, seed)
    sign = W.random_integer_tensor((B, Hq, N), 0, 1, seed + 1) * 2 - 1
    for s in range(0, N, 128):
        q[:, :, s, 7] = 127.0 * sign[:, :, s]
    x = torch.zeros(B, Hkv, half, D, dtype=torch.float64)
    x[..., :7] = W.random_integer_tensor((B, Hkv, half, 7), -1, 1, seed + 2)
    for s in range(0, N, 128):               # one +-127 in every 128-token block of [X; -X]
        r = s if s < half else s - half
        x[:, :, r, 8] = 127.0
    k = torch.cat([x, -x], dim=2)
    v = _choice(E4M3_SMALL, (B, Hkv, N, D), seed + 3)
    v[:, :, 0, :] = 448.0
    return tuple(t.to(torch.bfloat16) for t in (q, k, v))


def nvfp4_case(B=1, Hq=2, Hkv=2, N=256, D=64, L=None, seed=0):
    """(q, k, v) bf16 tensors for the lossless NVFP4 case.

    N % 128 == 0; keys valid below L (default N), L % 32 == 0.
    """
    L = N if L is None else L
    assert N % 128 == 0 and D % 16 == 0 and L % 32 == 0
    nv = D // 16
    # Q: per 128-token block [X; -X]; channels 0..6 of vector 0 in {-1,0,1};
    # channel 16v+15 = +-6 in every vector, partner (K) zero there.
    q = torch.zeros(B, Hq, N, D, dtype=torch.float64)
    xq = torch.zeros(B, Hq, N // 2, D, dtype=torch.float64)
    xq[..., :7] = W.random_integer_tensor((B, Hq, N // 2, 7), -1, 1, seed)
    sq = W.random_integer_tensor((B, Hq, N // 2, nv), 0, 1, seed + 1) * 12 - 6
    for j in range(nv):
        xq[..., 16 * j + 15] = sq[..., j]
    for blk in range(N // 128):
        a = xq[:, :, blk * 64:(blk + 1) * 64]
        q[:, :, blk * 128:blk * 128 + 64] = a
        q[:, :, blk * 128 + 64:(blk + 1) * 128] = -a
    # K: [Y; -Y] over the L valid tokens, rows repeated in groups of 16.
    nd = L // 32
    y = torch.zeros(B, Hkv, nd, D, dtype=torch.float64)
    y[..., :7] = W.random_integer_tensor((B, Hkv, nd, 7), -1, 1, seed + 2)
    sk = W.random_integer_tensor((B, Hkv, nd, nv), 0, 1, seed + 3) * 12 - 6
    for j in range(nv):
        y[..., 16 * j + 14] = sk[..., j]
    y = y.repeat_interleave(16, dim=2)
    k = torch.zeros(B, Hkv, N, D, dtype=torch.float64)
    k[:, :, :L] = torch.cat([y, -y], dim=2)
    # V: E2M1 grid values with a 6 in every 16-token vector of every channel.
    v = torch.zeros(B, Hkv, N, D, dtype=torch.float64)
    v[:, :, :L] = _choice(E2M1_VALUES, (B, Hkv, L, D), seed + 4)
    v[:, :, 0:L:16, :] = 6.0
    return tuple(t.to(torch.bfloat16) for t in (q, k, v))
