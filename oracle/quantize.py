"""Quantisation stage of SageAttention-style attention, as a plain CPU oracle.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

INT8/FP8 path (thu-ml/sageattention llms.txt: "sageattn_qk_int8_pv_fp16_triton"
-- per-block INT8 quantisation of Q and K with ``smooth_k``;
"sageattn_qk_int8_pv_fp8_cuda" -- INT8 Q/K and per-channel FP8 V):

1. K smoothing: subtract, from every K channel, its mean over the tokens
   (the mean is exact and rounded once to fp32; the subtraction is an fp32
   subtraction).  Softmax is unchanged by a per-row constant, so this only
   moves the quantisation error.
2. Q and K: blocks of 128 tokens x all D channels per (batch, head).  With
   a = max|x| over the block: scale = fp32(a / 127), inv = fp32(127 / a),
   code = clamp(round_half_even(fp32(x * inv)), -127, 127); a == 0 gives
   scale 0 and all-zero codes.  Padding tokens (n >= N) have code 0.
3. V: one scale per (batch, KV head, channel) over all tokens.  With
   a = max|v|: vscale = fp32(a / 448), inv = fp32(448 / a),
   code = E4M3_rn_satfinite(fp32(v * inv)); a == 0 gives vscale 0 and code
   0x00.  Stored transposed, [B, Hkv, D, N_pad], so each channel's tokens
   are contiguous.
4. q_dot_kmean[b, h, n] = sum_c q[b,h,n,c] * kmean[b, h // G, c] (float64),
   the term that turns the LSE of the smoothed scores back into the LSE of
   the original scores.

NVFP4 path ("flashinfer.nvfp4_attention_sm120_fwd": packed FP4 Q/K/V with
per-vector FP8 scale factors, V stored transposed, ``qk_correction`` with
one row per 128-token Q block, ``per_block_mean``, ``unpadded_k_len``):

1. K: mean over the first ``unpadded_k_len`` tokens, subtracted as above;
   rows at and beyond that length are zero.
2. Q: mean over each 128-token Q block (``per_block_mean``; the valid rows
   of the block) or over all Q tokens (global mean), subtracted in fp32.
3. Every 16-element vector (along D for Q and K, along tokens for the
   transposed V) with a = max|x|: sf = E4M3(fp32(a / 6)), s = value(sf);
   s == 0 gives zero codes, else inv = fp32(1 / s) and
   code = E2M1_rn_satfinite(fp32(x * inv)).
4. qk_correction[b, h, qb, j] = fp32(sum_c qmean[b,h,qb,c] * Ks[b,g,j,c])
   (float64 sum), the part of Q.K^T that the Q mean removed.
"""
from __future__ import annotations

import numpy as np

from . import formats as F

BLOCK = 128
NVFP4_VEC = 16


def _np64(t):
    """float64 numpy copy of a torch tensor or array (exact for bf16/fp16)."""
    try:
        import torch
        if isinstance(t, torch.Tensor):
            return t.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(t, dtype=np.float64)


def pad_to(n, b=BLOCK):
    return (n + b - 1) // b * b


def int8_block_quant(x, n_valid, block=BLOCK):
    """Per-block symmetric INT8 quantisation along tokens.

    x: float32-valued array [..., N, D] (N = valid tokens).  Returns
    (codes int8 [..., N_pad, D], scale float32 [..., N_pad / block]).
    """
    x = np.asarray(x, dtype=np.float64)
    lead, (N, D) = x.shape[:-2], x.shape[-2:]
    assert N == n_valid
    Np = pad_to(N, block)
    xp = np.zeros(lead + (Np, D), dtype=np.float32)
    xp[..., :N, :] = x
    nb = Np // block
    xb = xp.reshape(lead + (nb, block * D))
    a = np.max(np.abs(xb), axis=-1)                         # exact
    scale = np.float32(a) / np.float32(127.0)               # fp32 division
    with np.errstate(divide="ignore"):
        inv = np.where(a > 0, np.float32(127.0) / np.where(a > 0, a, 1).astype(np.float32),
                       np.float32(0))
    y = xb * inv.astype(np.float32)[..., None]              # fp32 product
    code = np.clip(np.rint(y), -127, 127).astype(np.int8)
    return code.reshape(lead + (Np, D)), scale.astype(np.float32)


def fp8_channel_quant(v):
    """Per-channel E4M3 quantisation of V over all tokens.

    v: [..., N, D] float32-valued.  Returns (codes uint8 [..., D, N_pad]
    transposed, vscale float32 [..., D]).
    """
    v = np.asarray(v, dtype=np.float32)
    lead, (N, D) = v.shape[:-2], v.shape[-2:]
    a = np.max(np.abs(v), axis=-2)                          # [..., D]
    vscale = a / np.float32(448.0)
    inv = np.where(a > 0, np.float32(448.0) / np.where(a > 0, a, 1).astype(np.float32),
                   np.float32(0)).astype(np.float32)
    y = v * inv[..., None, :]                               # fp32 product
    code = F.e4m3_encode(y.astype(np.float64))
    code = np.where((a > 0)[..., None, :], code, np.uint8(0)).astype(np.uint8)
    Np = pad_to(N)
    out = np.zeros(lead + (D, Np), dtype=np.uint8)
    out[..., :, :N] = np.swapaxes(code, -1, -2)
    return out, vscale.astype(np.float32)


def quantize_qkv_i8f8(q, k, v, smooth_k=True):
    """Oracle of the INT8/FP8 quantisation stage.

    q: [B, Hq, Nq, D]; k, v: [B, Hkv, Nk, D] (bf16/fp16 values; torch tensors
    or float arrays).  Returns a dict of numpy arrays with the layouts the
    CUDA path writes.
    """
    q, k, v = _np64(q), _np64(k), _np64(v)
    B, Hq, Nq, D = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    if smooth_k:
        km = F.exact_mean_f32(k)                            # [B, Hkv, D] fp32
    else:
        km = np.zeros((B, Hkv, D), dtype=np.float32)
    ks = k.astype(np.float32) - km[:, :, None, :]           # fp32 subtraction
    q_code, q_scale = int8_block_quant(q.astype(np.float32), Nq)
    k_code, k_scale = int8_block_quant(ks, Nk)
    v_code_t, v_scale = fp8_channel_quant(v.astype(np.float32))
    kmq = np.repeat(km.astype(np.float64), G, axis=1)       # KV head of Q head h is h // G
    qdk = np.einsum("bhnc,bhc->bhn", q, kmq)
    return dict(q=q_code, q_scale=q_scale, k=k_code, k_scale=k_scale, k_mean=km,
                v_t=v_code_t, v_scale=v_scale, q_dot_kmean=qdk,
                B=B, Hq=Hq, Hkv=Hkv, Nq=Nq, Nk=Nk, D=D)


def fp4_vector_quant(x):
    """NVFP4 quantisation of 16-element vectors along the last axis.

    x: float32-valued [..., L] with L % 16 == 0.  Returns (codes uint8
    [..., L] holding 0..15, scale-factor codes uint8 E4M3 [..., L/16]).
    """
    x = np.asarray(x, dtype=np.float32)
    lead, L = x.shape[:-1], x.shape[-1]
    xv = x.reshape(lead + (L // NVFP4_VEC, NVFP4_VEC))
    a = np.max(np.abs(xv), axis=-1)
    sf = F.e4m3_encode((a / np.float32(6.0)).astype(np.float64))   # fp32 division, then E4M3
    s = F.e4m3_decode(sf).astype(np.float32)
    inv = np.where(s > 0, np.float32(1.0) / np.where(s > 0, s, 1).astype(np.float32),
                   np.float32(0)).astype(np.float32)
    y = xv * inv[..., None]                                         # fp32 product
    code = F.e2m1_encode(y.astype(np.float64))
    code = np.where((s > 0)[..., None], code, np.uint8(0)).astype(np.uint8)
    return code.reshape(lead + (L,)), sf.astype(np.uint8)


def quantize_qkv_nvfp4(q, k, v, per_block_mean=True, unpadded_k_len=None):
    """Oracle of the NVFP4 quantisation stage (see module docstring).

    Returns unpacked codes (one E2M1 code per byte) plus the packed form the
    CUDA path writes (``*_packed``: element 2i in the low nibble).
    """
    q, k, v = _np64(q), _np64(k), _np64(v)
    B, Hq, Nq, D = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    L = Nk if unpadded_k_len is None else int(unpadded_k_len)
    Nqp, Nkp = pad_to(Nq), pad_to(Nk)
    km = F.exact_mean_f32(k[:, :, :L, :], count=L) if L > 0 else np.zeros((B, Hkv, D), np.float32)
    ks = np.zeros((B, Hkv, Nkp, D), dtype=np.float32)
    ks[:, :, :L] = k[:, :, :L].astype(np.float32) - km[:, :, None, :]
    vz = np.zeros((B, Hkv, Nkp, D), dtype=np.float32)
    vz[:, :, :L] = v[:, :, :L]
    nqb = Nqp // BLOCK
    qmean = np.zeros((B, Hq, nqb, D), dtype=np.float32)
    if per_block_mean:
        for qb in range(nqb):
            lo, hi = qb * BLOCK, min(Nq, (qb + 1) * BLOCK)
            qmean[:, :, qb] = F.exact_mean_f32(q[:, :, lo:hi, :], count=hi - lo)
    else:
        qmean[:] = F.exact_mean_f32(q, count=Nq)[:, :, None, :]
    qs = np.zeros((B, Hq, Nqp, D), dtype=np.float32)
    row_blk = np.arange(Nq) // BLOCK
    qs[:, :, :Nq] = q.astype(np.float32) - qmean[:, :, row_blk, :]
    q_code, q_sf = fp4_vector_quant(qs)
    k_code, k_sf = fp4_vector_quant(ks)
    v_code_t, v_sf_t = fp4_vector_quant(np.swapaxes(vz, -1, -2))   # [B, Hkv, D, Nkp]
    ksq = np.repeat(ks.astype(np.float64), G, axis=1)              # [B, Hq, Nkp, D]
    corr = np.einsum("bhqc,bhjc->bhqj", qmean.astype(np.float64), ksq).astype(np.float32)
    kmq = np.repeat(km.astype(np.float64), G, axis=1)
    qdk = np.einsum("bhnc,bhc->bhn", q, kmq)
    return dict(q=q_code, q_sf=q_sf, k=k_code, k_sf=k_sf, v_t=v_code_t, v_sf_t=v_sf_t,
                q_packed=F.pack_e2m1(q_code), k_packed=F.pack_e2m1(k_code),
                v_t_packed=F.pack_e2m1(v_code_t),
                qk_correction=corr, q_mean=qmean, k_mean=km, q_dot_kmean=qdk,
                B=B, Hq=Hq, Hkv=Hkv, Nq=Nq, Nk=Nk, D=D, unpadded_k_len=L,
                per_block_mean=bool(per_block_mean))
