"""Pins for oracle/quantize.py: error bounds, exact means, special values,
and the qk_correction identity (no GPU)."""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W


def _qkv(N=300, D=64, B=1, Hq=4, Hkv=2, seed=0, std=2.0):
    w = W.TINY.scaled(B=B, Hq=Hq, Hkv=Hkv, N=N, D=D, seed=seed, k_offset_std=std)
    return W.make_qkv(w)


def test_int8_block_codes_are_nearest_and_saturate_at_block_max():
    q, k, v = _qkv()
    x = q.double().numpy()
    codes, scale = O.int8_block_quant(x.astype(np.float32), x.shape[2])
    N = x.shape[2]
    for blk in range(scale.shape[-1]):
        lo, hi = blk * 128, min(N, blk * 128 + 128)
        xb = x[:, :, lo:hi]
        cb = codes[:, :, lo:hi].astype(np.float64)
        a = np.abs(xb).reshape(xb.shape[0], xb.shape[1], -1).max(-1)
        s = scale[..., blk].astype(np.float64)
        np.testing.assert_allclose(s, a / 127, rtol=2 ** -23)
        # the block's largest magnitude maps to +-127
        assert np.all(np.abs(cb).reshape(cb.shape[0], cb.shape[1], -1).max(-1) == 127)
        # every code is the integer nearest to x / scale (within rounding of inv)
        err = np.abs(cb - xb / s[..., None, None])
        assert err.max() <= 0.5 + 1e-5
    # padding rows of the last block are zero
    assert np.all(codes[:, :, N:] == 0)


def test_int8_zero_block():
    x = np.zeros((1, 1, 128, 64), np.float32)
    codes, scale = O.int8_block_quant(x, 128)
    assert scale[0, 0, 0] == 0 and np.all(codes == 0)


def test_smooth_k_uses_exact_channel_mean():
    q, k, v = _qkv(N=257)
    qz = O.quantize_qkv_i8f8(q, k, v, smooth_k=True)
    kk = k.double().numpy()
    for b, h, c in [(0, 0, 0), (0, 1, 5), (0, 1, 63)]:
        s = sum((Fraction(float(t)) for t in kk[b, h, :, c]), Fraction(0))
        assert qz["k_mean"][b, h, c] == np.float32(O.fraction_to_f32(s / 257))
    # the smoothed K has (nearly) zero channel means: reconstruct from codes
    ks = kk.astype(np.float32) - qz["k_mean"][:, :, None, :]
    assert np.abs(ks.mean(axis=2)).max() < 1e-5
    # smooth_k off -> zero mean vector and codes of K itself
    qz0 = O.quantize_qkv_i8f8(q, k, v, smooth_k=False)
    assert np.all(qz0["k_mean"] == 0)
    c0, _ = O.int8_block_quant(kk.astype(np.float32), 257)
    np.testing.assert_array_equal(qz0["k"], c0)


def test_v_fp8_per_channel_scale_and_transpose():
    q, k, v = _qkv(N=200)
    qz = O.quantize_qkv_i8f8(q, k, v)
    vv = v.double().numpy()
    a = np.abs(vv).max(axis=2)                                 # [B, Hkv, D]
    np.testing.assert_allclose(qz["v_scale"], a / 448, rtol=2 ** -23)
    dec = O.e4m3_decode(qz["v_t"]) * qz["v_scale"][..., None]  # [B, Hkv, D, Np]
    assert np.all(qz["v_t"][..., 200:] == 0)
    back = np.swapaxes(dec[..., :200], -1, -2)
    # E4M3 relative error <= 2**-4 for normals; absolute 2**-10 * scale below
    tol = np.maximum(np.abs(vv) * 2 ** -4, 2 ** -10 * qz["v_scale"][:, :, None, :])
    assert np.all(np.abs(back - vv) <= tol * (1 + 1e-6))
    # each channel's largest magnitude maps to code +-448 (0x7E / 0xFE)
    mx = np.max(np.abs(O.e4m3_decode(qz["v_t"])), axis=-1)
    assert np.all(mx == 448)


def test_q_dot_kmean_restores_unsmoothed_lse():
    """Shift invariance: LSE(Q, K) - LSE(Q, K - kmean) = sm_scale * q . kmean."""
    q, k, v = _qkv(N=256, D=64)
    qz = O.quantize_qkv_i8f8(q, k, v)
    km = torch.from_numpy(qz["k_mean"].astype(np.float64))
    ks = k.double() - km[:, :, None, :]
    out1, lse1 = O.exact_attention(q, k, v, sm_scale=0.125)
    out2, lse2 = O.exact_attention(q.double(), ks, v.double(), sm_scale=0.125)
    np.testing.assert_allclose(out1, out2, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse1 - lse2, 0.125 * qz["q_dot_kmean"], rtol=1e-9, atol=1e-9)


def test_fp4_vector_quant_bounds():
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(64, 128, generator=g) * 3).float().numpy()
    codes, sf = O.fp4_vector_quant(x)
    s = O.e4m3_decode(sf)
    dec = (O.e2m1_decode(codes).reshape(64, 8, 16) * s[..., None]).reshape(64, 128)
    a = np.abs(x.reshape(64, 8, 16)).max(-1)
    np.testing.assert_array_equal(sf, O.e4m3_encode((a / np.float32(6)).astype(np.float64)))
    # elementwise error is at most half a step of the E2M1 grid at that scale
    # (steps 0.5 / 1 / 2 for |y| < 2 / < 4 / <= 6), scale-relative.
    y = np.abs(x) / np.repeat(s, 16, axis=-1)
    step = np.where(y < 2, 0.5, np.where(y < 4, 1.0, 2.0))
    assert np.all(np.abs(dec - x) <= 0.5 * step * np.repeat(s, 16, axis=-1) * (1 + 1e-5) + 1e-6)


@pytest.mark.parametrize("per_block_mean", [True, False])
def test_nvfp4_qk_correction_identity(per_block_mean):
    """Q.Ks^T == (Q - qmean).Ks^T + qk_correction (the part the Q mean removed)."""
    q, k, v = _qkv(N=256, D=64, Hq=2, Hkv=1)
    qz = O.quantize_qkv_nvfp4(q, k, v, per_block_mean=per_block_mean, unpadded_k_len=240)
    qq = q.double().numpy()
    km = qz["k_mean"].astype(np.float64)
    kk = k.double().numpy()
    ks = np.zeros_like(kk)
    ks[:, :, :240] = (kk[:, :, :240].astype(np.float32) - qz["k_mean"][:, :, None]).astype(np.float64)
    G = 2
    for h in range(2):
        full = qq[0, h] @ ks[0, h // G].T
        qm = qz["q_mean"][0, h][np.arange(256) // 128].astype(np.float64)
        part = (qq[0, h] - qm) @ ks[0, h // G].T
        corr = qz["qk_correction"][0, h][np.arange(256) // 128][:, :256]
        np.testing.assert_allclose(part + corr, full, atol=2e-4 * np.abs(full).max())
    # block means of the smoothed Q vanish; K rows beyond unpadded length are zero
    assert np.all(qz["k"][:, :, 240:] == 0) and np.all(qz["k_sf"][:, :, 240:] == 0)
    del km


def test_nvfp4_global_mean_is_shared_by_blocks():
    q, k, v = _qkv(N=256, D=64, Hq=2, Hkv=2)
    qz = O.quantize_qkv_nvfp4(q, k, v, per_block_mean=False)
    np.testing.assert_array_equal(qz["q_mean"][:, :, 0], qz["q_mean"][:, :, 1])
    qzb = O.quantize_qkv_nvfp4(q, k, v, per_block_mean=True)
    assert not np.array_equal(qzb["q_mean"][:, :, 0], qzb["q_mean"][:, :, 1])


# ------------------------------------------------------------ NVFP4 means, pinned by exact sums
# ("flashinfer.nvfp4_attention_sm120_fwd": ``per_block_mean`` -- one Q mean per
# 128-token Q block, qk_correction "one row per 128-token Q block";
# ``unpadded_k_len`` -- keys at and beyond it are padding; thu-ml/sageattention
# llms.txt, "FP4 Attention for Blackwell GPUs": per_block_mean off uses one
# global mean instead)
def _offset_blocks(q, offsets):
    """Q with a constant added to every row of each 128-token block, so that
    block means differ by far more than the FP4 quantisation error."""
    q = q.clone().double()
    for blk, off in enumerate(offsets):
        q[:, :, blk * 128:(blk + 1) * 128] += off
    return q.to(torch.bfloat16)


def _frac_mean(x, lo, hi):
    return O.fraction_to_f32(sum((Fraction(float(t)) for t in x[lo:hi]), Fraction(0)) / (hi - lo))


@pytest.mark.parametrize("per_block_mean", [True, False])
def test_nvfp4_q_means_are_exact_means_of_the_valid_rows(per_block_mean):
    """N = 300: blocks of 128, 128 and 44 valid rows.  Each q_mean entry is
    the exact mean of exactly the valid rows of its block (or of all 300
    rows), rounded once to fp32: a divisor of 128 for the ragged block, rows
    assigned to the wrong block or padding rows in the sum all fail."""
    q, k, v = _qkv(N=300, D=64, Hq=2, Hkv=1, seed=21)
    q = _offset_blocks(q, [5.0, -3.0, 8.0])
    qz = O.quantize_qkv_nvfp4(q, k, v, per_block_mean=per_block_mean, unpadded_k_len=300)
    qq = q.double().numpy()
    assert qz["q_mean"].shape == (1, 2, 3, 64)
    for h in range(2):
        for c in (0, 17, 63):
            col = qq[0, h, :, c]
            for qb, (lo, hi) in enumerate([(0, 128), (128, 256), (256, 300)]):
                want = _frac_mean(col, lo, hi) if per_block_mean else _frac_mean(col, 0, 300)
                assert qz["q_mean"][0, h, qb, c] == np.float32(want), (h, c, qb)


def test_nvfp4_k_mean_is_over_the_unpadded_keys_only():
    """unpadded_k_len = 250 of N = 300, with the 50 padding rows far from the
    others (+10): the K mean is the exact mean of rows 0..249 alone, and the
    smoothed K reconstructed from its codes tracks K - that mean."""
    q, k, v = _qkv(N=300, D=64, Hq=2, Hkv=1, seed=22)
    k = k.clone().double()
    k[:, :, 250:] += 10.0
    k = k.to(torch.bfloat16)
    qz = O.quantize_qkv_nvfp4(q, k, v, per_block_mean=True, unpadded_k_len=250)
    kk = k.double().numpy()
    for c in range(64):
        assert qz["k_mean"][0, 0, c] == np.float32(_frac_mean(kk[0, 0, :, c], 0, 250)), c
    # deq(K codes) stays within the E2M1 half-step bound of K - kmean on the
    # valid rows; a mean over all 300 rows would be off by ~1.7 everywhere
    s = O.e4m3_decode(qz["k_sf"][0, 0, :250]).astype(np.float64)           # [250, 4]
    dec = (O.e2m1_decode(qz["k"][0, 0, :250]).reshape(250, 4, 16) * s[..., None]).reshape(250, 64)
    want = kk[0, 0, :250] - qz["k_mean"][0, 0].astype(np.float64)
    y = np.abs(want) / np.repeat(np.where(s > 0, s, 1), 16, axis=-1)
    half = np.where(y < 2, 0.25, np.where(y < 4, 0.5, 1.0)) * np.repeat(s, 16, axis=-1)
    assert np.all(np.abs(dec - want) <= half * (1 + 1e-5) + 1e-6)


@pytest.mark.parametrize("per_block_mean", [True, False])
def test_nvfp4_q_codes_follow_their_own_block_mean(per_block_mean):
    """With block offsets +5 / -3 / +8, deq(Q codes) must equal Q minus the
    exact mean of the row's own block (or the global mean) within the E2M1
    half-step bound: a row smoothed by another block's mean is off by >= 3."""
    q, k, v = _qkv(N=300, D=64, Hq=2, Hkv=1, seed=23)
    q = _offset_blocks(q, [5.0, -3.0, 8.0])
    qz = O.quantize_qkv_nvfp4(q, k, v, per_block_mean=per_block_mean, unpadded_k_len=300)
    qq = q.double().numpy()
    for h in range(2):
        for i in (0, 127, 128, 255, 256, 299):
            blk = i // 128 if per_block_mean else None
            lo, hi = ((blk * 128, min(300, blk * 128 + 128)) if per_block_mean else (0, 300))
            mean = np.array([_frac_mean(qq[0, h, :, c], lo, hi) for c in range(64)])
            s = O.e4m3_decode(qz["q_sf"][0, h, i]).astype(np.float64)          # [4]
            dec = (O.e2m1_decode(qz["q"][0, h, i]).reshape(4, 16) * s[:, None]).ravel()
            want = qq[0, h, i] - mean
            y = np.abs(want) / np.repeat(np.where(s > 0, s, 1), 16)
            half = np.where(y < 2, 0.25, np.where(y < 4, 0.5, 1.0)) * np.repeat(s, 16)
            assert np.all(np.abs(dec - want) <= half * (1 + 1e-5) + 1e-6), (h, i)
