"""GPU quantisation stage vs the oracle: codes, scales, K means and V
scales bit-exact; q_dot_kmean within fp32 rounding."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from gpu_util import lib

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    return lib()


def _compare(gz, oz, hq_sel=None, hkv_sel=None):
    hq_sel = slice(None) if hq_sel is None else hq_sel
    hkv_sel = slice(None) if hkv_sel is None else hkv_sel
    c = lambda t: t.cpu().numpy()  # noqa: E731
    np.testing.assert_array_equal(c(gz.q)[:, hq_sel], oz["q"], err_msg="q codes")
    np.testing.assert_array_equal(c(gz.q_scale)[:, hq_sel], oz["q_scale"], err_msg="q scales")
    np.testing.assert_array_equal(c(gz.k_mean)[:, hkv_sel], oz["k_mean"], err_msg="k mean")
    np.testing.assert_array_equal(c(gz.k)[:, hkv_sel], oz["k"], err_msg="k codes")
    np.testing.assert_array_equal(c(gz.k_scale)[:, hkv_sel], oz["k_scale"], err_msg="k scales")
    np.testing.assert_array_equal(c(gz.v)[:, hkv_sel], np.swapaxes(oz["v_t"], -1, -2), err_msg="v codes")
    np.testing.assert_array_equal(c(gz.v_scale)[:, hkv_sel], oz["v_scale"], err_msg="v scales")
    if gz.q_dot_kmean is not None:
        g = c(gz.q_dot_kmean)[:, hq_sel].astype(np.float64)
        r = oz["q_dot_kmean"]
        np.testing.assert_allclose(g, r, rtol=1e-5, atol=1e-5 * (np.abs(r).max() + 1))


@pytest.mark.parametrize("w", [
    W.TINY,
    W.TINY.scaled(B=2, Hq=4, Hkv=2, N=300, D=128, seed=11),          # ragged tail, GQA
    W.TINY.scaled(B=1, Hq=2, Hkv=2, N=1000, D=64, seed=12, k_offset_std=9.0),
    W.VIDEO_DIT.scaled(N=2048, Hq=2, Hkv=2),                          # V outliers
], ids=lambda w: f"{w.B}x{w.Hq}x{w.Hkv}x{w.N}x{w.D}")
def test_quantize_bit_exact(S, w):
    q, k, v = W.make_qkv(w)
    oz = O.quantize_qkv_i8f8(q, k, v)
    gz = S.sage_quantize_qkv(q.cuda(), k.cuda(), v.cuda())
    _compare(gz, oz)


def test_quantize_fp16_nhd_and_no_smoothing(S):
    w = W.TINY.scaled(B=2, Hq=4, Hkv=2, N=384, D=128, seed=13)
    q, k, v = W.make_qkv(w, dtype=torch.float16)
    oz = O.quantize_qkv_i8f8(q, k, v, smooth_k=False)
    qn, kn, vn = (t.transpose(1, 2).contiguous().cuda() for t in (q, k, v))   # physical NHD
    gz = S.sage_quantize_qkv(qn, kn, vn, smooth_k=False, layout="NHD")
    _compare(gz, oz)


def test_quantize_constant_keys_give_zero_block(S):
    w = W.TINY.scaled(N=256, D=64, seed=14)
    q, k, v = W.make_qkv(w)
    k[:, :, :, :] = k[:, :, :1, :]              # every token equal: K - mean == 0
    oz = O.quantize_qkv_i8f8(q, k, v)
    assert np.all(oz["k_scale"] == 0)
    gz = S.sage_quantize_qkv(q.cuda(), k.cuda(), v.cuda())
    _compare(gz, oz)


@pytest.mark.parametrize("w", [W.LLM_MASK, W.CAUSAL_GQA, W.VIDEO_DIT], ids=lambda w: w.name)
def test_quantize_full_size_sampled_heads(S, w):
    """Full-size workload on the GPU; the oracle checks two KV heads (and
    their Q heads) of the last batch bit for bit."""
    q, k, v = W.make_qkv(w)
    gz = S.sage_quantize_qkv(q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    G = w.Hq // w.Hkv
    b = w.B - 1
    for g in (0, w.Hkv - 1):
        hq = list(range(g * G, (g + 1) * G))
        oz = O.quantize_qkv_i8f8(q[b:b + 1, hq], k[b:b + 1, g:g + 1], v[b:b + 1, g:g + 1])
        sub = lambda t: t[b:b + 1]  # noqa: E731
        gsub = S.QuantizedQKV(sub(gz.q), sub(gz.q_scale), sub(gz.k), sub(gz.k_scale),
                              sub(gz.k_mean), sub(gz.v), sub(gz.v_scale), sub(gz.q_dot_kmean),
                              1, w.Hq, w.Hkv, w.N, w.N, w.D)
        _compare(gsub, oz, hq_sel=hq, hkv_sel=[g])
