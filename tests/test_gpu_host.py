"""sage_attn_fwd_host: the whole path on Q/K/V held in host memory, streamed
through the GPU in chunks of (batch entry, KV head) groups.

Every group is a problem of its own, so the chunked result must equal the
one-shot device call (sage_attn_fwd) bit for bit, whatever the chunking,
layout or host-memory kind; and it must meet the parity bound against the
oracle."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from gpu_util import assert_attention_close, lib

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    return lib()


def _host(t, pinned=True):
    h = t.detach().cpu().contiguous()
    return h.pin_memory() if pinned else h


def _device_reference(S, q, k, v, causal, sm_scale, lse, mask=None, layout="HND"):
    res = S.sage_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, sm_scale=sm_scale,
                          return_lse=lse, mask=mask, layout=layout)
    torch.cuda.synchronize()
    return res if lse else (res, None)


CASES = [
    # (workload, causal, chunk_groups)
    (W.TINY.scaled(B=2, Hq=6, Hkv=3, N=300, D=128, seed=71), True, 2),    # ragged last chunk
    (W.TINY.scaled(B=1, Hq=8, Hkv=2, N=640, D=128, seed=72), False, 0),   # automatic: one chunk
    (W.TINY.scaled(B=3, Hq=4, Hkv=4, N=200, D=64, seed=73), True, 1),     # a chunk per head
    (W.TINY.scaled(B=2, Hq=8, Hkv=4, N=384, D=128, seed=70), True, 0),    # automatic: chunks 1, 3, 3, 1
]


@pytest.mark.parametrize("w,causal,chunk", CASES, ids=lambda c: str(c) if not hasattr(c, "N")
                         else f"{c.B}x{c.Hq}x{c.Hkv}x{c.N}x{c.D}")
def test_host_path_matches_oracle_and_device_call(S, w, causal, chunk):
    q, k, v = W.make_qkv(w)
    ref = O.attention_i8f8(O.quantize_qkv_i8f8(q, k, v), causal=causal, sm_scale=w.sm_scale)
    out, lse = S.sage_attn_fwd_host(_host(q), _host(k), _host(v), causal=causal,
                                    sm_scale=w.sm_scale, return_lse=True, chunk_groups=chunk)
    torch.cuda.synchronize()
    assert not out.is_cuda and out.shape == q.shape and out.dtype == q.dtype
    assert_attention_close(out, lse, ref, what=w.name)
    d_out, d_lse = _device_reference(S, q, k, v, causal, w.sm_scale, True)
    assert torch.equal(out, d_out.cpu())
    assert torch.equal(lse, d_lse.cpu())


@pytest.mark.parametrize("chunk", [1, 2, 3])
def test_host_path_nhd_fp16_every_chunking_is_bit_identical(S, chunk):
    w = W.TINY.scaled(B=2, Hq=8, Hkv=4, N=384, D=128, seed=74)
    q, k, v = W.make_qkv(w, dtype=torch.float16)
    qn, kn, vn = (t.transpose(1, 2).contiguous() for t in (q, k, v))      # [B, N, H, D]
    out, lse = S.sage_attn_fwd_host(_host(qn), _host(kn), _host(vn), causal=True,
                                    return_lse=True, layout="NHD", chunk_groups=chunk)
    torch.cuda.synchronize()
    d_out, d_lse = _device_reference(S, qn, kn, vn, True, None, True, layout="NHD")
    assert out.shape == qn.shape and out.dtype == torch.float16
    assert torch.equal(out, d_out.cpu())
    assert torch.equal(lse, d_lse.cpu())


def test_host_path_pageable_memory_and_strided_output(S):
    """Pageable (not page-locked) inputs, no LSE, and an output that is a
    head-sliced view of a larger host buffer (per-head strided copies)."""
    w = W.TINY.scaled(B=2, Hq=4, Hkv=2, N=256, D=64, seed=75)
    q, k, v = W.make_qkv(w)
    big = torch.zeros(2, 6, 256, 64, dtype=q.dtype)
    out = big[:, 1:5]                                                      # sh = N*D, sb = 6*N*D
    res = S.sage_attn_fwd_host(_host(q, False), _host(k, False), _host(v, False), causal=False,
                               out=out, chunk_groups=1)
    torch.cuda.synchronize()
    assert res.data_ptr() == out.data_ptr()
    d_out, _ = _device_reference(S, q, k, v, False, None, False)
    assert torch.equal(out, d_out.cpu())
    assert torch.all(big[:, 0] == 0) and torch.all(big[:, 5] == 0)        # nothing outside the view


@pytest.mark.parametrize("per_head", [False, True])
def test_host_path_with_device_mask(S, per_head):
    w = W.TINY.scaled(B=2, Hq=4, Hkv=2, N=256, D=128, seed=76)
    q, k, v = W.make_qkv(w)
    g = torch.Generator().manual_seed(76)
    mask = torch.rand(2, 4 if per_head else 1, 256, 256, generator=g) > 0.3
    mask[..., :1] = True
    md = mask.cuda()
    out, lse = S.sage_attn_fwd_host(_host(q), _host(k), _host(v), return_lse=True, mask=md,
                                    chunk_groups=1)
    torch.cuda.synchronize()
    d_out, d_lse = _device_reference(S, q, k, v, False, None, True, mask=md)
    assert torch.equal(out, d_out.cpu())
    assert torch.equal(lse, d_lse.cpu())
    ref = O.attention_i8f8(O.quantize_qkv_i8f8(q, k, v), mask=mask.numpy())
    assert_attention_close(out, lse, ref, what="host path, device mask")


def test_host_path_back_to_back_calls_share_streams(S):
    """Two calls in a row on one stream with different data: each result is
    its own (the second call waits for the first one's copies)."""
    w = W.TINY.scaled(B=1, Hq=4, Hkv=2, N=512, D=128, seed=77)
    q, k, v = W.make_qkv(w)
    q2 = q.flip(2).contiguous()
    o1 = S.sage_attn_fwd_host(_host(q), _host(k), _host(v), chunk_groups=1)
    o2 = S.sage_attn_fwd_host(_host(q2), _host(k), _host(v), chunk_groups=1)
    torch.cuda.synchronize()
    d1, _ = _device_reference(S, q, k, v, False, None, False)
    d2, _ = _device_reference(S, q2, k, v, False, None, False)
    assert torch.equal(o1, d1.cpu()) and torch.equal(o2, d2.cpu())
    st, site = S.sage_get_device_status()
    assert st == S.SAGE_OK, site


NV_CASES = [
    # (workload, per_block_mean, causal, chunk_groups, layout)
    (W.NVFP4.scaled(B=2, Hq=4, Hkv=2, N=300, D=128, unpadded_k_len=260, seed=81), True, False, 1, "HND"),
    (W.NVFP4.scaled(B=1, Hq=6, Hkv=3, N=384, D=64, unpadded_k_len=384, seed=82), False, True, 2, "NHD"),
    (W.NVFP4.scaled(B=1, Hq=2, Hkv=2, N=256, D=128, unpadded_k_len=200, seed=83), True, True, 0, "HND"),
    (W.NVFP4.scaled(B=2, Hq=6, Hkv=3, N=256, D=128, unpadded_k_len=250, seed=84), True, False, 0, "NHD"),
]


@pytest.mark.parametrize("w,pbm,causal,chunk,layout", NV_CASES,
                         ids=lambda c: str(c) if not hasattr(c, "N") else f"{c.B}x{c.Hq}x{c.Hkv}x{c.N}x{c.D}")
def test_nvfp4_host_path_equals_device_calls(S, w, pbm, causal, chunk, layout):
    """sage_attn_fwd_nvfp4_host gives the bits of sage_quantize_qkv_nvfp4 +
    sage_attn_fwd_nvfp4 on the device, for every chunking and layout."""
    q, k, v = W.make_qkv(w)
    if layout == "NHD":
        q, k, v = (t.transpose(1, 2).contiguous() for t in (q, k, v))
    z = S.sage_quantize_qkv_nvfp4(q.cuda(), k.cuda(), v.cuda(), per_block_mean=pbm,
                                  unpadded_k_len=w.unpadded_k_len, layout=layout)
    d_out, d_lse = S.sage_attn_fwd_nvfp4(z, sm_scale=w.sm_scale, causal=causal, return_lse=True,
                                         out_dtype=q.dtype)
    torch.cuda.synchronize()
    out, lse = S.sage_attn_fwd_nvfp4_host(_host(q), _host(k), _host(v), sm_scale=w.sm_scale,
                                          causal=causal, per_block_mean=pbm,
                                          unpadded_k_len=w.unpadded_k_len, return_lse=True,
                                          layout=layout, chunk_groups=chunk)
    torch.cuda.synchronize()
    d_out = d_out.cpu() if layout == "HND" else d_out.transpose(1, 2).cpu()
    assert out.shape == q.shape and out.dtype == q.dtype
    assert torch.equal(out, d_out)
    assert torch.equal(lse, d_lse.cpu())
    st, site = S.sage_get_device_status()
    assert st == S.SAGE_OK, site
