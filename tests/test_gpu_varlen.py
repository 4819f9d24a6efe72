"""Variable-length (packed) attention on the GPU against the varlen oracle
(thu-ml/sageattention llms.txt, "sageattn_varlen"): every packed sequence is
its own dense problem."""
import numpy as np
import pytest
import torch

import oracle as O
from oracle.varlen import attention_varlen_i8f8
import workloads as W
from gpu_util import lib

pytestmark = pytest.mark.gpu
MAX_ABS = 2e-2
MIN_COS = 0.9995


@pytest.fixture(scope="module")
def S():
    return lib()


def _packed_case(lens_q, lens_k, Hq, Hkv, D, seed, dtype=torch.bfloat16):
    """Packed q [sum lens_q, Hq, D], k/v [sum lens_k, Hkv, D] drawn like the
    dense workloads (N(0,1), per-sequence K channel offsets of std 2)."""
    g = torch.Generator().manual_seed(seed)
    tq, tk = sum(lens_q), sum(lens_k)
    q = torch.randn(tq, Hq, D, generator=g)
    k = torch.randn(tk, Hkv, D, generator=g)
    v = torch.randn(tk, Hkv, D, generator=g)
    c = 0
    for n in lens_k:                                  # channel outliers, per sequence
        k[c:c + n] += 2.0 * torch.randn(1, Hkv, D, generator=g)
        c += n
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    return q.to(dtype), k.to(dtype), v.to(dtype), cu_q, cu_k


def _run(S, q, k, v, cu_q, cu_k, causal, return_lse=True, sm_scale=None):
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    cq, ck = torch.from_numpy(cu_q).cuda(), torch.from_numpy(cu_k).cuda()
    lq, lk = np.diff(cu_q), np.diff(cu_k)
    r = S.sage_attn_fwd_varlen(dq, dk, dv, cq, ck, int(lq.max()), int(lk.max()), causal=causal,
                               sm_scale=sm_scale, return_lse=return_lse)
    torch.cuda.synchronize()
    assert S.sage_get_device_status()[0] == S.SAGE_OK
    return r


def _compare(out, lse, ref):
    o = out.float().cpu().numpy().astype(np.float64)
    r = ref["out"]
    assert np.abs(o - r).max() <= MAX_ABS, np.abs(o - r).max()
    assert O.cosine(o, r) >= MIN_COS
    if lse is not None:
        lg, lr = lse.cpu().numpy().astype(np.float64), ref["lse"]
        fin = np.isfinite(lr)
        assert np.array_equal(np.isfinite(lg), fin)
        assert np.abs(lg[fin] - lr[fin]).max() <= MAX_ABS


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_pages_example_shape(S, causal):
    """The pages' example: lengths [512, 1024, 768], 16 heads, d=128, fp16."""
    lens = [512, 1024, 768]
    q, k, v, cu_q, cu_k = _packed_case(lens, lens, 16, 16, 128, seed=31, dtype=torch.float16)
    out, lse = _run(S, q, k, v, cu_q, cu_k, causal)
    ref = attention_varlen_i8f8(q, k, v, cu_q, cu_k, causal=causal)
    _compare(out, lse, ref)


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_ragged_gqa_empty_d64(S, causal):
    """Lengths off the 128 grid, a 1-token and a 3-token sequence, an empty
    one, Nq != Nk per sequence (bottom-right causal), GQA, d=64."""
    lens_q = [300, 1, 0, 129, 3, 640]
    lens_k = [300, 5, 0, 257, 3, 512]
    q, k, v, cu_q, cu_k = _packed_case(lens_q, lens_k, 4, 2, 64, seed=32)
    out, lse = _run(S, q, k, v, cu_q, cu_k, causal)
    ref = attention_varlen_i8f8(q, k, v, cu_q, cu_k, causal=causal)
    _compare(out, lse, ref)


def test_varlen_single_sequence_equals_dense_call(S):
    """One packed sequence runs the same kernels on the same codes as the
    dense call: identical outputs, bit for bit."""
    w = W.CAUSAL_GQA.scaled(B=1, Hq=8, Hkv=2, N=1000, D=128, seed=33)
    q, k, v = W.make_qkv(w, device="cuda")
    out_d, lse_d = S.sage_attn_fwd(q, k, v, causal=True, return_lse=True)
    pq, pk, pv = (t[0].transpose(0, 1).contiguous() for t in (q, k, v))
    cu = torch.tensor([0, 1000], dtype=torch.int32, device="cuda")
    out_v, lse_v = S.sage_attn_fwd_varlen(pq, pk, pv, cu, cu, 1000, 1000, causal=True,
                                          return_lse=True)
    torch.cuda.synchronize()
    assert torch.equal(out_v, out_d[0].transpose(0, 1))
    assert torch.equal(lse_v, lse_d[0].reshape(-1))


def test_varlen_sequences_do_not_interact(S):
    lens = [200, 333, 128]
    q, k, v, cu_q, cu_k = _packed_case(lens, lens, 2, 2, 128, seed=34)
    a = _run(S, q, k, v, cu_q, cu_k, causal=False, return_lse=False)
    k2, v2 = k.clone(), v.clone()
    k2[200:533] *= 4                                   # the middle sequence only
    v2[200:533] -= 3
    b = _run(S, q, k2, v2, cu_q, cu_k, causal=False, return_lse=False)
    assert torch.equal(a[:200], b[:200]) and torch.equal(a[533:], b[533:])
    assert not torch.equal(a[200:533], b[200:533])


def test_varlen_out_of_range_cu_seqlens_stay_in_bounds(S):
    """cu_seqlens beyond the packed length or max_seqlen are clamped on the
    device: the call completes without a fault and valid sequences are
    unaffected."""
    lens = [256, 256]
    q, k, v, cu_q, cu_k = _packed_case(lens, lens, 2, 2, 64, seed=35)
    good = _run(S, q, k, v, cu_q, cu_k, causal=False, return_lse=False)
    bad = np.array([0, 256, 100000], dtype=np.int32)    # second sequence runs off the end
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    cb = torch.from_numpy(bad).cuda()
    out = S.sage_attn_fwd_varlen(dq, dk, dv, cb, cb, 256, 256)
    torch.cuda.synchronize()
    assert S.sage_get_device_status()[0] == S.SAGE_OK
    assert torch.equal(out[:256], good[:256])
