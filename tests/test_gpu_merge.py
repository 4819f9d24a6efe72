"""The LSE merge kernel on the GPU (thu-ml/sageattention llms.txt, "Utilize
SageAttention for Distributed Inference"): attention over key shards, each
through the CUDA path with return_lse, merged by sage_lse_merge, against
the oracle merge of the oracle's per-shard results."""
import os
import socket

import numpy as np
import pytest
import torch

import oracle as O
from oracle.merge import merge_partials
import workloads as W
from gpu_util import MAX_ABS, MIN_COS, lib

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    return lib()


def _shard_mask(N, a, b, causal):
    m = np.zeros((N, N), bool)
    m[:, a:b] = True
    if causal:
        m &= np.tril(np.ones((N, N), bool))
    return m


@pytest.mark.parametrize("causal", [False, True])
def test_merge_of_key_shards_matches_oracle(S, causal):
    w = W.CAUSAL_GQA.scaled(B=1, Hq=4, Hkv=2, N=640, D=128, seed=61)
    q, k, v = W.make_qkv(w)
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    edges = [0, 128, 384, 640]                    # three shards of different lengths
    acc = torch.zeros(1, 4, 640, 128, dtype=torch.float32, device="cuda")
    acc_lse = torch.full((1, 4, 640), float("-inf"), device="cuda")
    parts = []
    for i in range(3):
        a, b = edges[i], edges[i + 1]
        mask = torch.from_numpy(_shard_mask(640, a, b, causal)).cuda()
        out, lse = S.sage_attn_fwd(dq, dk, dv, return_lse=True, mask=mask)
        S.sage_lse_merge(acc, acc_lse, out, lse, init=(i == 0))
        z = O.quantize_qkv_i8f8(q, k, v)
        r = O.attention_i8f8(z, mask=_shard_mask(640, a, b, causal)[None, None])
        parts.append((r["out_f64"], r["lse"]))
    out = S.sage_lse_merge_finalize(acc, torch.empty(1, 4, 640, 128, dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()
    ref_o, ref_l = merge_partials(parts)
    o = out.float().cpu().numpy().astype(np.float64)
    assert np.abs(o - ref_o).max() <= MAX_ABS
    assert O.cosine(o, ref_o) >= MIN_COS
    lg = acc_lse.cpu().numpy().astype(np.float64)
    assert np.array_equal(np.isfinite(lg), np.isfinite(ref_l))
    fin = np.isfinite(ref_l)
    assert np.abs(lg[fin] - ref_l[fin]).max() <= MAX_ABS
    # and the merge is the attention over all keys
    full, _ = O.exact_attention(q, k, v, causal=causal)
    assert O.cosine(o, full) >= 0.999


def test_merge_kernel_arithmetic(S):
    """Direct check of the combination rule with -inf rows, fp16 parts in an
    NHD layout, d=64."""
    g = torch.Generator().manual_seed(62)
    B, H, N, D = 2, 3, 50, 64
    o1 = torch.randn(B, N, H, D, generator=g).to(torch.float16).transpose(1, 2)   # NHD view
    o2 = torch.randn(B, N, H, D, generator=g).to(torch.float16).transpose(1, 2)
    l1 = torch.randn(B, H, N, generator=g)
    l2 = torch.randn(B, H, N, generator=g)
    l1[0, 0, :5] = float("-inf")
    l2[0, 0, 3:8] = float("-inf")                     # rows 3, 4: no key in either
    acc = torch.empty(B, H, N, D, device="cuda")
    acc_lse = torch.empty(B, H, N, device="cuda")
    S.sage_lse_merge(acc, acc_lse, o1.cuda(), l1.cuda(), init=True)
    S.sage_lse_merge(acc, acc_lse, o2.cuda(), l2.cuda())
    out = S.sage_lse_merge_finalize(acc, torch.empty(B, H, N, D, dtype=torch.float16, device="cuda"))
    torch.cuda.synchronize()
    ref_o, ref_l = merge_partials([(o1.double().numpy(), l1.double().numpy()),
                                   (o2.double().numpy(), l2.double().numpy())])
    np.testing.assert_allclose(acc.cpu().numpy(), ref_o, rtol=0, atol=2e-6)
    np.testing.assert_allclose(out.float().cpu().numpy(), ref_o, rtol=2.0 ** -10, atol=1e-6)
    lg = acc_lse.cpu().numpy()
    assert np.array_equal(np.isneginf(lg), np.isneginf(ref_l))
    fin = np.isfinite(ref_l)
    np.testing.assert_allclose(lg[fin], ref_l[fin], rtol=0, atol=2e-6)
    assert np.all(acc.cpu().numpy()[0, 0, 3:5] == 0)


def test_ring_attention_single_rank_equals_one_call(S):
    """ring_attention on a one-rank NCCL group is one attention call and an
    exact fp32 round trip of its output."""
    import torch.distributed as dist
    from quantized_attention_05_b200.ring import ring_attention
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        w = W.CAUSAL_GQA.scaled(B=1, Hq=4, Hkv=2, N=512, D=128, seed=63)
        q, k, v = W.make_qkv(w, device="cuda")
        out, lse = ring_attention(q, k, v, causal=True)
        ref, ref_lse = S.sage_attn_fwd(q, k, v, causal=True, return_lse=True)
        torch.cuda.synchronize()
        assert torch.equal(out, ref) and torch.equal(lse, ref_lse)
    finally:
        dist.destroy_process_group()
