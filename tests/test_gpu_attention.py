"""Fused INT8-QK / FP8-PV attention on the GPU vs the oracle.

Two entry points: sage_attn_fwd_quantized on the ORACLE's codes (isolates
the attention kernel) and sage_attn_fwd on bf16/fp16 inputs (the whole
path).  Bound: max |out - oracle| <= 2e-2 and cosine >= 0.9995, same for the
LSE; -inf LSE entries (rows with no visible key) must match exactly."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from gpu_util import assert_attention_close, lib, qkv_from_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    return lib()


CASES = [
    # (workload, causal, return_lse)
    (W.TINY, False, True),
    (W.TINY, True, True),
    (W.TINY.scaled(B=2, Hq=4, Hkv=2, N=300, D=128, seed=31), False, True),     # ragged, GQA
    (W.TINY.scaled(B=1, Hq=8, Hkv=2, N=640, D=128, seed=32), True, True),      # odd tile count
    (W.TINY.scaled(B=1, Hq=2, Hkv=1, N=1000, D=64, seed=33), True, False),
    (W.VIDEO_DIT.scaled(N=1024, Hq=2, Hkv=2), False, True),                    # V outliers
]


@pytest.mark.parametrize("w,causal,lse", CASES,
                         ids=lambda c: str(c) if not hasattr(c, "N") else f"{c.B}x{c.Hq}x{c.Hkv}x{c.N}x{c.D}")
def test_attention_on_oracle_codes(S, w, causal, lse):
    q, k, v = W.make_qkv(w)
    oz = O.quantize_qkv_i8f8(q, k, v)
    ref = O.attention_i8f8(oz, causal=causal, sm_scale=w.sm_scale)
    z = qkv_from_oracle(S, oz)
    res = S.sage_attn_fwd_quantized(z, causal=causal, sm_scale=w.sm_scale, return_lse=lse)
    out, l = res if lse else (res, None)
    assert_attention_close(out, l, ref, what=w.name)


@pytest.mark.parametrize("w,causal,lse", CASES[:4],
                         ids=lambda c: str(c) if not hasattr(c, "N") else f"{c.B}x{c.Hq}x{c.Hkv}x{c.N}x{c.D}")
def test_fused_path(S, w, causal, lse):
    q, k, v = W.make_qkv(w)
    ref = O.attention_i8f8(O.quantize_qkv_i8f8(q, k, v), causal=causal, sm_scale=w.sm_scale)
    res = S.sage_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, sm_scale=w.sm_scale,
                          return_lse=lse)
    out, l = res if lse else (res, None)
    assert out.shape == q.shape and out.dtype == q.dtype
    assert_attention_close(out, l, ref, what=w.name)


def test_fused_fp16_nhd(S):
    w = W.TINY.scaled(B=2, Hq=4, Hkv=2, N=256, D=128, seed=34)
    q, k, v = W.make_qkv(w, dtype=torch.float16)
    ref = O.attention_i8f8(O.quantize_qkv_i8f8(q, k, v), causal=True)
    qn, kn, vn = (t.transpose(1, 2).contiguous().cuda() for t in (q, k, v))
    out, l = S.sage_attn_fwd(qn, kn, vn, causal=True, return_lse=True, layout="NHD")
    assert out.shape == qn.shape and out.dtype == torch.float16
    assert_attention_close(out.transpose(1, 2), l, ref, what="fp16 NHD")


def test_mask_second_half_and_random_mask(S):
    w = W.TINY.scaled(B=2, Hq=4, Hkv=4, N=512, D=128, seed=35, mask="second_half_keys")
    q, k, v = W.make_qkv(w)
    oz = O.quantize_qkv_i8f8(q, k, v)
    z = qkv_from_oracle(S, oz)
    mask = W.make_mask(w)
    ref = O.attention_i8f8(oz, mask=mask.numpy())
    out, l = S.sage_attn_fwd_quantized(z, return_lse=True, mask=mask.cuda())
    assert_attention_close(out, l, ref, what="second half masked")
    g = torch.Generator().manual_seed(3)
    rm = torch.rand(2, 1, 512, 512, generator=g) < 0.5
    rm[:, :, 7, :] = False                         # a row with no visible key
    rm[:, :, :, 256:384] = True                    # a fully visible key tile
    rm[:, :, :, 384:] = False                      # a fully hidden key tile
    ref = O.attention_i8f8(oz, mask=rm.numpy(), causal=True)
    out, l = S.sage_attn_fwd_quantized(z, return_lse=True, mask=rm.cuda(), causal=True)
    assert_attention_close(out, l, ref, what="random mask + causal")
    assert torch.all(out[:, :, 7] == 0) and torch.all(torch.isneginf(l[:, :, 7]))


def test_mask_hides_every_key_from_one_q_tile_of_a_pair(S):
    """A CTA works on a pair of 128-row Q tiles, and the second tile's
    softmax starts after the first tile's first P tile.  With the first tile
    (or the second) seeing no key at all, nothing may wait for it: rows 0..127
    (then 128..255) are fully masked, the other tile of the pair sees a random
    half of the keys."""
    w = W.TINY.scaled(B=1, Hq=2, Hkv=2, N=512, D=128, seed=37)
    q, k, v = W.make_qkv(w)
    oz = O.quantize_qkv_i8f8(q, k, v)
    z = qkv_from_oracle(S, oz)
    g = torch.Generator().manual_seed(5)
    for hidden in (slice(0, 128), slice(128, 256)):
        rm = torch.rand(1, 1, 512, 512, generator=g) < 0.5
        rm[:, :, hidden, :] = False
        ref = O.attention_i8f8(oz, mask=rm.numpy())
        out, l = S.sage_attn_fwd_quantized(z, return_lse=True, mask=rm.cuda())
        assert S.sage_get_device_status()[0] == S.SAGE_OK
        assert_attention_close(out, l, ref, what=f"rows {hidden.start}.. hidden")
        assert torch.all(out[:, :, hidden] == 0) and torch.all(torch.isneginf(l[:, :, hidden]))


def test_mask_unaligned_key_length(S):
    w = W.TINY.scaled(B=1, Hq=2, Hkv=2, N=200, D=64, seed=36)
    q, k, v = W.make_qkv(w)
    oz = O.quantize_qkv_i8f8(q, k, v)
    g = torch.Generator().manual_seed(4)
    rm = torch.rand(1, 2, 200, 200, generator=g) < 0.6
    ref = O.attention_i8f8(oz, mask=rm.numpy())
    out, l = S.sage_attn_fwd_quantized(qkv_from_oracle(S, oz), return_lse=True, mask=rm.cuda())
    assert_attention_close(out, l, ref, what="per-head mask, Nk=200")


@pytest.mark.parametrize("causal", [False, True])
def test_float_mask(S, causal):
    """Float additive mask ("sageattn_qk_int8_pv_fp16_triton": boolean or
    float32 attention mask): random biases, -inf regions (a hidden key
    tile, a row that sees nothing), an all-zero tile, broadcast over heads."""
    w = W.TINY.scaled(B=2, Hq=4, Hkv=2, N=512, D=128, seed=37)
    q, k, v = W.make_qkv(w)
    oz = O.quantize_qkv_i8f8(q, k, v)
    g = torch.Generator().manual_seed(5)
    bias = 2.0 * torch.randn(2, 1, 512, 512, generator=g)
    bias[:, :, :, 384:] = float("-inf")           # a fully hidden key tile
    bias[:, :, :, 128:256] = 0.0                   # a tile without bias
    bias[:, :, 9, :] = float("-inf")               # a row with no visible key
    bias[:, :, :, 40:60] = float("-inf")
    ref = O.attention_i8f8(oz, bias=bias.double().numpy(), causal=causal)
    out, l = S.sage_attn_fwd_quantized(qkv_from_oracle(S, oz), return_lse=True, mask=bias.cuda(),
                                       causal=causal)
    assert_attention_close(out, l, ref, what=f"float mask causal={causal}")
    assert torch.all(out[:, :, 9] == 0) and torch.all(torch.isneginf(l[:, :, 9]))


def test_float_mask_unaligned_rows_and_zero_bias(S):
    """A per-head bias whose rows are not 16-byte aligned (scalar loads) on
    a ragged key length; and an all-zero bias equals no mask bit for bit."""
    w = W.TINY.scaled(B=1, Hq=2, Hkv=2, N=203, D=64, seed=38)
    q, k, v = W.make_qkv(w)
    oz = O.quantize_qkv_i8f8(q, k, v)
    z = qkv_from_oracle(S, oz)
    g = torch.Generator().manual_seed(6)
    bias = torch.randn(1, 2, 203, 203, generator=g)
    ref = O.attention_i8f8(oz, bias=bias.double().numpy())
    out, l = S.sage_attn_fwd_quantized(z, return_lse=True, mask=bias.cuda())
    assert_attention_close(out, l, ref, what="float mask, unaligned rows")
    plain, pl = S.sage_attn_fwd_quantized(z, return_lse=True)
    zero, zl = S.sage_attn_fwd_quantized(z, return_lse=True, mask=torch.zeros(1, 1, 203, 203).cuda())
    torch.cuda.synchronize()
    assert torch.equal(plain, zero) and torch.equal(pl, zl)


def test_causal_bottom_right_when_lengths_differ(S):
    for Nq, Nk in [(200, 333), (333, 200)]:
        wq = W.TINY.scaled(B=1, Hq=2, Hkv=1, N=Nq, D=128, seed=37)
        wk = W.TINY.scaled(B=1, Hq=2, Hkv=1, N=Nk, D=128, seed=38)
        q = W.make_qkv(wq)[0]
        _, k, v = W.make_qkv(wk)
        oz = O.quantize_qkv_i8f8(q, k, v)
        ref = O.attention_i8f8(oz, causal=True)
        out, l = S.sage_attn_fwd_quantized(qkv_from_oracle(S, oz), causal=True, return_lse=True)
        assert_attention_close(out, l, ref, what=f"causal Nq={Nq} Nk={Nk}")


def test_longest_supported_key_length(S):
    """The longest key sequence the kernels accept: 2048 key tiles (262144
    keys), the most the per-CTA list of visible key tiles holds in shared
    memory.  256 queries, non-causal and causal (bottom-right aligned),
    through the whole path (the quantiser included) against the oracle."""
    wq = W.TINY.scaled(B=1, Hq=2, Hkv=1, N=256, D=128, seed=41)
    wk = W.TINY.scaled(B=1, Hq=2, Hkv=1, N=128 * 2048, D=128, seed=42)
    q = W.make_qkv(wq)[0]
    _, k, v = W.make_qkv(wk)
    oz = O.quantize_qkv_i8f8(q, k, v)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    for causal in (False, True):
        ref = O.attention_i8f8(oz, causal=causal, sm_scale=wq.sm_scale)
        out, l = S.sage_attn_fwd(qd, kd, vd, causal=causal, sm_scale=wq.sm_scale, return_lse=True)
        assert_attention_close(out, l, ref, what=f"Nk=262144 causal={causal}")


def test_single_tokens_and_decode_shape(S):
    """One query and one key per head (a tile with one live row and one
    live key), causal and not; then one query against 300 keys, causal
    (bottom-right aligned, so the query sees every key: the decode shape)."""
    w = W.TINY.scaled(B=2, Hq=4, Hkv=2, N=1, D=128, seed=46)
    q, k, v = W.make_qkv(w)
    oz = O.quantize_qkv_i8f8(q, k, v)
    for causal in (False, True):
        ref = O.attention_i8f8(oz, causal=causal, sm_scale=w.sm_scale)
        out, l = S.sage_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, sm_scale=w.sm_scale,
                                 return_lse=True)
        assert_attention_close(out, l, ref, what=f"N=1 causal={causal}")
    _, k, v = W.make_qkv(W.TINY.scaled(B=2, Hq=4, Hkv=2, N=300, D=128, seed=47))
    ref = O.attention_i8f8(O.quantize_qkv_i8f8(q, k, v), causal=True, sm_scale=w.sm_scale)
    out, l = S.sage_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True, sm_scale=w.sm_scale,
                             return_lse=True)
    assert_attention_close(out, l, ref, what="Nq=1 Nk=300 causal")


def test_most_query_heads_one_call_takes(S):
    """B * Hq = 17 * 3855 = 65535, the most (batch entry, Q head) pairs one
    call takes (at most 4096 heads per entry), one token each and every Q
    head on its entry's one KV head.  Heads are independent given the shared
    K and V, so the oracle runs on a sample of them (first, last and 61
    random)."""
    w = W.TINY.scaled(B=17, Hq=3855, Hkv=1, N=1, D=64, seed=45)
    q, k, v = W.make_qkv(w)
    out, l = S.sage_attn_fwd(q.cuda(), k.cuda(), v.cuda(), sm_scale=w.sm_scale, return_lse=True)
    rng = np.random.default_rng(45)
    idx = torch.from_numpy(np.unique(np.concatenate([[0, 1, w.Hq - 1],
                                                     rng.choice(w.Hq, 61, replace=False)])))
    ref = O.attention_i8f8(O.quantize_qkv_i8f8(q[:, idx], k, v), sm_scale=w.sm_scale)
    assert_attention_close(out[:, idx.cuda()], l[:, idx.cuda()], ref, what="B*Hq=65535")


def test_calls_without_queries_return_empty_results(S):
    """No queries (Nq == 0 or B == 0): empty out and LSE from every
    whole-path call, nothing launched, the device status untouched."""
    g = torch.Generator().manual_seed(39)
    k = torch.randn(1, 2, 256, 128, generator=g).to(torch.bfloat16)
    v = torch.randn(1, 2, 256, 128, generator=g).to(torch.bfloat16)
    q = torch.empty(1, 4, 0, 128, dtype=torch.bfloat16)
    out, lse = S.sage_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True, return_lse=True)
    assert out.shape == (1, 4, 0, 128) and lse.shape == (1, 4, 0)
    out, lse = S.sage_attn_fwd_host(q, k, v, causal=True, return_lse=True)
    assert out.shape == (1, 4, 0, 128) and lse.shape == (1, 4, 0)
    out, lse = S.sage_attn_fwd_nvfp4_host(q, k, v, return_lse=True)
    assert out.shape == (1, 4, 0, 128) and lse.shape == (1, 4, 0)
    q0, k0 = torch.empty(0, 4, 256, 128, dtype=torch.bfloat16), torch.empty(0, 2, 256, 128, dtype=torch.bfloat16)
    out = S.sage_attn_fwd(q0.cuda(), k0.cuda(), k0.cuda())
    assert out.shape == q0.shape
    torch.cuda.synchronize()
    st, site = S.sage_get_device_status()
    assert st == S.SAGE_OK, site


def test_lossless_case_matches_exact_attention(S):
    """On the oracle's lossless inputs the GPU must also land on exact
    attention (up to its fp32 exp2 and bf16 output rounding)."""
    from lossless_cases import LN2, i8f8_case
    q, k, v = i8f8_case(B=1, Hq=2, Hkv=1, N=384, D=64, seed=3)
    ex, lse = O.exact_attention(q, k, v, causal=True, sm_scale=LN2)
    out, l = S.sage_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True, sm_scale=LN2, return_lse=True)
    # outputs here reach 448 (V holds +-448), so the bound is bf16-relative:
    # half a bf16 ulp (2**-8 relative) plus the fp32 exp2 error
    np.testing.assert_allclose(out.float().cpu().numpy(), ex, rtol=2.0 ** -8 + 1e-4, atol=1e-3)
    np.testing.assert_allclose(l.cpu().numpy(), lse, atol=1e-4)


@pytest.mark.parametrize("w", [W.LLM_MASK, W.CAUSAL_GQA, W.VIDEO_DIT], ids=lambda w: w.name)
def test_full_size_sampled(S, w):
    """The full workload through sage_attn_fwd (the call bench.py times);
    the oracle checks the sampled rows of the Q heads of two KV heads."""
    q, k, v = W.make_qkv(w)
    mask = W.make_mask(w)
    res = S.sage_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=w.causal, sm_scale=w.sm_scale,
                          return_lse=True, mask=None if mask is None else mask.cuda())
    out, l = res
    torch.cuda.synchronize()
    rows = W.sample_rows(w)
    G = w.Hq // w.Hkv
    b = w.B - 1
    for g in (0, w.Hkv - 1):
        hq = list(range(g * G, (g + 1) * G))
        oz = O.quantize_qkv_i8f8(q[b:b + 1, hq], k[b:b + 1, g:g + 1], v[b:b + 1, g:g + 1])
        m = None if mask is None else mask[b:b + 1].numpy()
        ref = O.attention_i8f8(oz, causal=w.causal, sm_scale=w.sm_scale, mask=m, rows=rows)
        assert_attention_close(out[b:b + 1, hq], l[b:b + 1, hq], ref, rows=rows, what=w.name)
