"""NVFP4 path on the GPU vs the oracle: quantiser codes, scale factors and
means bit-exact (qk_correction and q.kmean within fp32 tolerance), the
block-scaled FP4 attention within the parity bound, and the lossless NVFP4
case against exact attention."""
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


def nvfp4_from_oracle(S, oz, device="cuda"):
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(dt).to(device)  # noqa: E731
    return S.QuantizedNvfp4(
        q=t(oz["q_packed"], torch.uint8), q_sf=t(oz["q_sf"], torch.uint8),
        k=t(oz["k_packed"], torch.uint8), k_sf=t(oz["k_sf"], torch.uint8),
        v_t=t(oz["v_t_packed"], torch.uint8), v_sf_t=t(oz["v_sf_t"], torch.uint8),
        qk_correction=t(oz["qk_correction"], torch.float32), q_mean=t(oz["q_mean"], torch.float32),
        k_mean=t(oz["k_mean"], torch.float32),
        q_dot_kmean=t(oz["q_dot_kmean"].astype(np.float32), torch.float32),
        B=oz["B"], Hq=oz["Hq"], Hkv=oz["Hkv"], Nq=oz["Nq"], Nk=oz["Nk"], D=oz["D"],
        unpadded_k_len=oz["unpadded_k_len"], per_block_mean=oz["per_block_mean"])


def _compare_quant(gz, oz, hq=None, hkv=None):
    hq = slice(None) if hq is None else hq
    hkv = slice(None) if hkv is None else hkv
    c = lambda t: t.cpu().numpy()  # noqa: E731
    for g, o, sel, name in [(gz.q, oz["q_packed"], hq, "q codes"), (gz.q_sf, oz["q_sf"], hq, "q sf"),
                            (gz.q_mean, oz["q_mean"], hq, "q mean"),
                            (gz.k, oz["k_packed"], hkv, "k codes"), (gz.k_sf, oz["k_sf"], hkv, "k sf"),
                            (gz.k_mean, oz["k_mean"], hkv, "k mean"),
                            (gz.v_t, oz["v_t_packed"], hkv, "v codes"),
                            (gz.v_sf_t, oz["v_sf_t"], hkv, "v sf")]:
        np.testing.assert_array_equal(c(g)[:, sel], o, err_msg=name)
    corr, ocorr = c(gz.qk_correction)[:, hq].astype(np.float64), oz["qk_correction"].astype(np.float64)
    np.testing.assert_allclose(corr, ocorr, rtol=0, atol=1e-3 * np.abs(ocorr).max() + 1e-6)
    qdk = c(gz.q_dot_kmean)[:, hq].astype(np.float64)
    np.testing.assert_allclose(qdk, oz["q_dot_kmean"], rtol=1e-5, atol=1e-5 * (np.abs(qdk).max() + 1))


QCASES = [
    (W.NVFP4.scaled(B=1, Hq=2, Hkv=2, N=256, D=128, unpadded_k_len=200), True),
    (W.NVFP4.scaled(B=2, Hq=4, Hkv=2, N=300, D=128, unpadded_k_len=300, seed=7), True),
    (W.NVFP4.scaled(B=1, Hq=2, Hkv=1, N=384, D=64, unpadded_k_len=320, seed=8), False),
    (W.TINY.scaled(N=512, D=128, seed=9, nvfp4=True), True),      # with K channel offsets
]


@pytest.mark.parametrize("w,pbm", QCASES, ids=lambda c: str(c) if not hasattr(c, "N") else f"{c.B}x{c.Hq}x{c.Hkv}x{c.N}x{c.D}")
def test_nvfp4_quantize_bit_exact(S, w, pbm):
    q, k, v = W.make_qkv(w)
    L = w.unpadded_k_len or w.N
    oz = O.quantize_qkv_nvfp4(q, k, v, per_block_mean=pbm, unpadded_k_len=L)
    gz = S.sage_quantize_qkv_nvfp4(q.cuda(), k.cuda(), v.cuda(), per_block_mean=pbm, unpadded_k_len=L)
    torch.cuda.synchronize()
    _compare_quant(gz, oz)


@pytest.mark.parametrize("per_block_mean,L,causal", [(True, 256, False), (False, 224, False),
                                                     (True, 192, True)])
def test_nvfp4_attention_lossless_equals_exact(S, per_block_mean, L, causal):
    from lossless_cases import LN2, nvfp4_case
    q, k, v = nvfp4_case(B=1, Hq=2, Hkv=1, N=256, D=64, L=L, seed=L)
    oz = O.quantize_qkv_nvfp4(q, k, v, per_block_mean=per_block_mean, unpadded_k_len=L)
    z = nvfp4_from_oracle(S, oz)
    out, lse = S.sage_attn_fwd_nvfp4(z, sm_scale=LN2, causal=causal)
    ex, else_ = O.exact_attention(q, k, v, causal=causal, sm_scale=LN2, kv_len=L)
    np.testing.assert_allclose(out.float().cpu().numpy(), ex, rtol=2.0 ** -8 + 1e-4, atol=1e-3)
    np.testing.assert_allclose(lse.cpu().numpy(), else_, atol=1e-4)


ACASES = [
    (W.NVFP4.scaled(B=1, Hq=2, Hkv=2, N=256, D=128, unpadded_k_len=200), False),
    (W.NVFP4.scaled(B=1, Hq=4, Hkv=2, N=640, D=128, unpadded_k_len=600, seed=5), True),
    (W.NVFP4.scaled(B=2, Hq=2, Hkv=2, N=300, D=64, unpadded_k_len=300, seed=6), False),
]


@pytest.mark.parametrize("w,causal", ACASES, ids=lambda c: str(c) if not hasattr(c, "N") else f"{c.B}x{c.Hq}x{c.Hkv}x{c.N}x{c.D}")
def test_nvfp4_attention_on_oracle_codes(S, w, causal):
    q, k, v = W.make_qkv(w)
    oz = O.quantize_qkv_nvfp4(q, k, v, per_block_mean=True, unpadded_k_len=w.unpadded_k_len)
    ref = O.attention_nvfp4(oz, causal=causal, tie_band=TIE_BAND)
    out, lse = S.sage_attn_fwd_nvfp4(nvfp4_from_oracle(S, oz), causal=causal)
    if not causal:
        assert_attention_close(out, lse, ref, what=f"nvfp4 {w.N}")
    # Rows that see few keys (causal) hinge on single E2M1 roundings of P':
    # the oracle enumerates every rounding a relative change of P' below
    # TIE_BAND can flip and bounds the output move per element
    # (out_tie_bound); every row is held to that bound plus the parity bound,
    # the LSE (which uses the unquantised P) to the parity bound alone.
    o = out.float().cpu().numpy()
    excess = np.abs(o - ref["out"]) - ref["out_tie_bound"]
    assert excess.max() <= 2e-2, f"max excess {excess.max():.3g} over the tie bound"
    assert O.cosine(o, ref["out"]) >= 0.9995
    np.testing.assert_allclose(lse.cpu().numpy(), ref["lse"], rtol=0, atol=2e-2)


# The GPU's P' differs from the oracle's float64 one by its fp32 score
# arithmetic and MUFU exponentials: a few 1e-6 relative.
TIE_BAND = 1e-5


def test_nvfp4_longest_supported_key_length(S):
    """The longest key sequence the NVFP4 kernels accept (2048 key tiles),
    with the last 100 keys past unpadded_k_len: 256 queries, non-causal,
    through the whole path against the oracle."""
    wq = W.NVFP4.scaled(B=1, Hq=2, Hkv=1, N=256, D=128, unpadded_k_len=None, seed=43)
    wk = W.NVFP4.scaled(B=1, Hq=2, Hkv=1, N=128 * 2048, D=128, unpadded_k_len=None, seed=44)
    q = W.make_qkv(wq)[0]
    _, k, v = W.make_qkv(wk)
    L = 128 * 2048 - 100
    ref = O.attention_nvfp4(O.quantize_qkv_nvfp4(q, k, v, per_block_mean=True, unpadded_k_len=L))
    z = S.sage_quantize_qkv_nvfp4(q.cuda(), k.cuda(), v.cuda(), per_block_mean=True, unpadded_k_len=L)
    out, lse = S.sage_attn_fwd_nvfp4(z)
    assert_attention_close(out, lse, ref, what="nvfp4 Nk=262144")


@pytest.mark.parametrize("N,L,causal", [(1, 1, False), (1, 1, True), (256, 1, False), (256, 1, True)])
def test_nvfp4_degenerate_shapes(S, N, L, causal):
    """One token per head, and 256 queries that all see only the first key
    (unpadded_k_len = 1): P' of a row is then one vector holding a single
    non-zero entry.  Whole path against the oracle, with the tie bound."""
    w = W.NVFP4.scaled(B=2, Hq=4, Hkv=2, N=N, D=128, unpadded_k_len=L, seed=48 + N)
    q, k, v = W.make_qkv(w)
    ref = O.attention_nvfp4(O.quantize_qkv_nvfp4(q, k, v, per_block_mean=True, unpadded_k_len=L),
                            causal=causal, tie_band=TIE_BAND)
    z = S.sage_quantize_qkv_nvfp4(q.cuda(), k.cuda(), v.cuda(), per_block_mean=True, unpadded_k_len=L)
    out, lse = S.sage_attn_fwd_nvfp4(z, causal=causal)
    o = out.float().cpu().numpy()
    excess = np.abs(o - ref["out"]) - ref["out_tie_bound"]
    assert excess.max() <= 2e-2, f"max excess {excess.max():.3g} over the tie bound"
    assert O.cosine(o, ref["out"]) >= 0.9995
    np.testing.assert_allclose(lse.cpu().numpy(), ref["lse"], rtol=0, atol=2e-2)


def test_nvfp4_whole_path_global_mean(S):
    w = W.NVFP4.scaled(B=1, Hq=4, Hkv=4, N=512, D=128, unpadded_k_len=480, seed=11)
    q, k, v = W.make_qkv(w)
    ref = O.attention_nvfp4(O.quantize_qkv_nvfp4(q, k, v, per_block_mean=False, unpadded_k_len=480))
    z = S.sage_quantize_qkv_nvfp4(q.cuda(), k.cuda(), v.cuda(), per_block_mean=False, unpadded_k_len=480)
    out, lse = S.sage_attn_fwd_nvfp4(z)
    assert_attention_close(out, lse, ref, what="nvfp4 global mean")


def test_nvfp4_full_size_sampled(S):
    """The full NVFP4 workload (B=1, H=32, N=16384, unpadded 16000) on the
    GPU; the oracle checks two heads on the sampled rows."""
    w = W.NVFP4
    q, k, v = W.make_qkv(w)
    z = S.sage_quantize_qkv_nvfp4(q.cuda(), k.cuda(), v.cuda(), per_block_mean=True,
                                  unpadded_k_len=w.unpadded_k_len)
    out, lse = S.sage_attn_fwd_nvfp4(z)
    torch.cuda.synchronize()
    rows = W.sample_rows(w)
    for h in (0, w.Hq - 1):
        oz = O.quantize_qkv_nvfp4(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1], per_block_mean=True,
                                  unpadded_k_len=w.unpadded_k_len)
        sub = lambda t: t[:, h:h + 1]  # noqa: E731
        gsub = S.QuantizedNvfp4(*(sub(getattr(z, f)) for f in
                                  ("q", "q_sf", "k", "k_sf", "v_t", "v_sf_t", "qk_correction",
                                   "q_mean", "k_mean", "q_dot_kmean")),
                                1, 1, 1, w.N, w.N, w.D, w.unpadded_k_len, True)
        _compare_quant(gsub, oz)
        ref = O.attention_nvfp4(oz, rows=rows)
        assert_attention_close(out[:, h:h + 1], lse[:, h:h + 1], ref, rows=rows, what=f"nvfp4 h{h}")


@pytest.mark.parametrize("causal", [False, True])
def test_nvfp4_without_lse_matches_with_lse(S, causal):
    """return_lse=False (no LSE, no q.kmean needed) gives the same output as
    the LSE run, bit for bit, and needs no q_dot_kmean array."""
    w = W.NVFP4.scaled(B=1, Hq=2, Hkv=2, N=384, D=128, unpadded_k_len=350, seed=13)
    q, k, v = W.make_qkv(w)
    z = S.sage_quantize_qkv_nvfp4(q.cuda(), k.cuda(), v.cuda(), per_block_mean=True,
                                  unpadded_k_len=w.unpadded_k_len)
    out_lse, _ = S.sage_attn_fwd_nvfp4(z, causal=causal, return_lse=True)
    z.q_dot_kmean = None
    out = S.sage_attn_fwd_nvfp4(z, causal=causal, return_lse=False)
    torch.cuda.synchronize()
    assert torch.equal(out, out_lse)
    oz = O.quantize_qkv_nvfp4(q, k, v, per_block_mean=True, unpadded_k_len=w.unpadded_k_len)
    ref = O.attention_nvfp4(oz, causal=causal)
    o = out.float().cpu().numpy()
    assert O.cosine(o, ref["out"]) >= 0.9995
    if not causal:
        assert np.abs(o - ref["out"]).max() <= 2e-2


def test_nvfp4_quantize_fp16_and_both_head_dims(S):
    """Every (dtype, head_dim) instantiation of the quantiser launches (each
    sets its own shared-memory size), in an order that starts with d=64."""
    for D, dt in [(64, torch.float16), (128, torch.float16), (64, torch.bfloat16), (128, torch.bfloat16)]:
        w = W.NVFP4.scaled(B=1, Hq=2, Hkv=1, N=256, D=D, unpadded_k_len=256, seed=17)
        q, k, v = W.make_qkv(w, dtype=dt)
        oz = O.quantize_qkv_nvfp4(q, k, v, per_block_mean=True, unpadded_k_len=256)
        gz = S.sage_quantize_qkv_nvfp4(q.cuda(), k.cuda(), v.cuda(), per_block_mean=True,
                                       unpadded_k_len=256)
        torch.cuda.synchronize()
        _compare_quant(gz, oz)
