"""Pins for oracle/attention.py: lossless special cases against exact fp64
attention, invariants, mask/causal/GQA identities, brute-force integer
QK^T, and the pages' shape contracts (no GPU)."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from lossless_cases import LN2, i8f8_case, nvfp4_case

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_examples.json")))


# ------------------------------------------------------------ exact attention
def test_exact_attention_rows_sum_to_one_and_shift_invariance():
    q, k, v = W.make_qkv(W.TINY.scaled(Hq=2, Hkv=1, N=200))
    ones = torch.ones_like(v, dtype=torch.float64)
    out1, _ = O.exact_attention(q, k, ones, sm_scale=0.3)
    np.testing.assert_allclose(out1, 1.0, rtol=0, atol=1e-12)
    c = torch.randn(1, 1, 1, 64, dtype=torch.float64) * 5
    outa, lsea = O.exact_attention(q, k, v, sm_scale=0.3)
    outb, lseb = O.exact_attention(q, k.double() + c, v, sm_scale=0.3)
    np.testing.assert_allclose(outa, outb, rtol=1e-10, atol=1e-12)
    qc = np.einsum("bhnc,c->bhn", q.double().numpy(), c[0, 0, 0].numpy())
    np.testing.assert_allclose(lseb - lsea, 0.3 * qc, atol=1e-9)


def test_exact_attention_matches_torch_sdpa():
    q, k, v = W.make_qkv(W.TINY.scaled(N=130))
    for causal in (False, True):
        out, lse = O.exact_attention(q, k, v, causal=causal, sm_scale=0.2)
        ref = torch.nn.functional.scaled_dot_product_attention(
            q.double(), k.double(), v.double(), is_causal=causal, scale=0.2)
        np.testing.assert_allclose(out, ref.numpy(), atol=1e-12)
        s = 0.2 * q.double() @ k.double().transpose(-1, -2)
        if causal:
            s = s.masked_fill(torch.ones(130, 130, dtype=torch.bool).triu(1), -math.inf)
        np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), atol=1e-12)


# ------------------------------------------------------------ lossless INT8/FP8
@pytest.mark.parametrize("N,Hq,Hkv,causal", [(256, 2, 2, False), (256, 2, 2, True),
                                             (300, 4, 2, False), (200, 4, 1, True),
                                             (384, 2, 1, False)])
def test_i8f8_oracle_equals_exact_attention_when_lossless(N, Hq, Hkv, causal):
    q, k, v = i8f8_case(B=1, Hq=Hq, Hkv=Hkv, N=N, D=64, seed=N + Hq)
    qz = O.quantize_qkv_i8f8(q, k, v)
    # the construction really is lossless
    assert np.all(qz["q_scale"] == 1) and np.all(qz["k_scale"] == 1) and np.all(qz["v_scale"] == 1)
    assert np.all(qz["k_mean"] == 0)
    np.testing.assert_array_equal(qz["q"][:, :, :N], q.double().numpy())
    r = O.attention_i8f8(qz, causal=causal, sm_scale=LN2)
    ex, lse = O.exact_attention(q, k, v, causal=causal, sm_scale=LN2)
    np.testing.assert_allclose(r["out_f64"], ex, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(r["lse"], lse, rtol=1e-12, atol=1e-12)


def test_i8f8_lossless_with_mask():
    q, k, v = i8f8_case(B=1, Hq=2, Hkv=2, N=256, D=64, seed=9)
    g = torch.Generator().manual_seed(9)
    mask = torch.rand(1, 1, 256, 256, generator=g) < 0.7
    mask[..., 0] = True
    qz = O.quantize_qkv_i8f8(q, k, v)
    r = O.attention_i8f8(qz, sm_scale=LN2, mask=mask.numpy())
    ex, lse = O.exact_attention(q, k, v, sm_scale=LN2, mask=mask.numpy())
    np.testing.assert_allclose(r["out_f64"], ex, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(r["lse"], lse, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------ identities on random data
def _random_qz(N=300, Hq=4, Hkv=2, D=64, seed=0):
    q, k, v = W.make_qkv(W.TINY.scaled(N=N, Hq=Hq, Hkv=Hkv, D=D, seed=seed))
    return q, k, v, O.quantize_qkv_i8f8(q, k, v)


def test_mask_second_half_equals_truncated_keys():
    mcase = GOLDEN["mask_second_half"]
    assert mcase["visible_keys"] == "first half"
    q, k, v, qz = _random_qz(N=256, Hq=2, Hkv=2)
    mask = np.ones((1, 1, 256, 256), bool)
    mask[..., 128:] = False                     # mask[:, :, :, N // 2:] = False
    rm = O.attention_i8f8(qz, mask=mask)
    cut = dict(qz, Nk=128)                      # same codes and scales, keys 0..127 only
    rt = O.attention_i8f8(cut)
    np.testing.assert_array_equal(rm["out"], rt["out"])
    np.testing.assert_array_equal(rm["lse"], rt["lse"])


def test_causal_row_equals_truncated_keys():
    q, k, v, qz = _random_qz(N=300, Hq=2, Hkv=1)
    rows = [0, 5, 127, 128, 200, 299]
    rc = O.attention_i8f8(qz, causal=True, rows=rows)
    for i, r in enumerate(rows):
        rt = O.attention_i8f8(dict(qz, Nk=r + 1), rows=[r])
        np.testing.assert_array_equal(rc["out"][:, :, i], rt["out"][:, :, 0])
        np.testing.assert_array_equal(rc["lse"][:, :, i], rt["lse"][:, :, 0])


def test_gqa_equals_repeated_kv_heads():
    """16 Q heads over 4 KV heads: Q head h uses KV head h // 4."""
    q, k, v = W.make_qkv(W.TINY.scaled(Hq=8, Hkv=2, N=130))
    r = O.attention_i8f8(O.quantize_qkv_i8f8(q, k, v))
    k4, v4 = k.repeat_interleave(4, dim=1), v.repeat_interleave(4, dim=1)
    r4 = O.attention_i8f8(O.quantize_qkv_i8f8(q, k4, v4))
    np.testing.assert_array_equal(r["out"], r4["out"])
    np.testing.assert_array_equal(r["lse"], r4["lse"])


def test_fully_masked_row_gives_zero_and_minus_inf():
    q, k, v, qz = _random_qz(N=128, Hq=2, Hkv=2)
    mask = np.ones((1, 1, 128, 128), bool)
    mask[0, 0, 3, :] = False
    r = O.attention_i8f8(qz, mask=mask)
    assert np.all(r["out"][0, :, 3] == 0) and np.all(r["lse"][0, :, 3] == -np.inf)
    assert np.all(np.isfinite(r["lse"][0, :, 4]))


def test_sm_scale_default_is_inverse_sqrt_d():
    assert O.default_sm_scale(128) == pytest.approx(GOLDEN["nvfp4_layout"]["sm_scale_default"], rel=1e-15)
    q, k, v, qz = _random_qz(N=128, Hq=2, Hkv=2, D=64)
    np.testing.assert_array_equal(O.attention_i8f8(qz)["out"], O.attention_i8f8(qz, sm_scale=0.125)["out"])


def test_qk_int32_tile_brute_force():
    q, k, v, qz = _random_qz(N=256, Hq=2, Hkv=1, D=64)
    t = O.qk_int32_tile(qz, 0, 1, 1, 0)
    qc = qz["q"][0, 1, 128:256].tolist()
    kc = qz["k"][0, 0, 0:128].tolist()
    for i in range(0, 128, 7):
        for j in range(0, 128, 5):
            assert t[i, j] == sum(a * b for a, b in zip(qc[i], kc[j]))


def test_oracle_close_to_exact_attention_on_tiny_workload():
    """Sanity floor (the pages print no accuracy number): the INT8/FP8
    oracle is within cosine 0.999 of fp64 attention on the tiny workload,
    NVFP4 within 0.97."""
    w = W.TINY
    q, k, v = W.make_qkv(w)
    ex, lse = O.exact_attention(q, k, v, sm_scale=w.sm_scale)
    r = O.attention_i8f8(O.quantize_qkv_i8f8(q, k, v), sm_scale=w.sm_scale)
    assert O.cosine(r["out"], ex) > 0.999
    assert np.abs(r["lse"] - lse).max() < 0.05
    rn = O.attention_nvfp4(O.quantize_qkv_nvfp4(q, k, v), sm_scale=w.sm_scale)
    assert O.cosine(rn["out"], ex) > 0.97


# ------------------------------------------------------------ NVFP4
@pytest.mark.parametrize("per_block_mean,L,causal", [(True, 256, False), (False, 224, False),
                                                     (True, 192, True)])
def test_nvfp4_oracle_equals_exact_attention_when_lossless(per_block_mean, L, causal):
    q, k, v = nvfp4_case(B=1, Hq=2, Hkv=1, N=256, D=64, L=L, seed=L)
    qz = O.quantize_qkv_nvfp4(q, k, v, per_block_mean=per_block_mean, unpadded_k_len=L)
    assert np.all(qz["qk_correction"] == 0) and np.all(qz["k_mean"] == 0)
    assert np.all(O.e4m3_decode(qz["q_sf"]) == 1)
    r = O.attention_nvfp4(qz, causal=causal, sm_scale=LN2)
    ex, lse = O.exact_attention(q, k, v, causal=causal, sm_scale=LN2, kv_len=L)
    np.testing.assert_allclose(r["out_f64"], ex, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(r["lse"], lse, rtol=1e-12, atol=1e-12)


def test_nvfp4_layout_contract():
    lay = GOLDEN["nvfp4_layout"]
    q, k, v = W.make_qkv(W.NVFP4.scaled(Hq=2, Hkv=2, N=256, unpadded_k_len=200))
    qz = O.quantize_qkv_nvfp4(q, k, v, unpadded_k_len=200)
    D = 128
    assert qz["q_packed"].shape == (1, 2, 256, D // 2)                   # [B, Hqo, M_pad, D/2]
    assert qz["k_packed"].shape == (1, 2, 256, D // 2)                   # [B, Hkv, N_pad, D/2]
    assert qz["qk_correction"].shape[2] == 256 // 128                    # one row per Q block
    assert lay["q_fp4"][-1] == lay["head_dim"] // 2
    assert lay["qk_correction_rows_per_head"] == lay["M"] // 128
    # keys at and beyond unpadded_k_len are masked: changing them changes nothing
    r1 = O.attention_nvfp4(qz, rows=[0, 100, 255])
    qz2 = dict(qz)
    qz2["k"] = qz["k"].copy()
    qz2["k"][:, :, 200:] = 7
    qz2["k_sf"] = qz["k_sf"].copy()
    qz2["k_sf"][:, :, 200:] = 0x38
    r2 = O.attention_nvfp4(qz2, rows=[0, 100, 255])
    np.testing.assert_array_equal(r1["out"], r2["out"])


@pytest.mark.parametrize("case", GOLDEN["shape_cases"], ids=lambda c: c["cite"][-40:])
def test_page_shape_contracts(case):
    """out has q's shape and lse is [B, H, N] (N shortened to 128: the
    contract holds at any length)."""
    B, Hq, _, D = case["q"]
    Hkv = case["kv"][1]
    N = 128
    w = W.TINY.scaled(B=B, Hq=Hq, Hkv=Hkv, N=N, D=D)
    q, k, v = W.make_qkv(w)
    heads = [(0, 0), (B - 1, Hq - 1)]
    r = O.attention_i8f8(O.quantize_qkv_i8f8(q, k, v), causal=case.get("causal", False), heads=heads)
    assert r["out"].shape == (B, Hq, N, D) and tuple(case["out"][:2]) == (B, Hq)
    assert r["lse"].shape == (B, Hq, N) and tuple(case["lse"][:2]) == (B, Hq)
    assert case["out"][3] == D and case["lse"][2] == case["q"][2]


def test_nvfp4_short_causal_rows_are_tie_sensitive():
    """The oracle's own sensitivity that bounds GPU parity on short causal
    rows: a 2e-6 relative change of P' moves some output by more than 2e-2
    (this bounds what any fp32 implementation can match there)."""
    from oracle import attention as A
    w = W.NVFP4.scaled(B=1, Hq=4, Hkv=2, N=640, D=128, unpadded_k_len=600, seed=5)
    q, k, v = W.make_qkv(w)
    oz = O.quantize_qkv_nvfp4(q, k, v, per_block_mean=True, unpadded_k_len=600)
    ref = O.attention_nvfp4(oz, causal=True)
    rng = np.random.default_rng(0)
    orig = A._p_nvfp4
    try:
        A._p_nvfp4 = lambda pp: orig(pp * (1 + rng.uniform(-2e-6, 2e-6, pp.shape)))
        alt = O.attention_nvfp4(oz, causal=True)
    finally:
        A._p_nvfp4 = orig
    d = np.abs(alt["out"] - ref["out"])
    assert d.max() > 2e-2 and O.cosine(alt["out"], ref["out"]) > 0.9999
    assert np.all(np.argwhere(d > 2e-2)[:, 2] < 127)     # only rows that see < 128 keys


# ------------------------------------------------------------ float additive mask
# ("sageattn_qk_int8_pv_fp16_triton": an optional boolean or float32 attention
# mask; the float mask is added to the scaled scores, -inf hides a key)
def _bias_case(seed=71):
    w = W.TINY.scaled(B=1, Hq=2, Hkv=1, N=256, D=64, seed=seed)
    q, k, v = W.make_qkv(w)
    g = torch.Generator().manual_seed(seed)
    bias = torch.randn(1, 2, 256, 256, generator=g).double()
    bias[..., 200:] = float("-inf")
    bias[0, 1, 7, :] = float("-inf")                     # a row that sees nothing
    return q, k, v, bias


def test_exact_attention_float_mask_matches_torch_sdpa():
    q, k, v, bias = _bias_case()
    out, lse = O.exact_attention(q, k, v, bias=bias.numpy())
    qq, kk, vv = (t.double() for t in (q, k, v))
    kk = kk.repeat_interleave(2, dim=1)
    vv = vv.repeat_interleave(2, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=bias)
    ok = np.isfinite(lse)
    np.testing.assert_allclose(out[ok], ref.numpy()[ok], rtol=0, atol=1e-12)
    assert np.all(out[~ok] == 0) and not ok[0, 1, 7]


def test_float_mask_zero_and_minus_inf_reduce_to_no_mask_and_bool_mask():
    q, k, v, _ = _bias_case(72)
    z = O.quantize_qkv_i8f8(q, k, v)
    plain = O.attention_i8f8(z)
    zero = O.attention_i8f8(z, bias=np.zeros((1, 1, 256, 256)))
    np.testing.assert_array_equal(zero["out"], plain["out"])
    np.testing.assert_array_equal(zero["lse"], plain["lse"])
    keep = np.ones((1, 1, 256, 256), bool)
    keep[..., 100:180] = False
    bias = np.where(keep, 0.0, -np.inf)
    a = O.attention_i8f8(z, mask=keep)
    b = O.attention_i8f8(z, bias=bias)
    np.testing.assert_array_equal(a["out"], b["out"])
    np.testing.assert_array_equal(a["lse"], b["lse"])


def test_float_mask_lossless_equals_exact():
    """Lossless codes and a bias of 0 or -ln 2: the quantised oracle must
    equal exact attention with the same bias.  (Integer scores in [-7, 7]
    plus the bias keep every exponent gap within 15, and 448 * 2**-k is an
    exact E4M3 value for k <= 15.)"""
    q, k, v = i8f8_case(B=1, Hq=2, Hkv=2, N=256, D=64, seed=73)
    g = torch.Generator().manual_seed(73)
    bias = -LN2 * torch.randint(0, 2, (1, 2, 256, 256), generator=g).double().numpy()
    bias[..., 240:] = -np.inf
    r = O.attention_i8f8(O.quantize_qkv_i8f8(q, k, v), sm_scale=LN2, bias=bias)
    ex, ex_lse = O.exact_attention(q, k, v, sm_scale=LN2, bias=bias)
    np.testing.assert_allclose(r["out_f64"], ex, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["lse"], ex_lse, rtol=0, atol=1e-12)


def test_float_mask_row_constant_shifts_only_the_lse():
    q, k, v, _ = _bias_case(74)
    z = O.quantize_qkv_i8f8(q, k, v)
    shift = np.linspace(-3, 5, 256)[None, None, :, None]
    a = O.attention_i8f8(z)
    b = O.attention_i8f8(z, bias=np.broadcast_to(shift, (1, 1, 256, 256)))
    np.testing.assert_allclose(b["out_f64"], a["out_f64"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(b["lse"] - a["lse"], np.broadcast_to(shift[..., 0], a["lse"].shape),
                               rtol=0, atol=1e-12)


# ------------------------------------------------------------ NVFP4 P quantisation, by hand
# ("flashinfer.nvfp4_attention_sm120_fwd": P is quantised to NVFP4 for the PV
# product -- per 16 keys an E4M3 scale factor E4M3(amax / 6) and E2M1 codes of
# P' / scale, round to nearest with ties to the even code, saturating at 6.)
# Each vector's decoded values are worked out by hand from the E2M1 grid
# {0, .5, 1, 1.5, 2, 3, 4, 6} and the E4M3 grid, not by the oracle's code.
P_HAND = [
    # amax 1536: scale E4M3(256) = 256 exactly, so P'/256 is exact and every
    # tie lands on a midpoint: 2.5 -> 2, 1.75 -> 2, 1.25 -> 1, 0.75 -> 1, 0.25 -> 0
    ([1536, 1024, 768, 640, 512, 448, 384, 320, 256, 192, 128, 64, 100, 50, 1300, 1270],
     [1536, 1024, 768, 512, 512, 512, 384, 256, 256, 256, 128, 0, 128, 0, 1536, 1024]),
    # amax 2688 (the largest P' = 448 * 6): scale 448; no value near a midpoint
    ([2688, 2000, 1400, 1000, 700, 500, 300, 150, 90, 2300, 1600, 1200, 800, 550, 400, 0],
     [2688, 1792, 1344, 896, 672, 448, 224, 224, 0, 2688, 1792, 1344, 896, 448, 448, 0]),
    # amax 1000: amax/6 = 166.7 rounds to the E4M3 value 160 (grid step 16 in
    # [128, 256)); 1000/160 = 6.25 saturates to 6
    ([1000, 880, 720, 600, 520, 410, 300, 210, 130, 60, 30, 960, 640, 480, 320, 240],
     [960, 960, 640, 640, 480, 480, 320, 240, 160, 80, 0, 960, 640, 480, 320, 240]),
    # amax 0.05: amax/6 = 0.00833 is an E4M3 subnormal, 4 * 2^-9 = 2^-7
    ([0.05, 0.03, 0.01, 0.004, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0],
     [6 / 128, 4 / 128, 1.5 / 128, 0.5 / 128] + [0] * 12),
    # an all-zero vector (a key range the row does not see): scale 0, codes 0
    ([0] * 16, [0] * 16),
]


def test_p_nvfp4_hand_computed_vectors():
    from oracle import attention as A
    pp = np.array([v for v, _ in P_HAND], dtype=np.float64)          # 5 rows x 16 keys
    want = np.array([d for _, d in P_HAND], dtype=np.float64)
    np.testing.assert_array_equal(A._p_nvfp4(pp), want)
    # a 128-key tile is eight independent vectors: rotate the rows through it
    tile = np.concatenate([np.roll(pp, s, axis=0) for s in range(8)], axis=1)
    wtile = np.concatenate([np.roll(want, s, axis=0) for s in range(8)], axis=1)
    np.testing.assert_array_equal(A._p_nvfp4(tile), wtile)


def test_p_nvfp4_tie_bound_covers_every_small_perturbation():
    """The oracle's tie bound (``attention_nvfp4(tie_band=...)``) must hold
    every output that P' perturbed by less than the band produces: a
    perturbed run stays inside out +- out_tie_bound on every row, and the
    bound is non-trivial exactly on the rows that see few keys."""
    from oracle import attention as A
    w = W.NVFP4.scaled(B=1, Hq=4, Hkv=2, N=640, D=128, unpadded_k_len=600, seed=5)
    q, k, v = W.make_qkv(w)
    oz = O.quantize_qkv_nvfp4(q, k, v, per_block_mean=True, unpadded_k_len=600)
    band = 1e-5
    ref = O.attention_nvfp4(oz, causal=True, tie_band=band)
    bound = ref["out_tie_bound"]
    orig = A._p_nvfp4
    worst = 0.0
    try:
        for seed in range(3):
            rng = np.random.default_rng(seed)
            A._p_nvfp4 = lambda pp: orig(pp * (1 + rng.uniform(-0.9 * band, 0.9 * band, pp.shape)))
            alt = O.attention_nvfp4(oz, causal=True)
            d = np.abs(alt["out_f64"] - ref["out_f64"])
            assert np.all(d <= bound + 1e-12)
            worst = max(worst, d.max())
    finally:
        A._p_nvfp4 = orig
    assert worst > 2e-2                                  # the flips do happen here
    short = bound[:, :, :127].max()
    assert short > 2e-2 and bound[:, :, 256:].max() < 2e-2


def test_p_nvfp4_tie_bound_is_zero_without_nearby_midpoints():
    """Lossless NVFP4 inputs put every P' on a representable value (never
    within 1e-5 of a midpoint), so the tie bound vanishes."""
    from lossless_cases import LN2, nvfp4_case
    q, k, v = nvfp4_case(B=1, Hq=2, Hkv=1, N=256, D=64, L=256, seed=3)
    oz = O.quantize_qkv_nvfp4(q, k, v, per_block_mean=True, unpadded_k_len=256)
    r = O.attention_nvfp4(oz, causal=True, sm_scale=LN2, tie_band=1e-5)
    assert np.all(r["out_tie_bound"] == 0)
