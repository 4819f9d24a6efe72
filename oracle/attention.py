"""Attention stage of SageAttention-style quantised attention, as a plain
CPU oracle, plus exact fp64 attention.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

INT8-QK / FP8-PV (thu-ml/sageattention llms.txt,
"sageattn_qk_int8_pv_fp8_cuda" and "sageattn_qk_int8_pv_fp8_cuda_sm90":
INT8 Q/K, per-channel FP8 V, FP32 accumulation of PV, causal mask, LSE;
"sageattn -- Auto-selecting attention kernel": GQA, ``sm_scale`` default
1/sqrt(d), LSE of shape [B, H, N]; "SageAttention Triton INT8/FP16 Kernel
Examples": boolean mask, True = attend):

* scores s_ij = S_int_ij * q_scale(i) * k_scale(j) * sm_scale, with S_int the
  exact integer dot product of the INT8 codes;
* masked keys (causal j > i + Nk - Nq, boolean mask False, j >= Nk) get
  s = -inf;
* an online softmax over key tiles of 128, in ascending order: the running
  max m is exact; before each tile's P is quantised, acc and l are rescaled
  by exp(m_old - m_new); p = exp(s - m_new) (<= 1); l += sum p (the
  unquantised p); P8 = E4M3_rn_satfinite(448 * p); acc += P8 . V8 (V8 the
  decoded FP8 codes);
* out = acc * vscale / (448 * l), rounded to bf16; a row with no visible key
  gives out = 0 and lse = -inf;
* lse = m + ln(l) + sm_scale * (q . kmean): the natural-log LSE of the
  original (unsmoothed) scaled scores, so that shards can be merged.

NVFP4 ("flashinfer.nvfp4_attention_sm120_fwd"): scores are
sm_scale * (deq(Q4) . deq(K4) + qk_correction[q block, j]); keys at and
beyond ``unpadded_k_len`` are masked; P' = 2688 * p (448 * 6, so that the
per-16-key scale factors sit in E4M3's normal range) is quantised per 16
keys with the same rule as Q/K/V; out = acc / (2688 * l).

Everything is float64 except the quantisation steps, which follow the
formats in ``oracle/formats.py``.
"""
from __future__ import annotations

import math

import numpy as np

from . import formats as F
from .quantize import BLOCK, NVFP4_VEC, _np64

LOG448 = math.log(448.0)


def default_sm_scale(D):
    return 1.0 / math.sqrt(D)


def _visible(rows, keys, Nq, Nk, causal, mask_rows, kv_limit=None):
    """Boolean [R, K] of visible (row, key) pairs for one (b, h).

    Keys >= ``kv_limit`` (default Nk) are hidden.  The causal rule is
    bottom-right aligned: key j is visible to row i when j <= i + Nk - Nq.
    """
    lim = Nk if kv_limit is None else kv_limit
    vis = np.broadcast_to(keys[None, :] < lim, (len(rows), len(keys))).copy()
    if causal:
        vis &= keys[None, :] <= rows[:, None] + (Nk - Nq)
    if mask_rows is not None:
        vis &= mask_rows
    return vis


def exact_attention(q, k, v, causal=False, sm_scale=None, mask=None, rows=None,
                    kv_len=None, bias=None):
    """Unquantised attention in float64.

    q [B,Hq,Nq,D], k/v [B,Hkv,Nk,D]; mask broadcastable to [B,Hq,Nq,Nk]
    (True = attend); ``bias`` a float mask broadcastable to [B,Hq,Nq,Nk]
    added to the scaled scores (-inf hides a key); ``kv_len`` masks keys
    >= kv_len.  Returns (out [B,Hq,R,D], lse [B,Hq,R]) for the query rows
    ``rows`` (default all).
    """
    q, k, v = _np64(q), _np64(k), _np64(v)
    B, Hq, Nq, D = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    sm_scale = default_sm_scale(D) if sm_scale is None else sm_scale
    rows = np.arange(Nq) if rows is None else np.asarray(rows)
    keys = np.arange(Nk)
    L = Nk if kv_len is None else kv_len
    m4 = None if mask is None else np.broadcast_to(np.asarray(mask, bool), (B, Hq, Nq, Nk))
    b4 = None if bias is None else np.broadcast_to(_np64(bias), (B, Hq, Nq, Nk))
    out = np.zeros((B, Hq, len(rows), D))
    lse = np.full((B, Hq, len(rows)), -np.inf)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            s = sm_scale * (q[b, h, rows] @ k[b, g].T)
            if b4 is not None:
                s = s + b4[b, h][rows]
            vis = _visible(rows, keys, Nq, Nk, causal,
                           None if m4 is None else m4[b, h][rows], kv_limit=L)
            vis = vis & (s > -np.inf)
            s = np.where(vis, s, -np.inf)
            mx = s.max(axis=1)
            ok = np.isfinite(mx)
            p = np.where(vis, np.exp(s - np.where(ok, mx, 0)[:, None]), 0.0)
            den = p.sum(axis=1)
            out[b, h] = np.where(ok[:, None], (p @ v[b, g]) / np.where(ok, den, 1)[:, None], 0.0)
            lse[b, h] = np.where(ok, mx + np.log(np.where(ok, den, 1)), -np.inf)
    return out, lse


def _online_softmax_rows(s, vis, vdec, quantise_p, p_gain, p_delta=None):
    """Tile-ordered online softmax for a block of rows of one (b, h).

    s: [R, Nk] float64 scores; vis: visibility; vdec: [Nk, D] decoded V;
    quantise_p(P') maps the pre-scaled probabilities of a tile [R, 128] to
    their decoded quantised values.  Returns (acc, l, m, bnd) where
    out = acc / (p_gain * l).  With ``p_delta`` (P' -> the largest change of
    each decoded value under a small relative perturbation of P'), ``bnd``
    [R, D] bounds how far acc can move by such perturbations:
    sum over keys of |change| * |V|, rescaled like acc; otherwise None.
    """
    R, Nk = s.shape
    D = vdec.shape[1]
    m = np.full(R, -np.inf)
    l = np.zeros(R)
    acc = np.zeros((R, D))
    bnd = None if p_delta is None else np.zeros((R, D))
    for t0 in range(0, Nk, BLOCK):
        t1 = min(Nk, t0 + BLOCK)
        st = np.where(vis[:, t0:t1], s[:, t0:t1], -np.inf)
        m_new = np.maximum(m, st.max(axis=1))
        live = np.isfinite(m_new)
        base = np.where(live, m_new, 0.0)
        alpha = np.where(np.isfinite(m), np.exp(m - base), 0.0)
        p = np.where(vis[:, t0:t1], np.exp(st - base[:, None]), 0.0)
        l = l * alpha + p.sum(axis=1)
        pq = quantise_p(p_gain * p)
        acc = acc * alpha[:, None] + pq @ vdec[t0:t1]
        if bnd is not None:
            bnd = bnd * alpha[:, None] + p_delta(p_gain * p) @ np.abs(vdec[t0:t1])
        m = m_new
    return acc, l, m, bnd


def _bf16_keep_nan(x):
    """bf16 rounding of the computed entries; NaN marks heads not computed."""
    return np.where(np.isnan(x), np.nan, F.bf16_round(np.nan_to_num(x, nan=0.0)))


def _p_e4m3(pp):
    return F.e4m3_round(pp)


def _p_nvfp4(pp):
    """Quantise pre-scaled P' per 16 keys (rows x 128 tile) to NVFP4 and
    return the decoded values."""
    R, T = pp.shape
    Tp = (T + NVFP4_VEC - 1) // NVFP4_VEC * NVFP4_VEC
    x = np.zeros((R, Tp), dtype=np.float32)
    x[:, :T] = pp                                   # P' rounded to fp32 first
    xv = x.reshape(R, Tp // NVFP4_VEC, NVFP4_VEC)
    a = np.max(np.abs(xv), axis=-1)
    sf = F.e4m3_encode((a / np.float32(6.0)).astype(np.float64))
    s = F.e4m3_decode(sf).astype(np.float32)
    inv = np.where(s > 0, np.float32(1.0) / np.where(s > 0, s, 1).astype(np.float32),
                   np.float32(0)).astype(np.float32)
    y = (xv * inv[..., None]).astype(np.float64)
    dec = F.e2m1_round(y) * s.astype(np.float64)[..., None]
    return dec.reshape(R, Tp)[:, :T]


def _nearby_grid_values(x, grid, band):
    """For values x >= 0 and a sorted grid of non-negative representable
    values with round-to-nearest: the representable value x rounds to, and
    the one it would round to instead if it moved by a relative amount of
    at most ``band`` across a midpoint (the same value when no midpoint is
    that close).  Values above the grid's top saturate to it."""
    x = np.asarray(x, np.float64)
    mids = (grid[1:] + grid[:-1]) / 2
    i = np.searchsorted(mids, x, side="left")           # x <= mids[i]: rounds down to grid[i]
    i = np.minimum(i, len(grid) - 1)
    # nearest midpoint below / above x
    lo_mid = np.where(i > 0, mids[np.maximum(i - 1, 0)], -np.inf)
    hi_mid = np.where(i < len(mids), mids[np.minimum(i, len(mids) - 1)], np.inf)
    near_lo = x - lo_mid <= band * x
    near_hi = hi_mid - x <= band * x
    alt = np.where(near_hi, np.minimum(i + 1, len(grid) - 1), np.where(near_lo, np.maximum(i - 1, 0), i))
    return grid[i], grid[alt]


def _p_nvfp4_delta(pp, band):
    """The largest change of each decoded NVFP4 P' value (rows x keys of one
    tile) that a relative perturbation of P' of at most ``band`` can cause.

    Such a perturbation (the GPU's fp32 exponentials and score arithmetic
    differ from this oracle's float64 ones by a few 1e-6 relative) can move
    an element across an E2M1 rounding midpoint (one grid step times the
    vector's scale) or move the vector's amax/6 across an E4M3 midpoint, in
    which case the whole vector is quantised with the neighbouring scale.
    Every such alternative is enumerated; the result is elementwise
    max |alternative - nominal| (0 where no midpoint is within reach)."""
    R, T = pp.shape
    Tp = (T + NVFP4_VEC - 1) // NVFP4_VEC * NVFP4_VEC
    x = np.zeros((R, Tp), dtype=np.float32)
    x[:, :T] = pp
    xv = x.reshape(R, Tp // NVFP4_VEC, NVFP4_VEC).astype(np.float32)
    e4 = np.unique(F.e4m3_decode(np.arange(0x7F, dtype=np.uint8)))      # 0 .. 448
    a = np.max(np.abs(xv), axis=-1)
    r = (a / np.float32(6.0)).astype(np.float64)
    s_nom, s_alt = _nearby_grid_values(r, e4, band)
    nominal = _p_nvfp4(pp).reshape(R, -1)
    nominal = np.pad(nominal, ((0, 0), (0, Tp - T))).reshape(xv.shape)
    delta = np.zeros(xv.shape)
    for sc in (s_nom, s_alt):
        scf = sc.astype(np.float32)
        inv = np.where(scf > 0, np.float32(1.0) / np.where(scf > 0, scf, 1), np.float32(0))
        y = (xv * inv.astype(np.float32)[..., None]).astype(np.float64)
        for g in _nearby_grid_values(np.abs(y), F.E2M1_GRID, band):
            delta = np.maximum(delta, np.abs(g * sc[..., None] - nominal))
    return delta.reshape(R, Tp)[:, :T]


def attention_i8f8(qz, causal=False, sm_scale=None, mask=None, rows=None, heads=None,
                   return_internal=False, bias=None):
    """Oracle of the fused INT8-QK / FP8-PV attention on quantised inputs.

    qz: dict from ``quantize_qkv_i8f8``.  mask: boolean broadcastable to
    [B, Hq, Nq, Nk] or None.  bias: float mask broadcastable to
    [B, Hq, Nq, Nk] added to the scaled scores ("sageattn_qk_int8_pv_fp16_triton":
    an optional boolean or float32 attention mask; -inf hides a key), or
    None.  rows: query rows to compute (default all).
    heads: iterable of (b, h) pairs (default all).  Returns dict with
    ``out`` (bf16-rounded, float64 array [B, Hq, R, D]), ``out_f64`` (before
    rounding), ``lse`` [B, Hq, R]; entries for heads not computed are NaN.
    """
    B, Hq, Hkv, Nq, Nk, D = (qz[x] for x in ("B", "Hq", "Hkv", "Nq", "Nk", "D"))
    G = Hq // Hkv
    sm_scale = default_sm_scale(D) if sm_scale is None else float(sm_scale)
    rows = np.arange(Nq) if rows is None else np.asarray(rows)
    keys = np.arange(Nk)
    heads = [(b, h) for b in range(B) for h in range(Hq)] if heads is None else list(heads)
    m4 = None if mask is None else np.broadcast_to(np.asarray(mask, bool), (B, Hq, Nq, Nk))
    b4 = None if bias is None else np.broadcast_to(np.asarray(bias, np.float64), (B, Hq, Nq, Nk))
    out = np.full((B, Hq, len(rows), D), np.nan)
    lse = np.full((B, Hq, len(rows)), np.nan)
    for b, h in heads:
        g = h // G
        qc = qz["q"][b, h, rows].astype(np.float64)
        kc = qz["k"][b, g, :Nk].astype(np.float64)
        S = qc @ kc.T                                            # exact integers
        qs = qz["q_scale"][b, h, rows // BLOCK].astype(np.float64)
        ks = qz["k_scale"][b, g, keys // BLOCK].astype(np.float64)
        s = S * qs[:, None] * ks[None, :] * sm_scale
        if b4 is not None:
            s = s + b4[b, h][rows]
        vis = _visible(rows, keys, Nq, Nk, causal, None if m4 is None else m4[b, h][rows])
        vis &= s > -np.inf
        vdec = F.e4m3_decode(qz["v_t"][b, g, :, :Nk]).T          # [Nk, D]
        acc, l, m, _ = _online_softmax_rows(s, vis, vdec, _p_e4m3, 448.0)
        vs = qz["v_scale"][b, g].astype(np.float64)
        ok = l > 0
        o = np.where(ok[:, None], acc * vs[None, :] / (448.0 * np.where(ok, l, 1))[:, None], 0.0)
        out[b, h] = o
        lse[b, h] = np.where(ok, m + np.log(np.where(ok, l, 1)) + sm_scale * qz["q_dot_kmean"][b, h, rows],
                             -np.inf)
    return dict(out=_bf16_keep_nan(out), out_f64=out, lse=lse, rows=rows)


def attention_nvfp4(qz, causal=False, sm_scale=None, rows=None, heads=None, tie_band=None):
    """Oracle of the NVFP4 attention on the output of ``quantize_qkv_nvfp4``.

    With ``tie_band`` (a relative width, e.g. 1e-5) the result also holds
    ``out_tie_bound`` [B, Hq, R, D]: how far the output can move when P' is
    perturbed by at most that relative amount before its NVFP4 quantisation
    (``_p_nvfp4_delta``).  A row that sees few keys hinges on single E2M1
    roundings of P', so every output in out +- out_tie_bound is as correct as
    the oracle's own for an implementation whose P' differs by rounding."""
    B, Hq, Hkv, Nq, Nk, D = (qz[x] for x in ("B", "Hq", "Hkv", "Nq", "Nk", "D"))
    L = qz["unpadded_k_len"]
    G = Hq // Hkv
    sm_scale = default_sm_scale(D) if sm_scale is None else float(sm_scale)
    rows = np.arange(Nq) if rows is None else np.asarray(rows)
    keys = np.arange(Nk)
    heads = [(b, h) for b in range(B) for h in range(Hq)] if heads is None else list(heads)
    out = np.full((B, Hq, len(rows), D), np.nan)
    lse = np.full((B, Hq, len(rows)), np.nan)
    tie = None if tie_band is None else np.full((B, Hq, len(rows), D), np.nan)
    p_delta = None if tie_band is None else (lambda pp: _p_nvfp4_delta(pp, tie_band))

    def deq(code, sf, lead):
        vals = F.e2m1_decode(code).reshape(lead + (-1, NVFP4_VEC))
        return (vals * F.e4m3_decode(sf)[..., None]).reshape(lead + (-1,))

    for b, h in heads:
        g = h // G
        qd = deq(qz["q"][b, h, rows], qz["q_sf"][b, h, rows], (len(rows),))
        kd = deq(qz["k"][b, g, :Nk], qz["k_sf"][b, g, :Nk], (Nk,))
        corr = qz["qk_correction"][b, h][rows // BLOCK][:, :Nk].astype(np.float64)
        s = sm_scale * (qd @ kd.T + corr)
        vis = _visible(rows, keys, Nq, Nk, causal, None, kv_limit=L)
        vdec = deq(qz["v_t"][b, g], qz["v_sf_t"][b, g], (D,))[:, :Nk].T     # [Nk, D]
        acc, l, m, bnd = _online_softmax_rows(s, vis, vdec, _p_nvfp4, 448.0 * 6.0, p_delta)
        ok = l > 0
        out[b, h] = np.where(ok[:, None], acc / (2688.0 * np.where(ok, l, 1))[:, None], 0.0)
        if tie is not None:
            tie[b, h] = np.where(ok[:, None], bnd / (2688.0 * np.where(ok, l, 1))[:, None], 0.0)
        lse[b, h] = np.where(ok, m + np.log(np.where(ok, l, 1)) + sm_scale * qz["q_dot_kmean"][b, h, rows],
                             -np.inf)
    res = dict(out=_bf16_keep_nan(out), out_f64=out, lse=lse, rows=rows)
    if tie is not None:
        res["out_tie_bound"] = tie
    return res


def cosine(a, b):
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))


def qk_int32_tile(qz, b, h, qblk, kblk):
    """Exact integer QK^T of one 128x128 tile of INT8 codes (the int32
    block product the kernel's first MMA chain produces): rows qblk*128.., keys kblk*128.., of the
    Q head h and its KV head h // G.  Returns int64 [128, 128]; the float64
    matmul is exact because |S| < 2**53."""
    G = qz["Hq"] // qz["Hkv"]
    qc = qz["q"][b, h, qblk * BLOCK:(qblk + 1) * BLOCK].astype(np.float64)
    kc = qz["k"][b, h // G, kblk * BLOCK:(kblk + 1) * BLOCK].astype(np.float64)
    return (qc @ kc.T).astype(np.int64)
