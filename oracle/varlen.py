"""Oracle of variable-length (packed) attention.

TEST INFRASTRUCTURE ONLY (see the package header).

thu-ml/sageattention llms.txt, "sageattn_varlen": a batch of sequences of
different lengths is given as packed tensors q [total_q, Hq, D] and
k, v [total_k, Hkv, D] with cumulative length arrays cu_seqlens_q/k
(starting at 0), equivalent to flash_attn_varlen_func but with
SageAttention's quantisation (per-block INT8 QK, smooth_k).

Reading (the pages give the interface, not the quantisation boundaries):
every sequence is its own problem.  Its K mean is taken over its own keys,
its 128-token quantisation blocks start at its first token, its V channel
scales are its own, and the causal mask is bottom-right aligned within it.
The varlen result is therefore the dense oracle applied sequence by
sequence.  The LSE of a packed call is laid out as one [Hq, len_s] block per
sequence, concatenated in sequence order.
"""
import numpy as np

from .attention import attention_i8f8
from .quantize import quantize_qkv_i8f8


def _np64(x):
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.asarray(x, dtype=np.float64)


def check_cu_seqlens(cu, total):
    """cu: non-decreasing integers starting at 0 and ending at ``total``."""
    cu = np.asarray(cu, dtype=np.int64)
    if cu.ndim != 1 or len(cu) < 2 or cu[0] != 0 or cu[-1] != total or np.any(np.diff(cu) < 0):
        raise ValueError("cu_seqlens must start at 0, end at the packed length and not decrease")
    return cu


def attention_varlen_i8f8(q, k, v, cu_seqlens_q, cu_seqlens_k, causal=False, sm_scale=None,
                          smooth_k=True):
    """Varlen INT8-QK / FP8-PV attention.

    q: [total_q, Hq, D], k/v: [total_k, Hkv, D] (bf16/fp16 values).
    Returns dict ``out`` [total_q, Hq, D] (bf16-rounded), ``out_f64``,
    ``lse`` (flat, one [Hq, len_s] block per sequence) and ``per_seq``, the
    list of (quantised inputs, dense result) of every non-empty sequence.
    """
    q, k, v = _np64(q), _np64(k), _np64(v)
    total_q, Hq, D = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    cq = check_cu_seqlens(cu_seqlens_q, total_q)
    ck = check_cu_seqlens(cu_seqlens_k, total_k)
    if len(cq) != len(ck):
        raise ValueError("cu_seqlens_q and cu_seqlens_k describe different numbers of sequences")
    out = np.zeros((total_q, Hq, D))
    out_f64 = np.zeros((total_q, Hq, D))
    lse = np.zeros(Hq * total_q)
    per_seq = []
    for s in range(len(cq) - 1):
        q0, q1, k0, k1 = cq[s], cq[s + 1], ck[s], ck[s + 1]
        nq, nk = q1 - q0, k1 - k0
        if nq == 0:
            continue
        if nk == 0:                                  # no key at all: out 0, lse -inf
            lse[Hq * q0:Hq * q1] = -np.inf
            continue
        # one sequence as a dense [1, H, N, D] problem
        qs = np.transpose(q[q0:q1], (1, 0, 2))[None]
        ks = np.transpose(k[k0:k1], (1, 0, 2))[None]
        vs = np.transpose(v[k0:k1], (1, 0, 2))[None]
        qz = quantize_qkv_i8f8(qs, ks, vs, smooth_k=smooth_k)
        r = attention_i8f8(qz, causal=causal, sm_scale=sm_scale)
        out[q0:q1] = np.transpose(r["out"][0], (1, 0, 2))
        out_f64[q0:q1] = np.transpose(r["out_f64"][0], (1, 0, 2))
        lse[Hq * q0:Hq * q1] = r["lse"][0].reshape(-1)
        per_seq.append((s, qz, r))
    return dict(out=out, out_f64=out_f64, lse=lse, per_seq=per_seq)


def block_diagonal_mask(cu_seqlens_q, cu_seqlens_k, causal=False):
    """Boolean [total_q, total_k]: key j visible to query i of the packed
    batch (same sequence; bottom-right causal within it when ``causal``)."""
    cq = np.asarray(cu_seqlens_q, dtype=np.int64)
    ck = np.asarray(cu_seqlens_k, dtype=np.int64)
    m = np.zeros((cq[-1], ck[-1]), dtype=bool)
    for s in range(len(cq) - 1):
        nq, nk = cq[s + 1] - cq[s], ck[s + 1] - ck[s]
        blk = np.ones((nq, nk), dtype=bool)
        if causal:
            blk = np.arange(nk)[None, :] <= np.arange(nq)[:, None] + (nk - nq)
        m[cq[s]:cq[s + 1], ck[s]:ck[s + 1]] = blk
    return m
