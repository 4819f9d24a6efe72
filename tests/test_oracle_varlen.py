"""Pins for oracle/varlen.py (thu-ml/sageattention llms.txt, "sageattn_varlen").

The varlen oracle composes the dense one sequence by sequence; these pins
check that composition against definitions it does not use:
* lossless sequences packed together must equal exact fp64 attention on the
  whole packed batch under a block-diagonal (and, with causal, bottom-right
  per-sequence) mask, which pins the sequence boundaries, the per-sequence
  causal alignment and the packing;
* one sequence equals the dense oracle;
* a sequence's result does not depend on its neighbours;
* empty sequences and malformed cu_seqlens.
"""
import numpy as np
import pytest
import torch

import oracle as O
from oracle.varlen import attention_varlen_i8f8, block_diagonal_mask, check_cu_seqlens
import workloads as W
from lossless_cases import LN2, i8f8_case


def _pack(parts):
    """[1, H, n, D] tensors -> packed [sum n, H, D]."""
    return torch.cat([p[0].transpose(0, 1) for p in parts], dim=0)


def _lossless_varlen(lens, Hq=2, Hkv=1, D=64, seed=0):
    qs, ks, vs = [], [], []
    for i, n in enumerate(lens):
        q, k, v = i8f8_case(B=1, Hq=Hq, Hkv=Hkv, N=n, D=D, seed=seed + 10 * i)
        qs.append(q); ks.append(k); vs.append(v)
    cu = np.concatenate([[0], np.cumsum(lens)])
    return _pack(qs), _pack(ks), _pack(vs), cu


@pytest.mark.parametrize("causal", [False, True])
def test_lossless_varlen_equals_block_diagonal_exact_attention(causal):
    lens = [256, 130, 384, 2]                    # ragged, one tiny
    q, k, v, cu = _lossless_varlen(lens, seed=3)
    r = attention_varlen_i8f8(q, k, v, cu, cu, causal=causal, sm_scale=LN2)
    # the whole packed batch as one sequence with a block-diagonal mask
    qd = q.transpose(0, 1)[None]                 # [1, Hq, total, D]
    kd, vd = k.transpose(0, 1)[None], v.transpose(0, 1)[None]
    mask = block_diagonal_mask(cu, cu, causal=causal)
    ex, ex_lse = O.exact_attention(qd, kd, vd, sm_scale=LN2, mask=mask[None, None])
    np.testing.assert_allclose(r["out_f64"], np.transpose(ex[0], (1, 0, 2)), rtol=0, atol=1e-12)
    # LSE: one [Hq, len_s] block per sequence
    for s in range(len(lens)):
        blk = r["lse"][2 * cu[s]:2 * cu[s + 1]].reshape(2, lens[s])
        np.testing.assert_allclose(blk, ex_lse[0][:, cu[s]:cu[s + 1]], rtol=0, atol=1e-12)


def test_single_sequence_equals_dense_oracle():
    w = W.TINY.scaled(B=1, Hq=4, Hkv=2, N=300, D=64, seed=4)
    q, k, v = W.make_qkv(w)
    r = attention_varlen_i8f8(q[0].transpose(0, 1), k[0].transpose(0, 1), v[0].transpose(0, 1),
                              [0, 300], [0, 300], causal=True)
    d = O.attention_i8f8(O.quantize_qkv_i8f8(q, k, v), causal=True)
    np.testing.assert_array_equal(r["out"], np.transpose(d["out"][0], (1, 0, 2)))
    np.testing.assert_array_equal(r["lse"], d["lse"][0].reshape(-1))


def test_sequences_are_independent():
    """Changing one sequence's values changes none of the other outputs:
    no statistic (K mean, block scale, V scale) crosses a boundary."""
    w = W.TINY.scaled(B=1, Hq=2, Hkv=2, N=512, D=64, seed=5)
    q, k, v = W.make_qkv(w)
    pq, pk, pv = q[0].transpose(0, 1), k[0].transpose(0, 1), v[0].transpose(0, 1)
    cu = [0, 200, 512]
    a = attention_varlen_i8f8(pq, pk, pv, cu, cu)
    pk2, pv2 = pk.clone(), pv.clone()
    pk2[200:] *= 3                                # second sequence only
    pv2[200:] += 5
    b = attention_varlen_i8f8(pq, pk2, pv2, cu, cu)
    np.testing.assert_array_equal(a["out"][:200], b["out"][:200])
    assert not np.array_equal(a["out"][200:], b["out"][200:])


def test_empty_sequences():
    w = W.TINY.scaled(B=1, Hq=2, Hkv=2, N=256, D=64, seed=6)
    q, k, v = W.make_qkv(w)
    pq, pk, pv = q[0].transpose(0, 1), k[0].transpose(0, 1), v[0].transpose(0, 1)
    ref = attention_varlen_i8f8(pq, pk, pv, [0, 256], [0, 256])
    r = attention_varlen_i8f8(pq, pk, pv, [0, 0, 256, 256], [0, 0, 256, 256])
    np.testing.assert_array_equal(r["out"], ref["out"])
    # queries with no key at all: out 0, lse -inf
    r2 = attention_varlen_i8f8(pq[:10], pk[:0], pv[:0], [0, 10], [0, 0])
    assert np.all(r2["out"] == 0) and np.all(r2["lse"] == -np.inf)


def test_malformed_cu_seqlens_rejected():
    for cu in ([1, 5], [0, 3, 2, 5], [0, 4], [[0, 5]]):
        with pytest.raises(ValueError):
            check_cu_seqlens(cu, 5)
