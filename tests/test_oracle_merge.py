"""Pins for oracle/merge.py: merging exact attention over key shards must
give exact attention over all keys (the identity behind the pages' use of
return_lse for distributed inference), in any shard order and step by step;
empty shards and rows that see no key in some shard."""
import numpy as np
import pytest

import oracle as O
from oracle.merge import merge_partials, merge_step
import workloads as W


def _shards(Nk, cuts):
    edges = [0] + list(cuts) + [Nk]
    return [(edges[i], edges[i + 1]) for i in range(len(edges) - 1)]


@pytest.mark.parametrize("cuts", [[128], [100, 300], [1, 2, 511]])
def test_merge_of_shards_equals_full_attention(cuts):
    w = W.TINY.scaled(B=1, Hq=2, Hkv=2, N=512, D=64, seed=41)
    q, k, v = W.make_qkv(w)
    full, full_lse = O.exact_attention(q, k, v)
    parts = []
    for a, b in _shards(512, cuts):
        parts.append(O.exact_attention(q, k[:, :, a:b], v[:, :, a:b]))
    out, lse = merge_partials(parts)
    np.testing.assert_allclose(out, full, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, full_lse, rtol=0, atol=1e-12)
    # the same result step by step, in reverse shard order
    acc_o, acc_l = parts[-1]
    for o, l in reversed(parts[:-1]):
        acc_o, acc_l = merge_step(acc_o, acc_l, o, l)
    np.testing.assert_allclose(acc_o, full, rtol=0, atol=1e-12)
    np.testing.assert_allclose(acc_l, full_lse, rtol=0, atol=1e-12)


def test_merge_with_causal_shards_and_unseen_rows():
    """Causal attention split over key shards: early rows see nothing in
    later shards (lse -inf there) and the merge still equals the full
    causal attention."""
    w = W.TINY.scaled(B=1, Hq=2, Hkv=1, N=384, D=64, seed=42)
    q, k, v = W.make_qkv(w)
    full, full_lse = O.exact_attention(q, k, v, causal=True)
    parts = []
    for a, b in _shards(384, [128, 256]):
        mask = np.zeros((384, 384), bool)
        mask[:, a:b] = np.tril(np.ones((384, 384), bool))[:, a:b]
        parts.append(O.exact_attention(q, k, v, mask=mask[None, None]))
    assert np.any(np.isneginf(parts[2][1]))            # rows that see no key of the last shard
    out, lse = merge_partials(parts)
    np.testing.assert_allclose(out, full, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, full_lse, rtol=0, atol=1e-12)


def test_merge_all_empty_rows():
    o = np.zeros((3, 4))
    l = np.full(3, -np.inf)
    out, lse = merge_partials([(o, l), (o, l)])
    assert np.all(out == 0) and np.all(np.isneginf(lse))
