"""Oracle of the merge of partial attention results over key shards.

TEST INFRASTRUCTURE ONLY (see the package header).

thu-ml/sageattention llms.txt, "Utilize SageAttention for Distributed
Inference" and the ``return_lse`` of "sageattn_qk_int8_pv_fp8_cuda": the
log-sum-exp of each row is returned so that results computed over separate
parts of the keys (sequence parallelism, ring attention) can be combined.
For a row with partial results (o_i, lse_i) over disjoint key sets,

    lse = log sum_i exp(lse_i),    o = sum_i exp(lse_i - lse) * o_i,

which is the attention over the union of the key sets.  A part whose row
saw no key has lse_i = -inf and weight 0; a row that sees no key in any
part keeps o = 0, lse = -inf.
"""
import numpy as np


def merge_partials(parts):
    """parts: list of (out [..., D], lse [...]) float arrays over disjoint
    key sets.  Returns (out, lse) in float64."""
    lses = np.stack([np.asarray(l, dtype=np.float64) for _, l in parts])    # [P, ...]
    outs = np.stack([np.asarray(o, dtype=np.float64) for o, _ in parts])    # [P, ..., D]
    m = lses.max(axis=0)
    ok = np.isfinite(m)
    m0 = np.where(ok, m, 0.0)
    w = np.where(np.isfinite(lses), np.exp(lses - m0[None]), 0.0)           # [P, ...]
    tot = w.sum(axis=0)
    lse = np.where(ok, m0 + np.log(np.where(ok, tot, 1.0)), -np.inf)
    out = np.where(ok[..., None],
                   (w[..., None] * outs).sum(axis=0) / np.where(ok, tot, 1.0)[..., None], 0.0)
    return out, lse


def merge_step(acc_out, acc_lse, out, lse):
    """One step of a running merge (the order a ring visits the shards):
    the merge of (acc_out, acc_lse) with (out, lse)."""
    return merge_partials([(acc_out, acc_lse), (out, lse)])
