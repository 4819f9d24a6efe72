"""Sequence parallelism over key shards ("ring attention") with the LSE merge.

thu-ml/sageattention llms.txt, "Utilize SageAttention for Distributed
Inference": results computed over separate parts of the keys are combined
through the returned log-sum-exp.  Here the sequence is split into W
chunks, one per rank of a torch.distributed group (chunk r on rank r, for
queries and keys alike).  At step t rank r attends its query chunk to key
chunk j = (r - t) mod W while that chunk travels on to rank r + 1
(point-to-point over the group's backend: NCCL over NVLink for CUDA
tensors), and merges the partial result into its running one.  With causal
attention, chunk j > r is fully masked and skipped, chunk j == r is the
causal diagonal block and chunks j < r are fully visible.  Every rank
takes the same W - 1 exchange steps.

Each step quantises its own key chunk (its own K mean and blocks); the
merge through the LSE of the unsmoothed scores is exact, so the result is
the merge of per-chunk quantised attention.
"""
from typing import Callable, Optional

import torch
import torch.distributed as dist


def _gpu_attn(q, k, v, causal, sm_scale):
    from . import sage_attn_fwd
    return sage_attn_fwd(q, k, v, causal=causal, sm_scale=sm_scale, return_lse=True)


class _GpuMerge:
    """Running fp32 merge on the device (sage_lse_merge)."""

    def __init__(self, like: torch.Tensor):
        B, H, N, D = like.shape
        self.acc = torch.zeros(B, H, N, D, dtype=torch.float32, device=like.device)
        self.lse = torch.full((B, H, N), float("-inf"), dtype=torch.float32, device=like.device)
        self.first = True

    def add(self, out, lse):
        from . import sage_lse_merge
        sage_lse_merge(self.acc, self.lse, out, lse, init=self.first)
        self.first = False

    def result(self, out):
        from . import sage_lse_merge_finalize
        return sage_lse_merge_finalize(self.acc, out), self.lse


def ring_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, group=None,
                   causal: bool = False, sm_scale: Optional[float] = None,
                   attn: Optional[Callable] = None, merger: Optional[Callable] = None):
    """Attention of this rank's query chunk over the whole sequence.

    q: [B, Hq, Nc, D] (chunk ``rank`` of the queries), k/v: [B, Hkv, Nc, D]
    (chunk ``rank`` of the keys), all ranks with the same chunk length.
    Returns (out [B, Hq, Nc, D] in q's dtype, lse [B, Hq, Nc]).
    ``attn(q, k, v, causal, sm_scale) -> (out, lse)`` and ``merger(like)``
    (an object with ``add(out, lse)`` and ``result(out)``) default to the
    CUDA path; tests on CPU ranks pass their own.
    """
    W = dist.get_world_size(group)
    r = dist.get_rank(group)
    attn = attn or _gpu_attn
    merge = (merger or _GpuMerge)(q)
    nxt, prv = (r + 1) % W, (r - 1) % W
    g_nxt = dist.get_global_rank(group, nxt) if group is not None else nxt
    g_prv = dist.get_global_rank(group, prv) if group is not None else prv
    k_cur, v_cur = k.contiguous(), v.contiguous()
    for t in range(W):
        j = (r - t) % W
        reqs = []
        if t < W - 1:
            k_nxt, v_nxt = torch.empty_like(k_cur), torch.empty_like(v_cur)
            ops = [dist.P2POp(dist.isend, k_cur, g_nxt, group), dist.P2POp(dist.isend, v_cur, g_nxt, group),
                   dist.P2POp(dist.irecv, k_nxt, g_prv, group), dist.P2POp(dist.irecv, v_nxt, g_prv, group)]
            reqs = dist.batch_isend_irecv(ops)
        if not (causal and j > r):
            out_j, lse_j = attn(q, k_cur, v_cur, causal and j == r, sm_scale)
            merge.add(out_j, lse_j)
        for req in reqs:
            req.wait()
        if t < W - 1:
            k_cur, v_cur = k_nxt, v_nxt
    return merge.result(torch.empty_like(q))
