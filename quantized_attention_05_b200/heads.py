"""Head parallelism: the KV-head groups of one call split over the ranks of
a torch.distributed group.

Every KV head together with its G = Hq/Hkv query heads is a problem of its
own. It has its own K mean, V channel scales and Q blocks (thu-ml/sageattention
llms.txt, "sageattn -- Auto-selecting attention kernel": GQA, the query heads of
a group share one KV head). So rank r computes a contiguous range of KV heads
with no exchange, and a head's result does not depend on the rank that
computed it.

With ``gather`` the ranks all-gather out and LSE: one collective over the
group's backend, NCCL over NVLink for CUDA tensors. Without it, each rank keeps
its own heads.
"""
from typing import Callable, Optional, Tuple

import torch
import torch.distributed as dist


def kv_head_range(Hkv: int, rank: int, world: int) -> Tuple[int, int]:
    """The contiguous KV heads [g0, g1) of ``rank``.

    The first Hkv % world ranks take one head more than the others. A rank
    beyond Hkv - 1 gets an empty range."""
    base, extra = divmod(Hkv, world)
    g0 = rank * base + min(rank, extra)
    return g0, g0 + base + (1 if rank < extra else 0)


def _gpu_attn(q, k, v, causal, sm_scale):
    from . import sage_attn_fwd
    return sage_attn_fwd(q, k, v, causal=causal, sm_scale=sm_scale, return_lse=True)


def shard_heads(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, rank: int, world: int):
    """This rank's slice of full q [B, Hq, N, D] and k, v [B, Hkv, Nk, D]:
    KV heads ``kv_head_range(Hkv, rank, world)`` and their query heads (views,
    no copy).  A loader that places only these heads on the rank's GPU passes
    the same slices to ``head_parallel_attention(..., heads=(Hq, Hkv))``."""
    Hq, Hkv = q.shape[1], k.shape[1]
    G = Hq // Hkv
    g0, g1 = kv_head_range(Hkv, rank, world)
    return q[:, g0 * G:g1 * G], k[:, g0:g1], v[:, g0:g1]


def head_parallel_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, group=None,
                            causal: bool = False, sm_scale: Optional[float] = None,
                            gather: bool = True, attn: Optional[Callable] = None,
                            heads: Optional[Tuple[int, int]] = None):
    """Attention over all heads, with the KV-head groups split across the ranks.

    Without ``heads``, q: [B, Hq, N, D] and k, v: [B, Hkv, Nk, D] are the full
    tensors on every rank (HND layout), and rank r attends KV heads
    ``kv_head_range(Hkv, r, W)`` and their query heads.

    With ``heads=(Hq, Hkv)`` (the totals), each rank passes only its own slice
    (``shard_heads``): q [B, (g1-g0)*G, N, D], k, v [B, g1-g0, Nk, D] for
    (g0, g1) = kv_head_range(Hkv, r, W), possibly empty.  No rank then holds
    or moves more than its share of the inputs.

    With ``gather``, returns the full (out [B, Hq, N, D], lse [B, Hq, N]) on every
    rank. Without it, returns (out, lse, (h0, h1)): this rank's query heads
    h0..h1-1 only.

    ``attn(q, k, v, causal, sm_scale) -> (out, lse)`` defaults to the CUDA
    path. Tests on CPU ranks pass their own."""
    W = dist.get_world_size(group)
    r = dist.get_rank(group)
    attn = attn or _gpu_attn
    B, _, N, D = q.shape
    if heads is None:
        Hq, Hkv = q.shape[1], k.shape[1]
    else:
        Hq, Hkv = int(heads[0]), int(heads[1])
    if Hkv <= 0 or Hq % Hkv:
        raise ValueError("the query heads must be a multiple of the KV heads")
    G = Hq // Hkv
    # the library's LSE is fp32; fp64 inputs (CPU test ranks) keep fp64
    lse_dtype = torch.float64 if q.dtype == torch.float64 else torch.float32
    g0, g1 = kv_head_range(Hkv, r, W)
    h0, h1 = g0 * G, g1 * G
    if heads is None:
        q, k, v = q[:, h0:h1], k[:, g0:g1], v[:, g0:g1]
    elif q.shape[1] != h1 - h0 or k.shape[1] != g1 - g0 or v.shape[1] != g1 - g0:
        raise ValueError(f"rank {r} of {W}: expected the slices of query heads [{h0}, {h1}) and "
                         f"KV heads [{g0}, {g1}), got {q.shape[1]} and {k.shape[1]} heads")
    if g1 > g0:
        out, lse = attn(q, k, v, causal, sm_scale)
    else:
        out = q.new_empty(B, 0, N, D)
        lse = torch.empty(B, 0, N, dtype=lse_dtype, device=q.device)
    if not gather:
        return out, lse, (h0, h1)
    # equal-sized pieces for the collective: every rank pads its heads to the
    # largest share
    hmax = -(-Hkv // W) * G
    out_p = q.new_zeros(B, hmax, N, D)
    lse_p = torch.zeros(B, hmax, N, dtype=lse_dtype, device=q.device)
    out_p[:, :h1 - h0] = out
    lse_p[:, :h1 - h0] = lse
    outs = [torch.empty_like(out_p) for _ in range(W)]
    lses = [torch.empty_like(lse_p) for _ in range(W)]
    dist.all_gather(outs, out_p, group=group)
    dist.all_gather(lses, lse_p, group=group)
    full_out = q.new_empty(B, Hq, N, D)
    full_lse = torch.empty(B, Hq, N, dtype=lse_dtype, device=q.device)
    for rr in range(W):
        a0, a1 = kv_head_range(Hkv, rr, W)
        if a1 > a0:
            full_out[:, a0 * G:a1 * G] = outs[rr][:, :(a1 - a0) * G]
            full_lse[:, a0 * G:a1 * G] = lses[rr][:, :(a1 - a0) * G]
    return full_out, full_lse
