"""Seeded synthetic inputs for the quantized-attention path.

This module only draws random numbers and lays them out; it holds none of
the method's arithmetic (no quantisation, no softmax, no means).  Both the
CPU oracle side (tests, the bench's CPU baseline) and the CUDA side (tests,
bench, smoke) take their Q/K/V from here, so the two sides see identical
inputs.

The shapes and value distributions follow the workloads the SageAttention
pages use in their examples: LLM-shaped (B=2, H=32, N=8192, d=128) with a
boolean mask hiding the second half of the keys ("SageAttention Triton
INT8/FP16 Kernel Examples"), grouped-query attention with several Q heads per
KV head ("sageattn -- Auto-selecting attention kernel", 16 Q heads over 4 KV
heads), long video-DiT sequences, and the NVFP4 layout of
"flashinfer.nvfp4_attention_sm120_fwd" (padded K/V with ``unpadded_k_len``).

Recipe (all configs): a ``torch.Generator`` seeded with the config's seed
draws, in this order, fp32 ``randn`` for q, k, v, then a per-channel K
offset ``randn(B, Hkv, 1, D) * k_offset_std`` (one offset per channel shared
by every token: channel outliers), then the extras (V outlier positions).
Everything is rounded to bf16 (or fp16) at the end.  ``N(0, 4)`` in a config
description is read as variance 4, i.e. standard deviation 2.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    D: int
    seed: int
    causal: bool = False
    return_lse: bool = False
    k_offset_std: float = 0.0
    mask: str = "none"            # "none" | "second_half_keys"
    v_outlier_p: float = 0.0      # fraction of V entries scaled by v_outlier_scale
    v_outlier_scale: float = 1.0
    nvfp4: bool = False
    unpadded_k_len: Optional[int] = None   # K/V rows >= this are zero (NVFP4)
    per_block_mean: bool = True
    sm_scale: Optional[float] = None       # None -> 1/sqrt(D)

    @property
    def ops(self) -> float:
        """Nominal attention operations 4*B*Hq*N*N*D, halved for causal."""
        o = 4.0 * self.B * self.Hq * self.N * self.N * self.D
        return o / 2 if self.causal else o

    @property
    def visible_ops(self) -> float:
        """Operations on the (query, key) pairs the attention can see: ops,
        halved again when the mask hides the second half of the keys (the
        kernels skip key tiles a mask hides entirely)."""
        return self.ops / 2 if self.mask == "second_half_keys" else self.ops

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads.  Seed 0 is given for the tiny case; the others use 1..4.
TINY = Workload("tiny_b1_h2_n256_d64", B=1, Hq=2, Hkv=2, N=256, D=64, seed=0,
                k_offset_std=2.0, sm_scale=1.0 / 8.0)
LLM_MASK = Workload("llm_mask_b2_h32_n8192_d128", B=2, Hq=32, Hkv=32, N=8192, D=128,
                    seed=1, k_offset_std=2.0, mask="second_half_keys", return_lse=True)
CAUSAL_GQA = Workload("causal_gqa_b4_hq32_hkv8_n16384_d128", B=4, Hq=32, Hkv=8, N=16384,
                      D=128, seed=2, k_offset_std=2.0, causal=True, return_lse=True)
VIDEO_DIT = Workload("video_dit_b1_h24_n32768_d128", B=1, Hq=24, Hkv=24, N=32768, D=128,
                     seed=3, k_offset_std=3.0, v_outlier_p=0.01, v_outlier_scale=20.0)
NVFP4 = Workload("nvfp4_b1_h32_n16384_d128", B=1, Hq=32, Hkv=32, N=16384, D=128, seed=4,
                 nvfp4=True, unpadded_k_len=16000, per_block_mean=True, return_lse=True)

ALL = [TINY, LLM_MASK, CAUSAL_GQA, VIDEO_DIT, NVFP4]
BY_NAME = {w.name: w for w in ALL}


def make_qkv(w: Workload, device="cpu", dtype=torch.bfloat16, layout="HND"):
    """Draw (q, k, v) for workload ``w``.

    Returns tensors of logical shape (B, H, N, D).  With layout "NHD" the
    memory is (B, N, H, D) and the returned tensor is a permuted view of it,
    so its strides are those of an NHD tensor.  Values are drawn in
    fp32 on ``device`` with a generator seeded by ``w.seed`` and rounded to
    ``dtype`` at the end.  CPU and CUDA generators give different streams;
    parity tests draw on the CPU.
    """
    g = torch.Generator(device=device)
    g.manual_seed(w.seed)
    f32 = torch.float32
    q = torch.randn(w.B, w.Hq, w.N, w.D, generator=g, device=device, dtype=f32)
    k = torch.randn(w.B, w.Hkv, w.N, w.D, generator=g, device=device, dtype=f32)
    v = torch.randn(w.B, w.Hkv, w.N, w.D, generator=g, device=device, dtype=f32)
    if w.k_offset_std:
        off = torch.randn(w.B, w.Hkv, 1, w.D, generator=g, device=device, dtype=f32)
        k += off * w.k_offset_std
    if w.v_outlier_p:
        sel = torch.rand(w.B, w.Hkv, w.N, w.D, generator=g, device=device, dtype=f32) < w.v_outlier_p
        v = torch.where(sel, v * w.v_outlier_scale, v)
    if w.unpadded_k_len is not None and w.unpadded_k_len < w.N:
        k[:, :, w.unpadded_k_len:, :] = 0
        v[:, :, w.unpadded_k_len:, :] = 0
    q, k, v = q.to(dtype), k.to(dtype), v.to(dtype)
    if layout == "NHD":
        q, k, v = (t.transpose(1, 2).contiguous().transpose(1, 2) for t in (q, k, v))
    return q, k, v


def make_mask(w: Workload, device="cpu"):
    """Boolean key mask (True = attend), shape (B, 1, N, N), or None.

    "second_half_keys" hides keys N//2.. for every query, as in the pages'
    Triton example.
    """
    if w.mask == "none":
        return None
    if w.mask == "second_half_keys":
        m = torch.ones(w.B, 1, w.N, w.N, dtype=torch.bool, device=device)
        m[:, :, :, w.N // 2:] = False
        return m
    raise ValueError(w.mask)


def sample_rows(w: Workload, n_random=256, seed=1234):
    """Deterministic query-row sample for full-size attention parity.

    Rows 0..127, the last 128 rows, and ``n_random`` seeded random rows.
    """
    g = torch.Generator().manual_seed(seed + w.seed)
    head = list(range(min(128, w.N)))
    tail = list(range(max(0, w.N - 128), w.N))
    rnd = torch.randint(0, w.N, (n_random,), generator=g).tolist()
    return sorted(set(head + tail + rnd))


def random_integer_tensor(shape, low, high, seed):
    """Uniform integers in [low, high] as float64 (for the oracle's lossless cases)."""
    g = torch.Generator().manual_seed(seed)
    return torch.randint(low, high + 1, shape, generator=g).to(torch.float64)
