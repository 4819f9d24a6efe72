"""Plain, slow CPU oracle of SageAttention-style quantised attention.

TEST INFRASTRUCTURE ONLY.  This package is the independent definition that
the CUDA path is checked against.  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py`` may import it.  The product package
(``quantized_attention_05_b200``) never imports it, and it shares no code,
constant table or helper with the CUDA sources.

Modules
-------
formats    fp32/bf16 rounding, exact means, FP8 E4M3 and FP4 E2M1 codecs.
quantize   the quantisation stage (smooth_k, per-block INT8 Q/K, per-channel
           FP8 V; NVFP4 with per-block Q mean and qk_correction).
attention  exact fp64 attention and the tile-ordered online-softmax
           attention over the quantised codes (INT8-QK/FP8-PV and NVFP4).
varlen     packed variable-length batches (cu_seqlens): every sequence its
           own dense problem.
merge      the LSE merge of partial results over key shards.

Every function states the passage of the SageAttention / FlashInfer pages it
follows.  Where the pages are silent the plainest reading is taken; those
readings are listed in the repository's design notes.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against closed forms, brute force on tiny inputs, lossless special cases,
library conversions and invariants.  The NVFP4 means (per 128-token Q block
over its valid rows, or global; K over the first ``unpadded_k_len`` keys)
are pinned against exact rational sums, and the NVFP4 quantisation of P
against vectors worked out by hand from the E2M1 and E4M3 grids.  The NVFP4
attention's tie bound (``attention_nvfp4(tie_band=...)``) is checked to hold
every output a perturbation of P' within the band produces.
"""
from .formats import (bf16_round, e2m1_decode, e2m1_encode, e2m1_round, e4m3_decode,  # noqa: F401
                      e4m3_encode, e4m3_round, exact_mean_f32, f32, fraction_to_f32,
                      pack_e2m1, unpack_e2m1)
from .quantize import (BLOCK, fp4_vector_quant, fp8_channel_quant, int8_block_quant,  # noqa: F401
                       quantize_qkv_i8f8, quantize_qkv_nvfp4)
from .attention import (attention_i8f8, attention_nvfp4, cosine, default_sm_scale,  # noqa: F401
                        exact_attention, qk_int32_tile)
from .varlen import attention_varlen_i8f8, block_diagonal_mask, check_cu_seqlens  # noqa: F401
from .merge import merge_partials, merge_step  # noqa: F401
