/*
 * sage_b200.h -- C ABI of the B200 (sm_100a) SageAttention-style quantised
 * attention forward.
 *
 * The operation (thu-ml/sageattention llms.txt):
 *   "sageattn_qk_int8_pv_fp16_triton": per-block INT8 quantisation of Q and
 *     K, optional K smoothing ("smooth_k"), boolean attention mask
 *     broadcastable to [batch, heads, q_len, k_len] (True = attend), LSE.
 *   "sageattn_qk_int8_pv_fp8_cuda" / "sageattn_qk_int8_pv_fp8_cuda_sm90":
 *     INT8 Q/K with per-channel FP8 V, PV accumulated in FP32, causal mask,
 *     LSE of shape [batch, heads, seq].
 *   "sageattn -- Auto-selecting attention kernel": FP16/BF16 inputs in HND
 *     or NHD layout, group-query attention (several Q heads per KV head),
 *     sm_scale defaulting to 1/sqrt(head_dim).
 *
 * What each call computes, precisely:
 *   quantise:  kmean[b,g,c] = mean over tokens of K (exact, rounded once to
 *              fp32; zero when smooth_k == 0); Ks = fp32(K - kmean);
 *              per 128-token block of Q (resp. Ks), a = max|x|,
 *              scale = fp32(a/127), code = clamp(rint(fp32(x * fp32(127/a))), +-127);
 *              per V channel over all tokens, a = max|v|, vscale = fp32(a/448),
 *              code = e4m3_rn_satfinite(fp32(v * fp32(448/a))), stored transposed;
 *              q_dot_kmean[b,h,n] = sum_c q[b,h,n,c] * kmean[b,h/G,c].
 *   attention: s = S_int * q_scale * k_scale * sm_scale with S_int the exact
 *              int32 dot product of the codes; online softmax over 128-key
 *              tiles; P8 = e4m3(448 * exp(s - running_max)); O += P8 . V8 in
 *              FP32; out = O * vscale / (448 * l), l the sum of the
 *              unquantised probabilities; lse = natural-log LSE of the
 *              unsmoothed scores (smoothed LSE + sm_scale * q_dot_kmean).
 *   A query row with no visible key gives out = 0 and lse = -inf.
 *
 * Conventions (all entry points):
 *   - Every pointer argument named as device memory must point to memory
 *     of the device that is current on the calling thread; host pointers
 *     are the descriptor structs themselves and the tensors of
 *     sage_attn_fwd_host, whose arguments say which side each is on.  The library never
 *     allocates device memory: the caller owns every buffer, including the
 *     workspace, whose size the matching *_workspace_bytes query returns.
 *   - Work is enqueued asynchronously on `stream` (NULL = legacy default
 *     stream); the call returns after enqueueing.  Argument errors are
 *     detected on the host before anything is enqueued.
 *   - Errors: SAGE_ERR_INVALID_ARG (malformed argument, including a tensor
 *     with more than 65536 batch entries or 4096 heads), SAGE_ERR_UNSUPPORTED
 *     (valid but outside what the kernels handle: head_dim not in {64,128},
 *     more than 262144 tokens in a sequence, more than 65535 (batch entry, Q
 *     head) pairs in one device call -- (sequence, KV head) pairs for
 *     sage_attn_fwd_varlen; the *_host calls work a chunk at a time and are
 *     not bound by this -- or 2^31 or more padded rows in one tensor),
 *     SAGE_ERR_WORKSPACE (workspace too small), SAGE_ERR_CUDA (a CUDA call
 *     failed at launch).  Device-side failures (a bounded wait that
 *     ran out) set a device status word read by sage_get_device_status.
 *   - The calls are thread-safe.  Calls that share a workspace or outputs
 *     must be ordered by the caller (same stream or events).  Library state:
 *     the kernels' shared-memory opt-ins (set once) and, for
 *     sage_attn_fwd_host, two copy streams and a few events per device,
 *     created on first use and kept for the life of the process.
 */
#ifndef SAGE_B200_H
#define SAGE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* sage_stream_t; /* identical to cudaStream_t */

typedef enum {
  SAGE_OK = 0,
  SAGE_ERR_INVALID_ARG = 1,
  SAGE_ERR_UNSUPPORTED = 2,
  SAGE_ERR_WORKSPACE = 3,
  SAGE_ERR_CUDA = 4,
  SAGE_ERR_TIMEOUT = 5
} sage_status;

/* Input element types: the pages take FP16/BF16 Q/K/V ("SageAttention
 * Usage" notes). */
typedef enum { SAGE_BF16 = 0, SAGE_FP16 = 1 } sage_dtype;

/* A strided 4-D input tensor of logical shape [B, H, N, D].
 * ptr: device pointer to element [0,0,0,0], 16-byte aligned.
 * sb, sh, sn: element strides of the batch, head and token dimensions; the
 * channel stride is 1.  HND layout has sn = D, sh = N*D; NHD layout has
 * sn = H*D, sh = D ("tensor_layout" of the sageattn API).  sn must be a
 * multiple of 8 elements (16-byte rows). */
typedef struct {
  const void* ptr;
  int32_t dtype; /* sage_dtype */
  int64_t B, H, N, D;
  int64_t sb, sh, sn;
} sage_tensor;

/* Attention mask ("sageattn_qk_int8_pv_fp16_triton": an optional boolean or
 * float32 attention mask broadcastable to [batch, heads, q_len, k_len]).
 *   kind SAGE_MASK_BOOL: one byte per element, nonzero = attend
 *     ("mask[..., seq_len // 2:] = False  # mask out second half of keys");
 *   kind SAGE_MASK_FLOAT: fp32 added to the scaled scores (natural-log
 *     units, as a float attention mask adds to q.k^T * sm_scale); -inf hides
 *     a key; +inf and NaN are not allowed.  4-byte aligned.
 * Logical shape [B, H, Nq, Nk] broadcast over batch and heads: B is 1 or the
 * attention's batch, H is 1 or the number of Q heads.  sb, sh, sq: strides
 * in elements (ignored for a broadcast dimension of size 1); the key stride
 * is 1.  Device memory, owned by the caller, read-only. */
typedef enum { SAGE_MASK_BOOL = 0, SAGE_MASK_FLOAT = 1 } sage_mask_kind;
typedef struct {
  const void* ptr;
  int64_t B, H, Nq, Nk;
  int64_t sb, sh, sq;
  int32_t kind; /* sage_mask_kind */
} sage_mask;

/* Quantised Q/K/V of the INT8/FP8 path, all device memory owned by the
 * caller.  Nq_pad = ceil(Nq/128)*128, Nk_pad = ceil(Nk/128)*128; every
 * array is dense in the order given.  V keeps its own [token, channel]
 * order: the PV product reads each 128-token tile as an MN-major operand,
 * so no transposition is needed.
 *   q        int8  [B, Hq,  Nq_pad, D]   codes; rows >= Nq are 0
 *   q_scale  fp32  [B, Hq,  Nq_pad/128]  one scale per 128-token block
 *   k        int8  [B, Hkv, Nk_pad, D]   codes of K - kmean; rows >= Nk are 0
 *   k_scale  fp32  [B, Hkv, Nk_pad/128]
 *   k_mean   fp32  [B, Hkv, D]
 *   v        e4m3  [B, Hkv, Nk_pad, D]   V codes; rows >= Nk are 0
 *   v_scale  fp32  [B, Hkv, D]
 *   q_dot_kmean fp32 [B, Hq, Nq]  (may be NULL when no LSE is wanted)
 * The base pointers of q, k and v must be 16-byte aligned. */
typedef struct {
  int8_t* q;
  float* q_scale;
  int8_t* k;
  float* k_scale;
  float* k_mean;
  uint8_t* v;
  float* v_scale;
  float* q_dot_kmean;
  int64_t B, Hq, Hkv, Nq, Nk, D;
} sage_qkv_i8f8;

/* Quantised Q/K/V of the NVFP4 path ("flashinfer.nvfp4_attention_sm120_fwd":
 * packed FP4 Q/K/V with per-vector FP8 scale factors, V and its scales
 * stored transposed, a compact FP32 qk_correction with one row per 128-token
 * Q block, per_block_mean, unpadded_k_len).  Device memory owned by the
 * caller; Nq_pad / Nk_pad as for sage_qkv_i8f8; every array dense.
 *   q        u8   [B, Hq,  Nq_pad, D/2]  E2M1 codes, element 2i in the low nibble
 *   q_sf     u8   [B, Hq,  Nq_pad, D/16] E4M3 scale of each 16-element vector
 *   k        u8   [B, Hkv, Nk_pad, D/2]  codes of K - kmean (rows >= unpadded_k_len: 0)
 *   k_sf     u8   [B, Hkv, Nk_pad, D/16]
 *   v_t      u8   [B, Hkv, D, Nk_pad/2]  V transposed, 16-token vectors
 *   v_sf_t   u8   [B, Hkv, D, Nk_pad/16]
 *   qk_correction fp32 [B, Hq, Nq_pad/128, Nk_pad]: qmean(block) . Ks[j]
 *   q_mean   fp32 [B, Hq, Nq_pad/128, D]: the mean removed from each Q block
 *                 (the same vector in every block when per_block_mean == 0)
 *   k_mean   fp32 [B, Hkv, D]
 *   q_dot_kmean fp32 [B, Hq, Nq] (may be NULL when no LSE is wanted)
 * The base pointers of q, k, v_t, qk_correction and q_mean must be 16-byte
 * aligned. */
typedef struct {
  uint8_t* q;
  uint8_t* q_sf;
  uint8_t* k;
  uint8_t* k_sf;
  uint8_t* v_t;
  uint8_t* v_sf_t;
  float* qk_correction;
  float* q_mean;
  float* k_mean;
  float* q_dot_kmean;
  int64_t B, Hq, Hkv, Nq, Nk, D;
  int64_t unpadded_k_len;
  int32_t per_block_mean;
} sage_qkv_nvfp4;

/* ------------------------------------------------------------------ info */
/* A static, human-readable name of a status code ("unknown status" for a
 * value outside the enum).  Never NULL; the caller does not free it. */
const char* sage_status_str(sage_status status);
/* A static string naming the library and its target (sm_100a).  Never NULL. */
const char* sage_version(void);

/* Device status word: synchronises `stream`, returns SAGE_ERR_TIMEOUT if a
 * kernel of this library gave up a bounded wait since the last call (the
 * wait site is written to *site when site != NULL), SAGE_ERR_CUDA if the
 * stream reports an error, SAGE_OK otherwise, and clears the word. */
sage_status sage_get_device_status(sage_stream_t stream, uint32_t* site);

/* ----------------------------------------------------------- quantisation */
/* Workspace bytes sage_quantize_qkv needs for these sizes (per-split K sums
 * and V maxima of the reduction pass). */
size_t sage_quantize_workspace_bytes(int64_t B, int64_t Hkv, int64_t Nk, int64_t D);

/* Quantisation stage: smooth_k + per-block INT8 Q/K, per-channel FP8 V
 * (pages: "smooth_k", per-block INT8 QK, per-channel FP8 V).  q: [B, Hq, Nq, D]; k, v: [B, Hkv, Nk, D] (same dtype,
 * Hq % Hkv == 0, D in {64, 128}).  Writes every array of *out (whose shape
 * fields must match the inputs).  ws: device workspace of at least
 * sage_quantize_workspace_bytes(B, Hkv, Nk, D) bytes, 256-byte aligned. */
sage_status sage_quantize_qkv(const sage_tensor* q, const sage_tensor* k, const sage_tensor* v,
                              int smooth_k, const sage_qkv_i8f8* out, void* ws, size_t ws_bytes,
                              sage_stream_t stream);

/* --------------------------------------------------------------- attention */
/* Workspace bytes of sage_attn_fwd_quantized: the per-tile mask
 * classification (zero when mask == NULL). */
size_t sage_attn_quantized_workspace_bytes(const sage_qkv_i8f8* qkv, const sage_mask* mask);

/* Fused attention on quantised inputs (the second stage of the path:
 * INT8 QK^T, dequantise, online softmax, P -> FP8, FP8 PV with FP32
 * accumulation).
 *   causal:   keep key j for query i when j <= i + Nk - Nq.
 *   sm_scale: softmax scale; <= 0 selects 1/sqrt(D).
 *   mask:     NULL or a boolean mask (see sage_mask).
 *   out:      device, q's logical shape [B, Hq, Nq, D], element type
 *             out_dtype (sage_dtype), element strides out_sb/out_sh/out_sn
 *             (channel stride 1; 16-byte aligned rows).
 *   lse:      device fp32 [B, Hq, Nq], written iff return_lse (then
 *             q_dot_kmean must be non-NULL); NULL otherwise.
 *   ws:       device workspace of sage_attn_quantized_workspace_bytes bytes. */
sage_status sage_attn_fwd_quantized(const sage_qkv_i8f8* qkv, int causal, float sm_scale,
                                    int return_lse, const sage_mask* mask, void* out,
                                    int32_t out_dtype, int64_t out_sb, int64_t out_sh,
                                    int64_t out_sn, float* lse, void* ws, size_t ws_bytes,
                                    sage_stream_t stream);

/* Workspace bytes of sage_attn_fwd: the quantised Q/K/V plus the two
 * workspaces above. */
size_t sage_attn_fwd_workspace_bytes(int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq,
                                     int64_t Nk, int64_t D, const sage_mask* mask);

/* The whole path on FP16/BF16 inputs (q, k, v, causal, sm_scale,
 * num_kv_heads, return_lse; pages: "sageattn").
 * num_kv_heads must equal k->H.  smooth_k as in sage_quantize_qkv (the
 * pages' default is on).  out has q's dtype; the other arguments are those
 * of sage_attn_fwd_quantized.  Quantises into the workspace, then attends.
 * A call without queries (q->B == 0 or q->N == 0) has nothing to compute: its
 * sizes are checked (one dtype, matching batch, Hq % Hkv == 0, k and v of one
 * length, D 64 or 128, num_kv_heads == k->H), no pointer is looked at, and it
 * returns SAGE_OK without enqueuing anything.  Keys are required otherwise:
 * k->N == 0 with queries present is SAGE_ERR_INVALID_ARG. */
sage_status sage_attn_fwd(const sage_tensor* q, const sage_tensor* k, const sage_tensor* v,
                          int causal, float sm_scale, int num_kv_heads, int return_lse,
                          int smooth_k, const sage_mask* mask, void* out, int64_t out_sb,
                          int64_t out_sh, int64_t out_sn, float* lse, void* ws,
                          size_t ws_bytes, sage_stream_t stream);

/* ------------------------------------------------------- host-resident inputs */
/* Workspace bytes of sage_attn_fwd_host for chunks of `chunk_groups` (batch
 * entry, KV head) groups (0 = automatic: about 100 MB of inputs per chunk,
 * with a single group in the call's first and last chunks, which shortens
 * the copy before the first kernel and the work after the last copy):
 * three staging slots, each holding one chunk's Q/K/V, output and LSE, plus
 * the quantise + attend workspace of one chunk.  mask as for the call (only
 * its B and H matter).  0 for invalid sizes. */
size_t sage_attn_fwd_host_workspace_bytes(int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq,
                                          int64_t Nk, int64_t D, const sage_mask* mask,
                                          int64_t chunk_groups);

/* sage_attn_fwd for Q/K/V and outputs held in HOST memory ("sageattn" with
 * tensors that live on the host): the same arguments and results as
 * sage_attn_fwd, with these differences.
 *   q, k, v:  HOST tensors (sage_tensor ptr is a host address; same shapes,
 *             strides and alignment rules as sage_attn_fwd; q, k and v share
 *             the dtype);
 *   out, lse: HOST buffers, out with element strides (out_sb, out_sh, out_sn),
 *             lse [B, Hq, Nq] contiguous fp32 (written iff return_lse);
 *   mask:     DEVICE memory, as in sage_attn_fwd (or NULL);
 *   chunk_groups: (batch entry, KV head) groups per chunk, 0 = automatic;
 *   ws:       DEVICE workspace (256-byte aligned) of
 *             sage_attn_fwd_host_workspace_bytes(..., chunk_groups) bytes.
 * The problem is streamed through the GPU a chunk at a time.  Each group is a
 * problem of its own (its K mean, V channel scales and Q blocks), so the
 * result equals sage_attn_fwd's bit for bit.  The copies of later and
 * earlier chunks run on two library-owned streams, overlapped with the
 * kernels of the current chunk, which run on `stream`; `stream` waits for
 * every copy before it proceeds, so an event recorded on `stream` after the
 * call completes after the last byte has reached `out` and `lse`.
 * The host buffers must stay valid and unmodified until then.  Page-locked
 * host memory is needed for the copies to overlap; pageable memory gives the
 * same result with the copies serialised by the driver.  Concurrent calls are
 * serialised while they enqueue (the copy streams are shared per device).
 * On SAGE_ERR_CUDA, work already enqueued still runs and `stream` still waits
 * for it; out and lse are then undefined.  A call without queries returns as
 * sage_attn_fwd's does. */
sage_status sage_attn_fwd_host(const sage_tensor* q, const sage_tensor* k, const sage_tensor* v,
                               int causal, float sm_scale, int num_kv_heads, int return_lse,
                               int smooth_k, const sage_mask* mask, void* out, int64_t out_sb,
                               int64_t out_sh, int64_t out_sn, float* lse, int64_t chunk_groups,
                               void* ws, size_t ws_bytes, sage_stream_t stream);

/* Workspace bytes of sage_attn_fwd_nvfp4_host for chunks of `chunk_groups`
 * (batch entry, KV head) groups (0 = automatic: about 25 MB of inputs per
 * chunk, single-group first and last chunks as for sage_attn_fwd_host):
 * three staging slots plus the largest chunk's quantised NVFP4 arrays and
 * quantiser sums.  0 for invalid sizes. */
size_t sage_attn_fwd_nvfp4_host_workspace_bytes(int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq,
                                                int64_t Nk, int64_t D, int64_t chunk_groups);

/* The NVFP4 path (sage_quantize_qkv_nvfp4 then sage_attn_fwd_nvfp4) on Q/K/V
 * and outputs held in HOST memory, streamed through the GPU a chunk of (batch
 * entry, KV head) groups at a time exactly as sage_attn_fwd_host does; every
 * group is a problem of its own (its K mean over the first unpadded_k_len
 * keys, its Q means, its V vectors), so the result equals the two device calls
 * bit for bit.  q, k, v: HOST tensors of one dtype; out, lse: HOST buffers (out
 * with element strides out_sb/out_sh/out_sn, lse [B, Hq, Nq] contiguous fp32,
 * written iff return_lse); unpadded_k_len <= 0 means Nk; sm_scale <= 0
 * selects 1/sqrt(D); ws: DEVICE workspace (256-byte aligned) of
 * sage_attn_fwd_nvfp4_host_workspace_bytes(..., chunk_groups) bytes.  Streams,
 * ordering, host-memory kinds, errors and calls without queries as for
 * sage_attn_fwd_host (unpadded_k_len must still not exceed k->N). */
sage_status sage_attn_fwd_nvfp4_host(const sage_tensor* q, const sage_tensor* k,
                                     const sage_tensor* v, float sm_scale, int causal,
                                     int per_block_mean, int64_t unpadded_k_len, int return_lse,
                                     void* out, int64_t out_sb, int64_t out_sh, int64_t out_sn,
                                     float* lse, int64_t chunk_groups, void* ws, size_t ws_bytes,
                                     sage_stream_t stream);

/* --------------------------------------------------------- variable length */
/* Workspace bytes of sage_attn_fwd_varlen: the sequence table, quantised
 * Q/K/V of the packed sequences (each padded to 128 tokens per head), the
 * quantiser's reductions and, with return_lse, q.kmean.  0 for invalid
 * sizes. */
size_t sage_attn_fwd_varlen_workspace_bytes(int64_t nseq, int64_t Hq, int64_t Hkv,
                                            int64_t total_q, int64_t total_k,
                                            int64_t max_seqlen_q, int64_t max_seqlen_k,
                                            int64_t D, int return_lse);

/* Attention over a batch of variable-length sequences packed into flat
 * tensors (pages: "sageattn_varlen": packed q/k/v, cumulative length
 * arrays cu_seqlens_q/k starting at 0, max_seqlen_q/k, is_causal,
 * smooth_k; INT8 QK with per-block scales).  Every sequence is its own
 * problem: its own K mean, 128-token quantisation blocks from its first
 * token, per-channel V scales, and bottom-right causal alignment.
 *   q:        [total_q, Hq, D] as a sage_tensor with B = 1, N = total_q (any
 *             token / head strides, channel stride 1, 16-byte aligned);
 *   k, v:     [total_k, Hkv, D] likewise, q's dtype, Hq % Hkv == 0;
 *   cu_seqlens_q/k: DEVICE int32 [nseq + 1]; sequence s holds tokens
 *             [cu[s], cu[s+1]).  They are read on the device: offsets are
 *             clamped to [0, total] and lengths to [0, max_seqlen] and to
 *             the tokens left, so out-of-range values cannot make the
 *             kernels leave the buffers, but only the rows of valid
 *             sequences are defined;
 *   max_seqlen_q/k: bounds of the sequence lengths (they size the grids);
 *   out:      device [total_q, Hq, D] in q's dtype, token stride out_sn and
 *             head stride out_sh (elements, multiples of 8), 16-byte aligned;
 *             rows of empty-key sequences are 0;
 *   lse:      device fp32, written iff return_lse: one [Hq, len_s] block per
 *             sequence in sequence order (Hq * total_q values), natural-log
 *             LSE of the unsmoothed scores, -inf for rows that see no key;
 *   ws:       device workspace (256-byte aligned) of
 *             sage_attn_fwd_varlen_workspace_bytes bytes.
 * sm_scale <= 0 selects 1/sqrt(D).  Returns SAGE_ERR_INVALID_ARG /
 * _UNSUPPORTED / _WORKSPACE on the host before any launch. */
sage_status sage_attn_fwd_varlen(const sage_tensor* q, const sage_tensor* k, const sage_tensor* v,
                                 const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                 int64_t nseq, int64_t max_seqlen_q, int64_t max_seqlen_k,
                                 int causal, float sm_scale, int smooth_k, int return_lse,
                                 void* out, int64_t out_sn, int64_t out_sh, float* lse, void* ws,
                                 size_t ws_bytes, sage_stream_t stream);

/* ------------------------------------------------- merge over key shards */
/* Running merge of attention results computed over disjoint parts of the
 * keys (pages: "Utilize SageAttention for Distributed Inference", the
 * return_lse of "sageattn_qk_int8_pv_fp8_cuda"): per row
 *   lse' = log(exp(lse) + exp(lse_part)),
 *   acc' = exp(lse - lse') * acc + exp(lse_part - lse') * part,
 * -inf meaning "no key seen" (weight 0; a row with no key anywhere stays
 * 0 / -inf).
 *   acc:      device fp32 [B, H, N, D] dense, 16-byte aligned, updated in place;
 *   acc_lse:  device fp32 [B, H, N], updated in place;
 *   part:     device bf16/fp16 [B, H, N, D], element strides (sb, sh, sn),
 *             multiples of 8, channel stride 1, 16-byte aligned (the output
 *             of the attention calls);
 *   part_lse: device fp32 [B, H, N] (their LSE);
 *   init:     non-zero for the first part (acc, acc_lse take its values).
 * D in {64, 128}. */
sage_status sage_lse_merge(float* acc, float* acc_lse, const void* part, int32_t part_dtype,
                           int64_t sb, int64_t sh, int64_t sn, const float* part_lse, int64_t B,
                           int64_t H, int64_t N, int64_t D, int init, sage_stream_t stream);

/* The merged result converted to bf16/fp16 (round to nearest even) with
 * element strides (sb, sh, sn). */
sage_status sage_lse_merge_finalize(const float* acc, void* out, int32_t out_dtype, int64_t sb,
                                    int64_t sh, int64_t sn, int64_t B, int64_t H, int64_t N,
                                    int64_t D, sage_stream_t stream);

/* ------------------------------------------------------------------ NVFP4 */
/* Workspace bytes of sage_quantize_qkv_nvfp4 (per-split K and Q sums, and the
 * Q means split into bf16 hi and lo parts for the correction MMA). */
size_t sage_quantize_nvfp4_workspace_bytes(int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq,
                                           int64_t Nk, int64_t D);

/* NVFP4 quantisation ("nvfp4_attention_sm120_quantize_qkv" of the FlashInfer
 * page, named there): K minus its mean over the first unpadded_k_len tokens
 * (rows at and beyond it become zero); Q minus its mean over each 128-token
 * block (per_block_mean != 0) or over all tokens; every 16-element vector
 * (along D for Q and K, along tokens for the transposed V) gets
 * sf = e4m3(fp32(amax/6)) and codes e2m1(fp32(x * fp32(1/sf))); then
 * qk_correction = qmean . Ks^T per Q block.  unpadded_k_len <= 0 means Nk.
 * out's shape fields, per_block_mean and unpadded_k_len must match the call. */
sage_status sage_quantize_qkv_nvfp4(const sage_tensor* q, const sage_tensor* k,
                                    const sage_tensor* v, int per_block_mean,
                                    int64_t unpadded_k_len, const sage_qkv_nvfp4* out, void* ws,
                                    size_t ws_bytes, sage_stream_t stream);

/* NVFP4 attention on the output of sage_quantize_qkv_nvfp4
 * ("nvfp4_attention_sm120_fwd"): scores sm_scale * (deq(Q).deq(K) +
 * qk_correction[q block, key]), keys at and beyond unpadded_k_len masked,
 * online softmax over 128-key tiles, P = 2688 * exp(s - running max)
 * quantised to NVFP4 per 16 keys, block-scaled FP4 PV accumulated in FP32,
 * out = O / (2688 * l).  per_block_mean must equal the value the quantiser
 * was called with.  out / lse as in sage_attn_fwd_quantized (lse needs
 * q_dot_kmean). */
sage_status sage_attn_fwd_nvfp4(const sage_qkv_nvfp4* qkv, float sm_scale, int causal,
                                int per_block_mean, int return_lse, void* out, int32_t out_dtype,
                                int64_t out_sb, int64_t out_sh, int64_t out_sn, float* lse,
                                sage_stream_t stream);

/* ------------------------------------------------------------ test exports */
/* Exact int32 QK^T of one 128x128 tile of codes: rows qblk*128.. of Q head
 * h, keys kblk*128.. of KV head h / (Hq/Hkv), batch b, computed by one
 * tcgen05 kind::i8 MMA chain exactly as the attention kernel does.
 * tile: device int32 [128, 128] (row-major). */
sage_status sage_debug_qk_int32(const sage_qkv_i8f8* qkv, int64_t b, int64_t h, int64_t qblk,
                                int64_t kblk, int32_t* tile, sage_stream_t stream);

/* FP8 PV product of one tile as the attention kernel computes it: p is a
 * device e4m3 [128, 128] row-major matrix (written to shared memory by
 * threads in the kernel's swizzled layout), times the transposed V codes of
 * keys kblk*128.. of KV head h_kv, batch b.  acc: device fp32 [128, D]. */
sage_status sage_debug_pv_fp32(const sage_qkv_i8f8* qkv, const uint8_t* p, int64_t b,
                               int64_t h_kv, int64_t kblk, float* acc, sage_stream_t stream);

/* Launches one thread that waits on a shared-memory barrier nothing
 * arrives on, bounded by timeout_us microseconds; the wait gives up, sets
 * the device status word and the kernel returns.  Used to test the
 * bounded-wait path without hanging the GPU. */
sage_status sage_debug_wait_timeout(uint32_t timeout_us, sage_stream_t stream);

/* ------------------------------------------------- allocation-free variant */
/* No counterpart on the pages: an addition of this library.
 *
 * sage_quantize_qkv needs a scratch workspace for its per-split K sums and
 * V maxima, and the caller has to allocate it.  Some callers cannot: a
 * plugin inside a host framework that owns every device allocation, or a
 * latency-critical loop where a cudaMalloc (which may synchronise the
 * device) is not allowed.  This entry point computes exactly what
 * sage_quantize_qkv computes, with the same inputs and outputs (still
 * caller-owned), but keeps its scratch in a fixed array of
 * SAGE_NOALLOC_SCRATCH_BYTES of device memory that is part of the library
 * itself: every GPU that loads the library holds that array until the
 * process exits.  It calls no cudaMalloc, cudaFree or allocating library
 * routine.
 *   - Size limit: sage_quantize_workspace_bytes(B, Hkv, Nk, D) must not
 *     exceed SAGE_NOALLOC_SCRATCH_BYTES; larger problems are rejected with
 *     SAGE_ERR_WORKSPACE before anything is enqueued (use
 *     sage_quantize_qkv with a workspace for them).
 *   - Set-up: the first call on each device looks up the array's device
 *     address (cudaGetSymbolAddress, with that device current) and caches
 *     it; make that first call before any stream capture.
 *   - Sharing: every call on a device uses the same array, which keeps the
 *     contents of the last call.  The kernels overwrite every scratch entry
 *     they read before reading it, so nothing needs clearing, but calls
 *     that overlap on the GPU (e.g. on two streams at once) race on the
 *     array: order them. */
#define SAGE_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)
sage_status sage_quantize_qkv_noalloc(const sage_tensor* q, const sage_tensor* k,
                                      const sage_tensor* v, int smooth_k,
                                      const sage_qkv_i8f8* out, sage_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SAGE_B200_H */
