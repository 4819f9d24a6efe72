// quantize_i8f8.cuh -- quantisation stage of the INT8-QK / FP8-PV attention
// (thu-ml/sageattention llms.txt: "smooth_k", per-block INT8 Q/K in
// "sageattn_qk_int8_pv_fp16_triton", per-channel FP8 V in
// "sageattn_qk_int8_pv_fp8_cuda").
//
// Three launches, HBM-bound, 128-bit coalesced loads:
//   pass A  per (batch, KV head, token split): exact-in-practice K channel
//           sums (double-double accumulation, fixed reduction order) and V
//           channel maxima into the workspace;
//   stats   per (batch, KV head): the splits combined in fixed order into
//           k_mean, v_scale and the V channel maxima;
//   pass B  one CTA per 128-token block of Q, K or V: the block's amax,
//           scale and INT8 codes (Q, K - kmean), or the per-channel E4M3
//           codes of V, stored in V's own [token, channel] order.
// Every arithmetic step that decides a code uses an explicitly rounded
// IEEE operation (__fsub_rn, __fmul_rn, __fdiv_rn, cvt.rn), so the codes and
// scales are reproducible bit for bit.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sage_ptx.cuh"
#include "seqs.cuh"

namespace sage {

constexpr int QB = 128;           // tokens per quantisation block
constexpr int QUANT_THREADS = 256;

struct QuantArgs {
  const void* q;
  const void* k;
  const void* v;
  int64_t q_sb, q_sh, q_sn, k_sb, k_sh, k_sn, v_sb, v_sh, v_sn;
  int B, Hq, Hkv, G, Nq, Nk, Nqp, Nkp, nqt, nkt;
  int smooth_k;
  int splits, split_tokens;       // pass A token splits
  double* part_hi;                // [B*Hkv, splits, D]
  double* part_lo;
  float* part_amax;
  int8_t* q8;
  float* q_scale;
  int8_t* k8;
  float* k_scale;
  float* k_mean;
  uint8_t* v8;
  float* v_scale;
  float* va;                      // [B*Hkv, D] V channel maxima (workspace)
  float* qdk;                     // may be null
  int kv_limit;                   // tokens of K/V used for the mean / codes (Nk)
  // sequences: B of them; `seqs` (device table, see seqs.cuh) for a packed
  // variable-length call, null for a dense one.  max_nqt / max_nkt bound
  // the 128-token blocks of any sequence (the block grid is sized by them).
  const int* seqs;
  int max_nqt, max_nkt;
};

// Element offset of sequence s in an input tensor: packed tokens for a
// variable-length call, the batch stride for a dense one.
__device__ __forceinline__ int64_t seq_in_offset(const QuantArgs& a, int64_t tok0, int s,
                                                 int64_t sn, int64_t sb) {
  return a.seqs ? tok0 * sn : (int64_t)s * sb;
}

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <>
__device__ __forceinline__ float to_f32<__half>(__half x) {
  return __half2float(x);
}

// 8 consecutive elements (one 16-byte load) as fp32.
template <typename T>
__device__ __forceinline__ void unpack8(const uint4& raw, float* f) {
  const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
  for (int i = 0; i < 8; ++i) f[i] = to_f32<T>(e[i]);
}

// max(|a|, |b|) of two packed pairs of T (elementwise), and the fp32 value of
// the low / high element of a pair.
template <typename T>
__device__ __forceinline__ uint32_t absmax2(uint32_t a, uint32_t b);
template <>
__device__ __forceinline__ uint32_t absmax2<__nv_bfloat16>(uint32_t a, uint32_t b) {
  const __nv_bfloat162 r = __hmax2(__habs2(*reinterpret_cast<const __nv_bfloat162*>(&a)),
                                   __habs2(*reinterpret_cast<const __nv_bfloat162*>(&b)));
  return *reinterpret_cast<const uint32_t*>(&r);
}
template <>
__device__ __forceinline__ uint32_t absmax2<__half>(uint32_t a, uint32_t b) {
  const __half2 r = __hmax2(__habs2(*reinterpret_cast<const __half2*>(&a)),
                            __habs2(*reinterpret_cast<const __half2*>(&b)));
  return *reinterpret_cast<const uint32_t*>(&r);
}
template <typename T>
__device__ __forceinline__ float lo_f32(uint32_t w) {
  return to_f32<T>(*reinterpret_cast<const T*>(&w));
}
template <typename T>
__device__ __forceinline__ float hi_f32(uint32_t w) {
  return to_f32<T>(*(reinterpret_cast<const T*>(&w) + 1));
}

__device__ __forceinline__ uint4 ldg16(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// ------------------------------------------------------------ double-double
struct DD {
  double hi, lo;
};
// hi + lo += x without rounding error in hi + x (error-free transformation).
__device__ __forceinline__ void dd_add(DD& acc, double x) {
  const double s = __dadd_rn(acc.hi, x);
  const double bb = __dsub_rn(s, acc.hi);
  const double err = __dadd_rn(__dsub_rn(acc.hi, __dsub_rn(s, bb)), __dsub_rn(x, bb));
  acc.hi = s;
  acc.lo = __dadd_rn(acc.lo, err);
}
__device__ __forceinline__ void dd_add(DD& acc, const DD& y) {
  dd_add(acc, y.hi);
  acc.lo = __dadd_rn(acc.lo, y.lo);
}
// fp32 value of (hi + lo) / n rounded once.  With the remainder of the
// division carried exactly, this equals the correctly rounded mean unless the
// exact value lies within ~2^-100 (relative) of an fp32 rounding boundary,
// which bf16/fp16 sums of fewer than 2^31 terms cannot do.
__device__ __forceinline__ float dd_mean_f32(const DD& s, double n) {
  const double q1 = __ddiv_rn(s.hi, n);
  const double r = __fma_rn(-q1, n, s.hi);  // exact remainder of the division
  const double q2 = __ddiv_rn(__dadd_rn(r, s.lo), n);
  return __double2float_rn(__dadd_rn(q1, q2));
}

// ------------------------------------------------------------ pass A
// 16-byte asynchronous copy global -> shared (L1 bypassed), one commit group
// per call of cp_async_commit, and the waits.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// grid (splits, B*Hkv), 256 threads.  Thread layout: D/8 threads per token
// row (16 bytes each), 256/(D/8) rows per pass.  Each thread copies its own
// 16 bytes of K and V of the next passes into shared memory by cp.async, a
// ring of PA_SLOTS passes (PA_SLOTS - 1 in flight: no registers hold them,
// so four CTAs fit per SM), and accumulates its channels in row order.
constexpr int PA_SLOTS = 6;
template <typename T, int D>
__global__ void __launch_bounds__(QUANT_THREADS) kmean_vamax_partial_kernel(QuantArgs a) {
  constexpr int TPR = D / 8;
  constexpr int RPP = QUANT_THREADS / TPR;
  constexpr int ROWB = D * (int)sizeof(T);
  constexpr int SLOT = 2 * RPP * ROWB;            // K rows, then V rows, of one pass
  constexpr int RED = RPP * D * (8 + 8 + 4);      // the per-row-group partials
  constexpr int BUF = PA_SLOTS * SLOT > RED ? PA_SLOTS * SLOT : RED;
  __shared__ __align__(16) uint8_t s_buf[BUF];

  const int split = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / a.Hkv, h = bh % a.Hkv;
  const SeqView sq = seq_view(a.seqs, b, a.Nq, a.kv_limit);
  const int cg = threadIdx.x % TPR, rs = threadIdx.x / TPR;
  const int n0 = split * a.split_tokens;
  const int n1 = min(sq.nk, n0 + a.split_tokens);

  DD acc[8];
  float am[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    acc[i] = {0.0, 0.0};
    am[i] = 0.f;
  }
  const char* kb = reinterpret_cast<const char*>(a.k) +
                   (seq_in_offset(a, sq.ck, b, a.k_sn, a.k_sb) + h * a.k_sh + cg * 8) *
                       (int64_t)sizeof(T);
  const char* vb = reinterpret_cast<const char*>(a.v) +
                   (seq_in_offset(a, sq.ck, b, a.v_sn, a.v_sb) + h * a.v_sh + cg * 8) *
                       (int64_t)sizeof(T);
  // pass p covers rows n0 + p*RPP + rs; every call commits one group (empty
  // past the split), so the group count stays uniform
  auto issue = [&](int p) {
    const int n = n0 + p * RPP + rs;
    uint8_t* slot = s_buf + (p % PA_SLOTS) * SLOT + rs * ROWB + cg * 16;
    if (n < n1) {
      if (a.smooth_k) cp_async16(slot, kb + (int64_t)n * a.k_sn * sizeof(T));
      cp_async16(slot + RPP * ROWB, vb + (int64_t)n * a.v_sn * sizeof(T));
    }
    cp_async_commit();
  };
  const int npass = n1 > n0 ? (n1 - n0 + RPP - 1) / RPP : 0;
#pragma unroll
  for (int p = 0; p < PA_SLOTS - 1; ++p) issue(p);
  for (int p = 0; p < npass; ++p) {
    issue(p + PA_SLOTS - 1);         // into the slot this thread read at pass p - 1
    cp_async_wait<PA_SLOTS - 1>();   // pass p's copies (this thread's own) are done
    if (n0 + p * RPP + rs >= n1) break;
    const uint8_t* slot = s_buf + (p % PA_SLOTS) * SLOT + rs * ROWB + cg * 16;
    float f[8];
    if (a.smooth_k) {
      unpack8<T>(*reinterpret_cast<const uint4*>(slot), f);
#pragma unroll
      for (int i = 0; i < 8; ++i) dd_add(acc[i], (double)f[i]);
    }
    unpack8<T>(*reinterpret_cast<const uint4*>(slot + RPP * ROWB), f);
#pragma unroll
    for (int i = 0; i < 8; ++i) am[i] = fmaxf(am[i], fabsf(f[i]));
  }
  cp_async_wait_all();
  __syncthreads();   // the ring is reused for the partials below
  double* s_hi = reinterpret_cast<double*>(s_buf);
  double* s_lo = s_hi + RPP * D;
  float* s_am = reinterpret_cast<float*>(s_lo + RPP * D);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    s_hi[rs * D + cg * 8 + i] = acc[i].hi;
    s_lo[rs * D + cg * 8 + i] = acc[i].lo;
    s_am[rs * D + cg * 8 + i] = am[i];
  }
  __syncthreads();
  if (threadIdx.x < D) {
    const int c = threadIdx.x;
    DD s = {0.0, 0.0};
    float m = 0.f;
    for (int r = 0; r < RPP; ++r) {  // fixed order: deterministic
      dd_add(s, DD{s_hi[r * D + c], s_lo[r * D + c]});
      m = fmaxf(m, s_am[r * D + c]);
    }
    const int64_t o = ((int64_t)bh * a.splits + split) * D + c;
    a.part_hi[o] = s.hi;
    a.part_lo[o] = s.lo;
    a.part_amax[o] = m;
  }
}

// ------------------------------------------------------------ stats
// grid B*Hkv, D threads: the splits of KV head bh combined in fixed order
// into k_mean (0 without smoothing), the V channel maxima and v_scale.
template <int D>
__global__ void __launch_bounds__(D) kv_stats_kernel(QuantArgs a) {
  const int bh = blockIdx.x, c = threadIdx.x;
  const int nk = seq_view(a.seqs, bh / a.Hkv, a.Nq, a.kv_limit).nk;
  DD s = {0.0, 0.0};
  float m = 0.f;
  // eight splits' partials loaded before they are combined, in split order
  constexpr int U = 8;
  for (int sp0 = 0; sp0 < a.splits; sp0 += U) {
    double hi[U], lo[U];
    float am[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t o = ((int64_t)bh * a.splits + sp0 + u) * D + c;
      const bool live = sp0 + u < a.splits;
      hi[u] = live ? a.part_hi[o] : 0.0;
      lo[u] = live ? a.part_lo[o] : 0.0;
      am[u] = live ? a.part_amax[o] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (sp0 + u >= a.splits) break;
      dd_add(s, DD{hi[u], lo[u]});
      m = fmaxf(m, am[u]);
    }
  }
  a.k_mean[(int64_t)bh * D + c] = a.smooth_k && nk > 0 ? dd_mean_f32(s, (double)nk) : 0.f;
  a.va[(int64_t)bh * D + c] = m;
  a.v_scale[(int64_t)bh * D + c] = __fdiv_rn(m, 448.f);
}

__device__ __forceinline__ float block_max(float v, float* s_red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) s_red[w] = v;
  __syncthreads();
  float r = s_red[0];
#pragma unroll
  for (int i = 1; i < QUANT_THREADS / 32; ++i) r = fmaxf(r, s_red[i]);
  return r;
}

// Eight INT8 codes rint(fp32(x[i] * inv)) (round half to even) packed into
// two words, x[0] in the low byte.  |x * inv| <= 127 by construction (inv =
// 127/amax of the block), so adding 1.5*2^23 to the fp32 product leaves the
// integer in the low mantissa bits and their low byte is the two's-complement
// code: FMA-pipe arithmetic and byte permutes instead of float-to-int
// conversions.  The product and the sum are scalar IEEE-rounded operations
// (__fmul_rn, __fadd_rn): the codes must be those of the two roundings, bit
// for bit.
__device__ __forceinline__ uint2 int8x8_codes(const float* x, float inv) {
  uint32_t t[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) t[i] = __float_as_uint(__fadd_rn(__fmul_rn(x[i], inv), 12582912.f));
  return make_uint2(
      __byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410),
      __byte_perm(__byte_perm(t[4], t[5], 0x0040), __byte_perm(t[6], t[7], 0x0040), 0x5410));
}

// Row sums over the TPR threads of each row, for the ITERS = TPR/2 rows a
// thread holds: a transposed butterfly (each level hands half of the
// remaining partial sums to the partner lane and keeps the other half), so
// ITERS rows cost ITERS shuffles instead of ITERS * log2(TPR).  Returns the
// full sum of row (cg >> 1) of the thread's rows; lanes cg and cg ^ 1 hold
// the same row.
template <int TPR>
__device__ __forceinline__ float rows_sum_transposed(float* v, int cg) {
  constexpr int ITERS = TPR / 2;
#pragma unroll
  for (int half = ITERS / 2; half >= 1; half >>= 1) {
    const bool up = (cg & (2 * half)) != 0;    // this lane keeps the upper half
#pragma unroll
    for (int j = 0; j < half; ++j) {
      const float keep = up ? v[j + half] : v[j];
      const float give = up ? v[j] : v[j + half];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, give, 2 * half);
    }
  }
  return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
}

// ------------------------------------------------------------ pass B
// One CTA per 128-token block: first the K and V blocks, KV heads in
// descending order (pass A reads the heads in ascending order, so the K and
// V rows it read last are still in L2 when pass B starts), K and V blocks of
// a head alternating; then the Q blocks.  Each thread copies its 16-byte
// pieces of the block into shared memory by cp.async and reads them for the
// amax and again for the codes.
template <typename T, int D>
__global__ void __launch_bounds__(QUANT_THREADS, 6) quant_blocks_kernel(QuantArgs a) {
  constexpr int TPR = D / 8;
  constexpr int RPP = QUANT_THREADS / TPR;
  constexpr int ITERS = QB / RPP;
  __shared__ float s_c[D];      // k_mean (Q with LSE, K) or 448 / V channel max (V)
  __shared__ float s_red[QUANT_THREADS / 32];

  const int nKb = a.B * a.Hkv * a.max_nkt;
  const int job = blockIdx.x;
  const int cg = threadIdx.x % TPR, rs = threadIdx.x / TPR;
  // the block's rows in shared memory: each thread copies its own 16 bytes
  // of its ITERS rows by cp.async (no registers hold them in flight) and
  // reads them back for the amax and for the codes; rows past `limit` are 0
  __shared__ __align__(16) uint8_t s_blk[QB * D * sizeof(T)];
  auto stage = [&](const char* base, int64_t sn, int row0, int limit) {
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
      const int r = rs + it * RPP;
      uint8_t* dst = s_blk + (r * D + cg * 8) * sizeof(T);
      if (row0 + r < limit)
        cp_async16(dst, base + (int64_t)(row0 + r) * sn * sizeof(T));
      else
        *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
    }
    cp_async_wait_all();
  };
  auto raw = [&](int it) -> uint4 {
    return *reinterpret_cast<const uint4*>(s_blk + ((rs + it * RPP) * D + cg * 8) * sizeof(T));
  };
  // K/V job -> (KV head, block, K or V)
  const int kvh = a.B * a.Hkv - 1 - job / (2 * a.max_nkt);
  const int kvt = (job % (2 * a.max_nkt)) >> 1;
  const bool is_v = job & 1;

  if (job >= 2 * nKb) {
    // ---------------- Q block
    const int bh = (job - 2 * nKb) / a.max_nqt, qt = (job - 2 * nKb) % a.max_nqt;
    const int b = bh / a.Hq, h = bh % a.Hq;
    const int g = h / a.G;
    const SeqView sq = seq_view(a.seqs, b, a.Nq, a.kv_limit);
    const int nqt = (sq.nq + 127) / 128, Nqp = nqt * 128;
    if (qt >= nqt) return;                  // beyond this sequence (whole CTA)
    const int64_t row0 = (int64_t)a.Hq * sq.cqp + (int64_t)h * Nqp;   // q8 row of token 0
    if (a.qdk)
      for (int c = threadIdx.x; c < D; c += blockDim.x) s_c[c] = a.k_mean[(int64_t)(b * a.Hkv + g) * D + c];
    const char* base = reinterpret_cast<const char*>(a.q) +
                       (seq_in_offset(a, sq.cq, b, a.q_sn, a.q_sb) + h * a.q_sh + cg * 8) *
                           (int64_t)sizeof(T);
    stage(base, a.q_sn, qt * QB, sq.nq);
    // |x| max on packed pairs of the input type (exact: every bf16/fp16
    // value is an fp32 value, and the max of magnitudes is one of them)
    uint32_t m2 = 0u;
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
      const uint4 r = raw(it);
      m2 = absmax2<T>(m2, absmax2<T>(absmax2<T>(r.x, r.y), absmax2<T>(r.z, r.w)));
    }
    const float am = fmaxf(lo_f32<T>(m2), hi_f32<T>(m2));
    const float amax = block_max(am, s_red);  // also orders s_c
    const float inv = amax > 0.f ? __fdiv_rn(127.f, amax) : 0.f;
    float dsum[ITERS];
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
      const int n = qt * QB + rs + it * RPP;
      float f[8];
      unpack8<T>(raw(it), f);
      *reinterpret_cast<uint2*>(a.q8 + (row0 + n) * D + cg * 8) = int8x8_codes(f, inv);
      if (a.qdk) {
        uint64_t d2 = f2_pack(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < 8; i += 2)
          d2 = f2_fma(f2_pack(f[i], f[i + 1]), f2_pack(s_c[cg * 8 + i], s_c[cg * 8 + i + 1]), d2);
        float d0, d1;
        f2_unpack(d2, d0, d1);
        dsum[it] = d0 + d1;
      }
    }
    if (a.qdk) {
      // row (cg >> 1) of this thread's rows, complete in lanes cg and cg ^ 1
      const float d = rows_sum_transposed<TPR>(dsum, cg);
      const int n = qt * QB + rs + (cg >> 1) * RPP;
      if ((cg & 1) == 0 && n < sq.nq) a.qdk[(int64_t)a.Hq * sq.cq + (int64_t)h * sq.nq + n] = d;
    }
    if (threadIdx.x == 0)
      a.q_scale[(int64_t)a.Hq * (sq.cqp / 128) + (int64_t)h * nqt + qt] = __fdiv_rn(amax, 127.f);
    return;
  }
  if (!is_v) {
    // ---------------- K block: codes of K - kmean
    const int bh = kvh, kt = kvt;
    const int b = bh / a.Hkv, h = bh % a.Hkv;
    const SeqView sq = seq_view(a.seqs, b, a.Nq, a.kv_limit);
    const int nkt = (sq.nk + 127) / 128, Nkp = nkt * 128;
    if (kt >= nkt) return;                  // beyond this sequence (whole CTA)
    const int64_t row0 = (int64_t)a.Hkv * sq.ckp + (int64_t)h * Nkp;
    for (int c = threadIdx.x; c < D; c += blockDim.x) s_c[c] = a.k_mean[(int64_t)bh * D + c];
    const char* base = reinterpret_cast<const char*>(a.k) +
                       (seq_in_offset(a, sq.ck, b, a.k_sn, a.k_sb) + h * a.k_sh + cg * 8) *
                           (int64_t)sizeof(T);
    stage(base, a.k_sn, kt * QB, sq.nk);
    __syncthreads();
    // K - kmean, one IEEE-rounded subtraction per element
    float km[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) km[i] = s_c[cg * 8 + i];
    auto smooth = [&](const uint4& r, float* f) {
      unpack8<T>(r, f);
#pragma unroll
      for (int i = 0; i < 8; ++i) f[i] = __fsub_rn(f[i], km[i]);
    };
    float am = 0.f;
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
      const int n = kt * QB + rs + it * RPP;
      float f[8];
      smooth(raw(it), f);
      if (n < sq.nk) {
#pragma unroll
        for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(f[i]));
      }
    }
    const float amax = block_max(am, s_red);
    const float inv = amax > 0.f ? __fdiv_rn(127.f, amax) : 0.f;
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
      const int n = kt * QB + rs + it * RPP;
      float f[8];
      smooth(raw(it), f);
      const uint2 w = n < sq.nk ? int8x8_codes(f, inv) : make_uint2(0u, 0u);
      *reinterpret_cast<uint2*>(a.k8 + (row0 + n) * D + cg * 8) = w;
    }
    if (threadIdx.x == 0)
      a.k_scale[(int64_t)a.Hkv * (sq.ckp / 128) + (int64_t)h * nkt + kt] = __fdiv_rn(amax, 127.f);
    return;
  }
  {
    // ---------------- V block: per-channel E4M3 codes, [token, channel] order
    const int bh = kvh, vt = kvt;
    const int b = bh / a.Hkv, h = bh % a.Hkv;
    const SeqView sq = seq_view(a.seqs, b, a.Nq, a.kv_limit);
    const int nkt = (sq.nk + 127) / 128, Nkp = nkt * 128;
    if (vt >= nkt) return;                  // beyond this sequence (whole CTA)
    const int64_t row0 = (int64_t)a.Hkv * sq.ckp + (int64_t)h * Nkp;
    for (int c = threadIdx.x; c < D; c += blockDim.x) {
      const float m = a.va[(int64_t)bh * D + c];
      s_c[c] = m > 0.f ? __fdiv_rn(448.f, m) : 0.f;
    }
    const char* base = reinterpret_cast<const char*>(a.v) +
                       (seq_in_offset(a, sq.ck, b, a.v_sn, a.v_sb) + h * a.v_sh + cg * 8) *
                           (int64_t)sizeof(T);
    stage(base, a.v_sn, vt * QB, sq.nk);
    __syncthreads();
    float inv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) inv[i] = s_c[cg * 8 + i];
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
      const int n = vt * QB + rs + it * RPP;
      float f[8];
      unpack8<T>(raw(it), f);
      uint32_t w[2] = {0u, 0u};
      if (n < sq.nk) {
#pragma unroll
        for (int i = 0; i < 8; i += 4)
          w[i >> 2] = cvt_e4m3x4(__fmul_rn(f[i], inv[i]), __fmul_rn(f[i + 1], inv[i + 1]),
                                 __fmul_rn(f[i + 2], inv[i + 2]), __fmul_rn(f[i + 3], inv[i + 3]));
      }
      *reinterpret_cast<uint2*>(a.v8 + (row0 + n) * D + cg * 8) = make_uint2(w[0], w[1]);
    }
  }
}

}  // namespace sage
