// quantize_nvfp4.cuh -- NVFP4 quantisation stage
// ("flashinfer.nvfp4_attention_sm120_fwd": packed FP4 Q/K/V with per-vector
// FP8 scale factors, V transposed, qk_correction with one row per 128-token Q
// block, per_block_mean, unpadded_k_len; "sageattn3_blackwell": FP4
// microscaling with per-block mean smoothing).
//
//   nv_colsum_kernel     per (batch, head, token split) double-double column
//                        sums of K (tokens < unpadded_k_len), and of Q when
//                        one global Q mean is asked for;
//   nv_means_kernel      the K mean and the global Q mean, each rounded once
//                        to fp32 (a per-block Q mean is formed by the block's
//                        quantiser CTA from the rows it has loaded);
//   nv_quant_kernel      one CTA per 128-token block of Q, V or K: every
//                        16-element vector gets sf = e4m3(fp32(amax/6)) and
//                        codes e2m1(fp32(x * fp32(1/sf))), packed two per byte
//                        (element 2i in the low nibble); V is transposed so
//                        its vectors run along tokens;
//   nv_corr_kernel       qk_correction = qmean . Ks^T on the tensor pipe (tcgen05
//                        bf16 MMAs of hi/lo splits, fp32 accumulation in TMEM).
// Every step that decides a code or a scale uses an explicitly rounded IEEE
// operation, so codes and scale factors are reproducible bit for bit.
#pragma once

#include "quantize_i8f8.cuh"

namespace sage {

struct NvQuantArgs {
  const void* q;
  const void* k;
  const void* v;
  int64_t q_sb, q_sh, q_sn, k_sb, k_sh, k_sn, v_sb, v_sh, v_sn;
  int B, Hq, Hkv, G, Nq, Nk, Nqp, Nkp, nqt, nkt;
  int L;                      // unpadded_k_len
  int per_block_mean;
  int k_splits, k_split_tokens;
  int q_splits, q_split_tokens;
  double* k_hi;               // [B*Hkv, k_splits, D]
  double* k_lo;
  double* q_hi;               // [B*Hq, q_splits, D]
  double* q_lo;
  uint8_t* q4;
  uint8_t* q_sf;
  uint8_t* k4;
  uint8_t* k_sf;
  uint8_t* v4t;
  uint8_t* v_sf_t;
  float* corr;
  float* q_mean;              // [B*Hq, nqt, D]
  uint16_t* qm_bhi;           // [B*Hq, nqt, D] bf16 bits: q_mean = hi + lo (+ 2^-18 relative)
  uint16_t* qm_blo;
  float* k_mean;              // [B*Hkv, D]
  float* qdk;                 // may be null
};

// ------------------------------------------------------------ fp4 helpers
// Eight fp32 values to eight E2M1 codes (rn, satfinite), x[0] in the lowest nibble.
__device__ __forceinline__ uint32_t e2m1x8(const float* x) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(x[0]), "f"(x[1]), "f"(x[2]), "f"(x[3]), "f"(x[4]), "f"(x[5]), "f"(x[6]), "f"(x[7]));
  return out;
}

// E4M3 code of one fp32 value (rn, satfinite).
__device__ __forceinline__ uint32_t e4m3_code(float x) { return cvt_e4m3x2(x, 0.f) & 0xFFu; }

// fp32 value of an E4M3 code (exact: every E4M3 value is an f16 value).
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  uint32_t h2;
  const uint16_t c = (uint16_t)(code & 0xFFu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// x / 6 rounded to nearest even, for every fp32 x whose quotient is normal
// (checked exhaustively against the IEEE division by tests/test_div6.py):
// the product with RN(1/6), then one correction with the exact residual
// fma(-q0, 6, x) -- Markstein's residual correction of a reciprocal product
// (P. Markstein, "Computation of elementary functions on the IBM RISC
// System/6000 processor", IBM J. Res. Dev. 34(1), 1990).  Smaller quotients can be one unit off, which no E4M3 code
// sees (they are below half its smallest subnormal, 2^-10).
__device__ __forceinline__ float div6_rn(float x) {
  const float c = 0.16666667f;   // RN(1/6) = 0x1.555556p-3
  const float q0 = __fmul_rn(x, c);
  const float r = __fmaf_rn(-q0, 6.f, x);
  return __fmaf_rn(r, c, q0);
}

// 1 / value(E4M3 code) for the 128 non-negative codes (0 for code 0), the
// table nvfp4_vector reads; filled by a CTA's threads before first use.
__device__ __forceinline__ void fill_e4m3_inverse(float* s_inv) {
  for (int i = threadIdx.x; i < 256; i += blockDim.x) {
    const float v = i < 128 ? e4m3_value((uint32_t)i) : 0.f;
    s_inv[i] = v > 0.f ? __frcp_rn(v) : 0.f;
  }
}

// NVFP4 quantisation of one 16-element vector: returns the scale-factor
// code; writes the 8 packed bytes (two words) of codes.  sf = e4m3(amax / 6)
// with the quotient of div6_rn (the IEEE one wherever an E4M3 code can tell),
// 1 / value(sf) from the table of fill_e4m3_inverse (the IEEE reciprocal).
__device__ __forceinline__ uint32_t nvfp4_vector(const float* x, const float* s_inv, uint32_t* w0,
                                                 uint32_t* w1) {
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(x[i]));
  const uint32_t sf = e4m3_code(div6_rn(a));
  const float inv = s_inv[sf];
  if (inv > 0.f) {
    float y[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) y[i] = __fmul_rn(x[i], inv);
    *w0 = e2m1x8(y);
    *w1 = e2m1x8(y + 8);
  } else {
    *w0 = 0u;
    *w1 = 0u;
  }
  return sf;
}

// bf16 hi / lo parts of x (round to nearest): x - hi is exact in fp32 and lo
// = bf16(x - hi) holds its next 8 bits, |x - hi - lo| <= 2^-18 |x|.
__device__ __forceinline__ void bf16_split(float x, uint16_t& hi, uint16_t& lo) {
  const __nv_bfloat16 h = __float2bfloat16_rn(x);
  hi = __bfloat16_as_ushort(h);
  lo = __bfloat16_as_ushort(__float2bfloat16_rn(__fsub_rn(x, __bfloat162float(h))));
}

// ------------------------------------------------------------ column sums
// grid (splits, B*H), 256 threads: per split of tokens [s*T, min(limit,(s+1)*T)),
// double-double sums of every channel.  D/8 threads per row (16 bytes each);
// each thread copies its own 16 bytes of the next passes into shared memory
// by cp.async (a ring of CS_SLOTS passes, CS_SLOTS - 1 in flight) and adds
// its channels in row order.
constexpr int CS_SLOTS = 8;
template <typename T, int D>
__global__ void __launch_bounds__(QUANT_THREADS)
    nv_colsum_kernel(const void* src, int64_t sb, int64_t sh, int64_t sn, int H, int limit,
                     int splits, int split_tokens, double* part_hi, double* part_lo) {
  constexpr int TPR = D / 8;
  constexpr int RPP = QUANT_THREADS / TPR;
  constexpr int ROWB = D * (int)sizeof(T);
  constexpr int SLOT = RPP * ROWB;
  constexpr int RED = RPP * D * 16;
  constexpr int BUF = CS_SLOTS * SLOT > RED ? CS_SLOTS * SLOT : RED;
  __shared__ __align__(16) uint8_t s_buf[BUF];
  const int split = blockIdx.x, bh = blockIdx.y;
  const int b = bh / H, h = bh % H;
  const int cg = threadIdx.x % TPR, rs = threadIdx.x / TPR;
  const int n0 = split * split_tokens, n1 = min(limit, n0 + split_tokens);
  DD acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = {0.0, 0.0};
  const char* base = reinterpret_cast<const char*>(src) + (b * sb + h * sh + cg * 8) * (int64_t)sizeof(T);
  auto issue = [&](int p) {
    const int n = n0 + p * RPP + rs;
    if (n < n1)
      cp_async16(s_buf + (p % CS_SLOTS) * SLOT + rs * ROWB + cg * 16, base + (int64_t)n * sn * sizeof(T));
    cp_async_commit();
  };
  const int npass = n1 > n0 ? (n1 - n0 + RPP - 1) / RPP : 0;
#pragma unroll
  for (int p = 0; p < CS_SLOTS - 1; ++p) issue(p);
  for (int p = 0; p < npass; ++p) {
    issue(p + CS_SLOTS - 1);         // into the slot this thread read at pass p - 1
    cp_async_wait<CS_SLOTS - 1>();   // pass p's copy (this thread's own) is done
    if (n0 + p * RPP + rs >= n1) break;
    float f[8];
    unpack8<T>(*reinterpret_cast<const uint4*>(s_buf + (p % CS_SLOTS) * SLOT + rs * ROWB + cg * 16), f);
#pragma unroll
    for (int i = 0; i < 8; ++i) dd_add(acc[i], (double)f[i]);
  }
  cp_async_wait_all();
  __syncthreads();   // the ring is reused for the partials below
  double* s_hi = reinterpret_cast<double*>(s_buf);
  double* s_lo = s_hi + RPP * D;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    s_hi[rs * D + cg * 8 + i] = acc[i].hi;
    s_lo[rs * D + cg * 8 + i] = acc[i].lo;
  }
  __syncthreads();
  if (threadIdx.x < D) {
    const int c = threadIdx.x;
    DD s = {0.0, 0.0};
    for (int r = 0; r < RPP; ++r) dd_add(s, DD{s_hi[r * D + c], s_lo[r * D + c]});
    const int64_t o = ((int64_t)bh * splits + split) * D + c;
    part_hi[o] = s.hi;
    part_lo[o] = s.lo;
  }
}

// grid (B*Hkv [+ B*Hq*ceil(nqt/NVM_QBLOCKS) for a global Q mean]): the K mean
// of each KV head, then the global Q mean written to NVM_QBLOCKS consecutive
// 128-token blocks of one Q head per CTA (each of the head's CTAs forms it).
constexpr int NVM_QBLOCKS = 8;
template <int D>
__global__ void __launch_bounds__(D) nv_means_kernel(NvQuantArgs a) {
  const int c = threadIdx.x;
  int id = blockIdx.x;
  if (id < a.B * a.Hkv) {
    DD s = {0.0, 0.0};
    for (int sp = 0; sp < a.k_splits; ++sp) {
      const int64_t o = ((int64_t)id * a.k_splits + sp) * D + c;
      dd_add(s, DD{a.k_hi[o], a.k_lo[o]});
    }
    a.k_mean[(int64_t)id * D + c] = a.L > 0 ? dd_mean_f32(s, (double)a.L) : 0.f;
    return;
  }
  id -= a.B * a.Hkv;
  const int ngrp = (a.nqt + NVM_QBLOCKS - 1) / NVM_QBLOCKS;
  const int grp = id % ngrp;
  id /= ngrp;
  const int qb0 = grp * NVM_QBLOCKS, qb1 = min(a.nqt, qb0 + NVM_QBLOCKS);
  float* qm = a.q_mean + (int64_t)id * a.nqt * D;
  // the global Q mean (per-block means are formed by the quantiser CTAs)
  DD s = {0.0, 0.0};
  for (int sp = 0; sp < a.q_splits; ++sp) {
    const int64_t o = ((int64_t)id * a.q_splits + sp) * D + c;
    dd_add(s, DD{a.q_hi[o], a.q_lo[o]});
  }
  const float m = dd_mean_f32(s, (double)a.Nq);
  uint16_t mh, ml;
  bf16_split(m, mh, ml);
  for (int qb = qb0; qb < qb1; ++qb) {
    qm[qb * D + c] = m;
    a.qm_bhi[((int64_t)id * a.nqt + qb) * D + c] = mh;
    a.qm_blo[((int64_t)id * a.nqt + qb) * D + c] = ml;
  }
}

// ------------------------------------------------------------ block quantiser
// One CTA per 128-token block: first the Q blocks, heads in descending order
// (the Q column sums, when there are any, read the heads in ascending order
// just before), then the V blocks, then the K blocks in descending head order
// (so that the correction kernel, which starts at head 0, finds the K rows
// read last in L2).  The block is copied into shared memory by cp.async (no
// registers hold it in flight, so more CTAs fit per SM).  Q/K: D/16 threads
// per row, one 16-element vector each.  V: every thread quantises 16-token
// vectors of one channel.
template <typename T, int D>
__global__ void __launch_bounds__(QUANT_THREADS) nv_quant_kernel(NvQuantArgs a) {
  constexpr int VPR = D / 16;                 // vectors per row
  constexpr int RPP = QUANT_THREADS / VPR;    // rows per pass
  constexpr int ITERS = QB / RPP;
  constexpr int CPR = D / 8;                  // 16-byte chunks per row
  // the means, one padding word per 16 channels: the eight threads of a row
  // read channels vi*16 + i in eight different banks
  __shared__ float s_m[D + D / 16];
  __shared__ float s_km[D + D / 16];
  __shared__ __align__(16) T s_v[QB][D + 8];
  __shared__ DD s_dd[QUANT_THREADS / D][D];
  __shared__ float s_inv[256];
  fill_e4m3_inverse(s_inv);   // ordered before its first use by the __syncthreads below
  const int nQb = a.B * a.Hq * a.nqt;
  const int nKb = a.B * a.Hkv * a.nkt;
  int job = blockIdx.x;
  const int vi = threadIdx.x % VPR, rs = threadIdx.x / VPR;
  // rows row0 .. row0+127 of one head into s_v (rows at and past `limit`
  // become zero); coalesced: consecutive threads copy consecutive 16 bytes
  auto stage = [&](const void* src, int64_t sb, int64_t sh, int64_t sn, int b, int h, int row0,
                   int limit) {
    const char* base = reinterpret_cast<const char*>(src) + (b * sb + h * sh) * (int64_t)sizeof(T);
    for (int q = threadIdx.x; q < QB * CPR; q += QUANT_THREADS) {
      const int r = q / CPR, c = q % CPR;
      T* dst = &s_v[r][c * 8];
      if (row0 + r < limit)
        cp_async16(dst, base + ((int64_t)(row0 + r) * sn + c * 8) * (int64_t)sizeof(T));
      else
        *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
    }
    cp_async_wait_all();
  };
  // the thread's 16 elements of block row r
  auto row16 = [&](int r, float* f) {
    unpack8<T>(*reinterpret_cast<const uint4*>(&s_v[r][vi * 16]), f);
    unpack8<T>(*reinterpret_cast<const uint4*>(&s_v[r][vi * 16 + 8]), f + 8);
  };

  if (job < nQb) {
    const int bh = a.B * a.Hq - 1 - job / a.nqt, qt = job % a.nqt;
    const int b = bh / a.Hq, h = bh % a.Hq, g = h / a.G;
    stage(a.q, a.q_sb, a.q_sh, a.q_sn, b, h, qt * QB, a.Nq);
    for (int c = threadIdx.x; c < D; c += blockDim.x) s_km[c + (c >> 4)] = a.k_mean[((int64_t)b * a.Hkv + g) * D + c];
    __syncthreads();
    if (a.per_block_mean) {
      // the block's mean: double-double column sums of the valid rows (TPC
      // threads per channel, combined in a fixed order), rounded once to fp32
      constexpr int TPC = QUANT_THREADS / D;
      constexpr int RPT = QB / TPC;
      const int c = threadIdx.x % D, part = threadIdx.x / D;
      const int cnt = min(a.Nq, (qt + 1) * QB) - qt * QB;
      // four interleaved accumulators (shorter dependency chains), combined in order
      DD acc[4] = {{0.0, 0.0}, {0.0, 0.0}, {0.0, 0.0}, {0.0, 0.0}};
      const int r1 = min(cnt, (part + 1) * RPT);
      for (int r = part * RPT; r < r1; r += 4)
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (r + u < r1) dd_add(acc[u], (double)to_f32<T>(s_v[r + u][c]));
      dd_add(acc[0], acc[1]);
      dd_add(acc[2], acc[3]);
      dd_add(acc[0], acc[2]);
      s_dd[part][c] = acc[0];
      __syncthreads();
      if (threadIdx.x < D) {
        DD sum = s_dd[0][c];
#pragma unroll
        for (int pp = 1; pp < TPC; ++pp) dd_add(sum, s_dd[pp][c]);
        const float m = dd_mean_f32(sum, (double)cnt);
        s_m[c + (c >> 4)] = m;
        const int64_t o = ((int64_t)bh * a.nqt + qt) * D + c;
        a.q_mean[o] = m;
        uint16_t mh, ml;
        bf16_split(m, mh, ml);
        a.qm_bhi[o] = mh;
        a.qm_blo[o] = ml;
      }
    } else {
      for (int c = threadIdx.x; c < D; c += blockDim.x) s_m[c + (c >> 4)] = a.q_mean[((int64_t)bh * a.nqt + qt) * D + c];
    }
    __syncthreads();
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
      const int r = rs + it * RPP, n = qt * QB + r;
      float x[16];
      float dq = 0.f;
      if (n < a.Nq) {
        float f[16];
        row16(r, f);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          x[i] = __fsub_rn(f[i], s_m[vi * 17 + i]);
          dq = fmaf(f[i], s_km[vi * 17 + i], dq);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = 0.f;
      }
      uint32_t w0, w1;
      const uint32_t sf = nvfp4_vector(x, s_inv, &w0, &w1);
      const int64_t row = (int64_t)bh * a.Nqp + n;
      *reinterpret_cast<uint2*>(a.q4 + row * (D / 2) + vi * 8) = make_uint2(w0, w1);
      a.q_sf[row * (D / 16) + vi] = (uint8_t)sf;
      if (a.qdk) {
#pragma unroll
        for (int o = VPR / 2; o > 0; o >>= 1) dq += __shfl_xor_sync(0xffffffffu, dq, o);
        if (vi == 0 && n < a.Nq) a.qdk[(int64_t)bh * a.Nq + n] = dq;
      }
    }
    return;
  }
  job -= nQb;
  if (job >= nKb) {
    job -= nKb;
    const int bh = a.B * a.Hkv - 1 - job / a.nkt, kt = job % a.nkt;
    const int b = bh / a.Hkv, h = bh % a.Hkv;
    stage(a.k, a.k_sb, a.k_sh, a.k_sn, b, h, kt * QB, a.L);
    for (int c = threadIdx.x; c < D; c += blockDim.x) s_km[c + (c >> 4)] = a.k_mean[(int64_t)bh * D + c];
    __syncthreads();
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
      const int r = rs + it * RPP, n = kt * QB + r;
      float x[16];
      if (n < a.L) {
        float f[16];
        row16(r, f);
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = __fsub_rn(f[i], s_km[vi * 17 + i]);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = 0.f;
      }
      uint32_t w0, w1;
      const uint32_t sf = nvfp4_vector(x, s_inv, &w0, &w1);
      const int64_t row = (int64_t)bh * a.Nkp + n;
      *reinterpret_cast<uint2*>(a.k4 + row * (D / 2) + vi * 8) = make_uint2(w0, w1);
      a.k_sf[row * (D / 16) + vi] = (uint8_t)sf;
    }
    return;
  }
  {
    const int bh = job / a.nkt, vt = job % a.nkt;
    const int b = bh / a.Hkv, h = bh % a.Hkv;
    stage(a.v, a.v_sb, a.v_sh, a.v_sn, b, h, vt * QB, a.L);
    __syncthreads();
    // vector (channel c, 16-token group gq): threads cover channels fastest
    for (int idx = threadIdx.x; idx < D * (QB / 16); idx += blockDim.x) {
      const int c = idx % D, gq = idx / D;
      float x[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) x[i] = to_f32<T>(s_v[gq * 16 + i][c]);
      uint32_t w0, w1;
      const uint32_t sf = nvfp4_vector(x, s_inv, &w0, &w1);
      const int64_t row = (int64_t)bh * D + c;
      *reinterpret_cast<uint2*>(a.v4t + row * (a.Nkp / 2) + vt * (QB / 2) + gq * 8) =
          make_uint2(w0, w1);
      a.v_sf_t[row * (a.Nkp / 16) + vt * (QB / 16) + gq] = (uint8_t)sf;
    }
  }
}

// ------------------------------------------------------------ qk_correction
// qk_correction[b,h,qb,j] = qmean[b,h,qb] . Ks[b,g,j] on the tensor pipe.
// Both operands are split into bf16 parts, x = hi + lo with
// |x - hi - lo| <= 2^-18 |x|, and the MMAs hi.hi + hi.lo + lo.hi accumulate
// in fp32 in TMEM; the omitted lo.lo and the split leave a relative error of
// about 2^-16 per product (the fp32 reference sum rounds at 2^-24).
// grid (nkt, B*Hkv), 256 threads, three CTAs per SM.  Per chunk of 128 Q-mean
// vectors the D channels are taken 64 at a time: all threads stage that half
// of the 128 keys (the MMA's M side, split here; the next half's rows are
// loaded while the MMAs of this one run) and of the 128 vectors (its N side,
// split once where the means are formed, copied by cp.async); thread 0
// issues the MMAs, and the next half overwrites the tiles once they have
// completed.  The scores land in TMEM as [key][vector], so for each vector
// the 32 lanes of a warp store 32 consecutive keys: every store instruction
// writes 128 contiguous bytes of a correction row, with no staging.
// Shared memory: A_hi, A_lo (128 keys x 64 channels), B_hi, B_lo (128
// vectors x 64 channels), bf16, K-major with the 128-byte swizzle: row r at
// r * 128, 16-byte chunk c at (c ^ (r % 8)) * 16.
constexpr int NVC_THREADS = 256;
template <int D>
struct NvCorrLayout {
  static constexpr int TILE = 128 * 64 * 2;   // one operand half: 128 rows x 64 bf16
  static constexpr int OFF_AHI = 0, OFF_ALO = TILE, OFF_BHI = 2 * TILE, OFF_BLO = 3 * TILE;
  static constexpr int BYTES = 4 * TILE + 1024;   // + alignment slack
};

// Channels 8*c .. 8*c+7 (c < 8) of row r into a swizzled 64-channel tile.
__device__ __forceinline__ void nvc_put(uint8_t* tile, int r, int c, const uint4& v) {
  *reinterpret_cast<uint4*>(tile + r * 128 + ((c ^ (r & 7)) << 4)) = v;
}

// bf16 hi / lo parts of 8 floats, two per word (lower channel in the low half).
// x - hi is exact in fp32, so lo = bf16(x - hi) is x's next 8 bits.  Pairs
// are converted by one packed round-to-nearest conversion each.
__device__ __forceinline__ void nvc_split8(const float* x, uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 hp = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
    const float2 hf = __bfloat1622float2(hp);
    const __nv_bfloat162 lp = __floats2bfloat162_rn(__fsub_rn(x[2 * i], hf.x), __fsub_rn(x[2 * i + 1], hf.y));
    h[i] = *reinterpret_cast<const uint32_t*>(&hp);
    l[i] = *reinterpret_cast<const uint32_t*>(&lp);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

template <typename T, int D>
__global__ void __launch_bounds__(NVC_THREADS, 3) nv_corr_kernel(NvQuantArgs a) {
  using L = NvCorrLayout<D>;
  extern __shared__ uint8_t nvc_raw[];
  uint8_t* sm = nvc_raw + ((1024u - (smem_u32(nvc_raw) & 1023u)) & 1023u);
  __shared__ uint64_t mma_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ float s_km[D + D / 8];   // one padding word per 8 channels (no bank conflicts)
  const int kt = blockIdx.x, bg = blockIdx.y;
  const int b = bg / a.Hkv, g = bg % a.Hkv;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  constexpr int PER = 128 * 8 / NVC_THREADS;   // 16-byte chunks per thread per operand half
  for (int c = t; c < D; c += NVC_THREADS) s_km[c + (c >> 3)] = a.k_mean[(int64_t)bg * D + c];
  if (t == 0) {
    mbar_init(&mma_bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  // the Q means of a chunk are 128 consecutive rows of q_mean: vector v of
  // KV head g is row (b*Hq + g*G)*nqt + v
  const int nvec = a.G * a.nqt;
  const uint16_t* qmh_base = a.qm_bhi + ((int64_t)b * a.Hq + (int64_t)g * a.G) * a.nqt * D;
  const uint16_t* qml_base = a.qm_blo + ((int64_t)b * a.Hq + (int64_t)g * a.G) * a.nqt * D;
  float* corr_base = a.corr + ((int64_t)b * a.Hq + (int64_t)g * a.G) * a.nqt * a.Nkp + kt * 128;
  const char* kbase = reinterpret_cast<const char*>(a.k) + (b * a.k_sb + g * a.k_sh) * (int64_t)sizeof(T);
  uint32_t phase = 0;
  bool ok = true;
  // K rows of one 64-channel half: chunk q = t + 256 i is channels
  // hf*64 + 8*(q % 8) .. of key q / 8
  uint4 kraw[PER];
  auto load_k = [&](int hf) {
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int q = t + NVC_THREADS * i, row = q >> 3, c = q & 7;
      const int n = kt * 128 + row;
      kraw[i] = n < a.L ? ldg16(kbase + ((int64_t)n * a.k_sn + hf * 64 + c * 8) * (int64_t)sizeof(T))
                        : make_uint4(0, 0, 0, 0);
    }
  };
  for (int v0 = 0; ok && v0 < nvec; v0 += 128) {
    load_k(0);
    for (int hf = 0; ok && hf < D / 64; ++hf) {
      // B: the Q means' hi and lo parts (split where the means were formed),
      // copied straight into the swizzled tiles; zero rows past nvec
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int q = t + NVC_THREADS * i, row = q >> 3, c = q & 7;
        uint8_t* dh = sm + L::OFF_BHI + row * 128 + ((c ^ (row & 7)) << 4);
        uint8_t* dl = sm + L::OFF_BLO + row * 128 + ((c ^ (row & 7)) << 4);
        if (v0 + row < nvec) {
          const int64_t o = (int64_t)(v0 + row) * D + hf * 64 + c * 8;
          cp_async16(dh, qmh_base + o);
          cp_async16(dl, qml_base + o);
        } else {
          *reinterpret_cast<uint4*>(dh) = make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(dl) = make_uint4(0, 0, 0, 0);
        }
      }
      // A: Ks = fp32(K - kmean) for keys < L, 0 beyond, split into hi + lo
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int q = t + NVC_THREADS * i, row = q >> 3, c = q & 7;
        const bool live = kt * 128 + row < a.L;
        float f[8];
        unpack8<T>(kraw[i], f);
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = live ? __fsub_rn(f[e], s_km[hf * 72 + c * 9 + e]) : 0.f;
        uint4 hi, lo;
        nvc_split8(f, hi, lo);
        nvc_put(sm + L::OFF_AHI, row, c, hi);
        nvc_put(sm + L::OFF_ALO, row, c, lo);
      }
      cp_async_wait_all();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      if (t == 0) {
        constexpr uint32_t ID = instr_desc(kDF32, 1u, 1u, 128, 128);   // bf16 x bf16 -> fp32
        const uint32_t ah = smem_u32(sm + L::OFF_AHI), al = smem_u32(sm + L::OFF_ALO);
        const uint32_t bh = smem_u32(sm + L::OFF_BHI), bl = smem_u32(sm + L::OFF_BLO);
        const uint32_t pa[3] = {ah, ah, al}, pb[3] = {bh, bl, bh};
#pragma unroll
        for (int pass = 0; pass < 3; ++pass)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_f16(tmem, smem_desc(pa[pass] + 32 * k, 1024, 128), smem_desc(pb[pass] + 32 * k, 1024, 128),
                    ID, (hf | pass | k) ? 1u : 0u);
        tc_commit(&mma_bar);
      }
      __syncwarp();
      // the next half's K rows are in flight while these MMAs run
      if (hf + 1 < D / 64) load_k(hf + 1);
      // the tiles are rewritten by the next half only after the MMAs are done
      ok = __all_sync(0xffffffffu, mbar_wait(&mma_bar, phase & 1, SITE_MMA_DONE));
      ++phase;
      tc_fence_after();
    }
    // TMEM [key][vector] -> correction rows: warp w holds keys 32*(w%4) ..
    // and vectors 64*(w/4) .. of the chunk
    if (ok) {
      const int key = (warp & 3) * 32 + lane;
      const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
#pragma unroll
      for (int cb = (warp >> 2) * 64; cb < (warp >> 2) * 64 + 64; cb += 32) {
        uint32_t o[32];
        SAGE_TMEM_LD32(tl + cb, o);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (v0 + cb + e < nvec) corr_base[(int64_t)(v0 + cb + e) * a.Nkp + key] = __uint_as_float(o[e]);
      }
    }
    // TMEM is rewritten by the next chunk
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  // every MMA issued above has completed (each half waited for its commit);
  // after a wait that gave up, warp 0 first lets the last MMAs finish
  if (warp == 0) {
    if (!ok && phase > 0) mbar_drain(&mma_bar, (phase - 1) & 1);
    tmem_dealloc(tmem, 128);
  }
}

}  // namespace sage
