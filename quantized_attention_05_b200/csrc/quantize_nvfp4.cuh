// quantize_nvfp4.cuh -- NVFP4 quantisation stage
// ("flashinfer.nvfp4_attention_sm120_fwd": packed FP4 Q/K/V with per-vector
// FP8 scale factors, V transposed, qk_correction with one row per 128-token Q
// block, per_block_mean, unpadded_k_len; "sageattn3_blackwell": FP4
// microscaling with per-block mean smoothing).
//
//   nv_colsum_kernel     per (batch, head, token split) double-double column
//                        sums of K (tokens < unpadded_k_len) or Q;
//   nv_means_kernel      the K mean and the Q means (per 128-token block or
//                        global), each rounded once to fp32;
//   nv_quant_kernel      one CTA per 128-token block of Q, K or V: every
//                        16-element vector gets sf = e4m3(fp32(amax/6)) and
//                        codes e2m1(fp32(x * fp32(1/sf))), packed two per byte
//                        (element 2i in the low nibble); V is transposed so
//                        its vectors run along tokens;
//   nv_corr_kernel       qk_correction = qmean . Ks^T in fp32, register-blocked.
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

// NVFP4 quantisation of one 16-element vector: returns the scale-factor
// code; writes the 8 packed bytes (two words) of codes.
__device__ __forceinline__ uint32_t nvfp4_vector(const float* x, uint32_t* w0, uint32_t* w1) {
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(x[i]));
  const uint32_t sf = e4m3_code(__fdiv_rn(a, 6.f));
  const float s = e4m3_value(sf);
  if (s > 0.f) {
    const float inv = __frcp_rn(s);
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

// ------------------------------------------------------------ column sums
// grid (splits, B*H), 256 threads: per split of tokens [s*T, min(limit,(s+1)*T)),
// double-double sums of every channel.
template <typename T, int D>
__global__ void __launch_bounds__(QUANT_THREADS)
    nv_colsum_kernel(const void* src, int64_t sb, int64_t sh, int64_t sn, int H, int limit,
                     int splits, int split_tokens, double* part_hi, double* part_lo) {
  constexpr int TPR = D / 8;
  constexpr int RPP = QUANT_THREADS / TPR;
  __shared__ double s_hi[RPP][D];
  __shared__ double s_lo[RPP][D];
  const int split = blockIdx.x, bh = blockIdx.y;
  const int b = bh / H, h = bh % H;
  const int cg = threadIdx.x % TPR, rs = threadIdx.x / TPR;
  const int n0 = split * split_tokens, n1 = min(limit, n0 + split_tokens);
  DD acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = {0.0, 0.0};
  const char* base = reinterpret_cast<const char*>(src) + (b * sb + h * sh + cg * 8) * (int64_t)sizeof(T);
  for (int n = n0 + rs; n < n1; n += RPP) {
    float f[8];
    unpack8<T>(ldg16(base + (int64_t)n * sn * sizeof(T)), f);
#pragma unroll
    for (int i = 0; i < 8; ++i) dd_add(acc[i], (double)f[i]);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    s_hi[rs][cg * 8 + i] = acc[i].hi;
    s_lo[rs][cg * 8 + i] = acc[i].lo;
  }
  __syncthreads();
  if (threadIdx.x < D) {
    const int c = threadIdx.x;
    DD s = {0.0, 0.0};
    for (int r = 0; r < RPP; ++r) dd_add(s, DD{s_hi[r][c], s_lo[r][c]});
    const int64_t o = ((int64_t)bh * splits + split) * D + c;
    part_hi[o] = s.hi;
    part_lo[o] = s.lo;
  }
}

// grid (B*Hkv + B*Hq): the K mean of each KV head, the Q mean(s) of each Q head.
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
  float* qm = a.q_mean + (int64_t)id * a.nqt * D;
  if (a.per_block_mean) {  // q splits are exactly the 128-token blocks
    for (int qb = 0; qb < a.nqt; ++qb) {
      const int64_t o = ((int64_t)id * a.q_splits + qb) * D + c;
      const int cnt = min(a.Nq, (qb + 1) * QB) - qb * QB;
      qm[qb * D + c] = dd_mean_f32(DD{a.q_hi[o], a.q_lo[o]}, (double)cnt);
    }
  } else {
    DD s = {0.0, 0.0};
    for (int sp = 0; sp < a.q_splits; ++sp) {
      const int64_t o = ((int64_t)id * a.q_splits + sp) * D + c;
      dd_add(s, DD{a.q_hi[o], a.q_lo[o]});
    }
    const float m = dd_mean_f32(s, (double)a.Nq);
    for (int qb = 0; qb < a.nqt; ++qb) qm[qb * D + c] = m;
  }
}

// ------------------------------------------------------------ block quantiser
// One CTA per 128-token block: [0, nQb) Q, [nQb, nQb+nKb) K, then V blocks.
// Q/K: D/16 threads per row, one 16-element vector each.  V: the block is
// staged in shared memory and every thread quantises 16-token vectors of one
// channel.
template <typename T, int D>
__global__ void __launch_bounds__(QUANT_THREADS) nv_quant_kernel(NvQuantArgs a) {
  constexpr int VPR = D / 16;                 // vectors per row
  constexpr int RPP = QUANT_THREADS / VPR;    // rows per pass
  __shared__ float s_m[D];
  __shared__ float s_km[D];
  __shared__ __align__(16) T s_v[QB][D + 8];
  const int nQb = a.B * a.Hq * a.nqt;
  const int nKb = a.B * a.Hkv * a.nkt;
  int job = blockIdx.x;
  const int vi = threadIdx.x % VPR, rs = threadIdx.x / VPR;

  if (job < nQb) {
    const int bh = job / a.nqt, qt = job % a.nqt;
    const int b = bh / a.Hq, h = bh % a.Hq, g = h / a.G;
    for (int c = threadIdx.x; c < D; c += blockDim.x) {
      s_m[c] = a.q_mean[((int64_t)bh * a.nqt + qt) * D + c];
      s_km[c] = a.k_mean[((int64_t)b * a.Hkv + g) * D + c];
    }
    __syncthreads();
    const char* base = reinterpret_cast<const char*>(a.q) +
                       (b * a.q_sb + h * a.q_sh + vi * 16) * (int64_t)sizeof(T);
    for (int r = rs; r < QB; r += RPP) {
      const int n = qt * QB + r;
      float x[16];
      float dq = 0.f;
      if (n < a.Nq) {
        float f[16];
        const char* p = base + (int64_t)n * a.q_sn * sizeof(T);
        unpack8<T>(ldg16(p), f);
        unpack8<T>(ldg16(p + 8 * sizeof(T)), f + 8);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          x[i] = __fsub_rn(f[i], s_m[vi * 16 + i]);
          dq = fmaf(f[i], s_km[vi * 16 + i], dq);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = 0.f;
      }
      uint32_t w0, w1;
      const uint32_t sf = nvfp4_vector(x, &w0, &w1);
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
  if (job < nKb) {
    const int bh = job / a.nkt, kt = job % a.nkt;
    const int b = bh / a.Hkv, h = bh % a.Hkv;
    for (int c = threadIdx.x; c < D; c += blockDim.x) s_km[c] = a.k_mean[(int64_t)bh * D + c];
    __syncthreads();
    const char* base = reinterpret_cast<const char*>(a.k) +
                       (b * a.k_sb + h * a.k_sh + vi * 16) * (int64_t)sizeof(T);
    for (int r = rs; r < QB; r += RPP) {
      const int n = kt * QB + r;
      float x[16];
      if (n < a.L) {
        float f[16];
        const char* p = base + (int64_t)n * a.k_sn * sizeof(T);
        unpack8<T>(ldg16(p), f);
        unpack8<T>(ldg16(p + 8 * sizeof(T)), f + 8);
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = __fsub_rn(f[i], s_km[vi * 16 + i]);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = 0.f;
      }
      uint32_t w0, w1;
      const uint32_t sf = nvfp4_vector(x, &w0, &w1);
      const int64_t row = (int64_t)bh * a.Nkp + n;
      *reinterpret_cast<uint2*>(a.k4 + row * (D / 2) + vi * 8) = make_uint2(w0, w1);
      a.k_sf[row * (D / 16) + vi] = (uint8_t)sf;
    }
    return;
  }
  job -= nKb;
  {
    const int bh = job / a.nkt, vt = job % a.nkt;
    const int b = bh / a.Hkv, h = bh % a.Hkv;
    constexpr int TPR = D / 8;
    const int cg = threadIdx.x % TPR, rr = threadIdx.x / TPR;
    const char* base = reinterpret_cast<const char*>(a.v) +
                       (b * a.v_sb + h * a.v_sh + cg * 8) * (int64_t)sizeof(T);
    for (int r = rr; r < QB; r += QUANT_THREADS / TPR) {
      const int n = vt * QB + r;
      uint4 raw = make_uint4(0, 0, 0, 0);
      if (n < a.L) raw = ldg16(base + (int64_t)n * a.v_sn * sizeof(T));
      *reinterpret_cast<uint4*>(&s_v[r][cg * 8]) = raw;
    }
    __syncthreads();
    // vector (channel c, 16-token group gq): threads cover channels fastest
    for (int idx = threadIdx.x; idx < D * (QB / 16); idx += blockDim.x) {
      const int c = idx % D, gq = idx / D;
      float x[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) x[i] = to_f32<T>(s_v[gq * 16 + i][c]);
      uint32_t w0, w1;
      const uint32_t sf = nvfp4_vector(x, &w0, &w1);
      const int64_t row = (int64_t)bh * D + c;
      *reinterpret_cast<uint2*>(a.v4t + row * (a.Nkp / 2) + vt * (QB / 2) + gq * 8) =
          make_uint2(w0, w1);
      a.v_sf_t[row * (a.Nkp / 16) + vt * (QB / 16) + gq] = (uint8_t)sf;
    }
  }
}

// ------------------------------------------------------------ qk_correction
// grid (nkt, B*Hkv), 256 threads, dynamic smem: Ks^T tile [D][128] fp32 and
// 64 Q-mean vectors [64][D].  Thread: 4 consecutive keys x 8 Q-mean vectors.
// Rows are (Q head of the group, Q block) pairs, G * nqt of them.
template <typename T, int D>
__global__ void __launch_bounds__(256) nv_corr_kernel(NvQuantArgs a) {
  extern __shared__ float4 corr_smem[];
  float* s_kt = reinterpret_cast<float*>(corr_smem);  // [D][128]
  float* s_qm = s_kt + D * 128;                        // [64][D]
  const int kt = blockIdx.x, bg = blockIdx.y;
  const int b = bg / a.Hkv, g = bg % a.Hkv;
  // Ks = fp32(K - kmean) for keys < L, 0 beyond; consecutive threads take
  // consecutive keys, so the transposed shared-memory stores are
  // conflict-free
  for (int idx = threadIdx.x; idx < 128 * (D / 8); idx += blockDim.x) {
    const int key = idx % 128, cg = idx / 128;
    const int n = kt * 128 + key;
    float f[8];
    if (n < a.L) {
      unpack8<T>(ldg16(reinterpret_cast<const char*>(a.k) +
                       (b * a.k_sb + g * a.k_sh + (int64_t)n * a.k_sn + cg * 8) * (int64_t)sizeof(T)),
                 f);
      const float* km = a.k_mean + (int64_t)bg * D + cg * 8;
#pragma unroll
      for (int i = 0; i < 8; ++i) f[i] = __fsub_rn(f[i], __ldg(km + i));
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) f[i] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) s_kt[(cg * 8 + i) * 128 + key] = f[i];
  }
  const int kq = threadIdx.x % 32;   // keys 4*kq .. 4*kq+3
  const int vq = threadIdx.x / 32;   // vectors 8*vq .. 8*vq+7 of the chunk
  const int nvec = a.G * a.nqt;
  for (int v0 = 0; v0 < nvec; v0 += 64) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < 64 * D; idx += blockDim.x) {
      const int vv = idx / D, c = idx % D;
      const int v = v0 + vv;
      float val = 0.f;
      if (v < nvec) {
        const int h = g * a.G + v / a.nqt, qb = v % a.nqt;
        val = a.q_mean[(((int64_t)b * a.Hq + h) * a.nqt + qb) * D + c];
      }
      s_qm[vv * D + c] = val;
    }
    __syncthreads();
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    for (int c = 0; c < D; c += 4) {
      float4 kv[4];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) kv[cc] = *reinterpret_cast<const float4*>(&s_kt[(c + cc) * 128 + 4 * kq]);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 qv = *reinterpret_cast<const float4*>(&s_qm[(vq * 8 + i) * D + c]);
        const float qa[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          acc[i][0] = fmaf(qa[cc], kv[cc].x, acc[i][0]);
          acc[i][1] = fmaf(qa[cc], kv[cc].y, acc[i][1]);
          acc[i][2] = fmaf(qa[cc], kv[cc].z, acc[i][2]);
          acc[i][3] = fmaf(qa[cc], kv[cc].w, acc[i][3]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int v = v0 + vq * 8 + i;
      if (v < nvec) {
        const int h = g * a.G + v / a.nqt, qb = v % a.nqt;
        float* dst = a.corr + (((int64_t)b * a.Hq + h) * a.nqt + qb) * a.Nkp + kt * 128 + 4 * kq;
        *reinterpret_cast<float4*>(dst) = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
      }
    }
  }
}

}  // namespace sage
