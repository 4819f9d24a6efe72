// merge.cuh -- combining attention results over disjoint key shards
// (thu-ml/sageattention llms.txt, "Utilize SageAttention for Distributed
// Inference": the row log-sum-exp returned with return_lse lets partial
// results over parts of the keys be combined).  For a row with running
// (o, lse) and a new part (o_p, lse_p):
//   lse' = log(exp(lse) + exp(lse_p)),  o' = exp(lse - lse') o + exp(lse_p - lse') o_p,
// with -inf meaning "no key seen" (weight 0).  HBM-bound elementwise work:
// each thread owns 8 channels of one row (16-byte loads of the part).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "attn_fwd_i8f8.cuh"
#include "quantize_i8f8.cuh"

namespace sage {

struct MergeArgs {
  float* acc;            // fp32 [B, H, N, D] dense
  float* acc_lse;        // fp32 [B, H, N]
  const void* part;      // bf16/fp16, strides (sb, sh, sn)
  int64_t sb, sh, sn;
  const float* part_lse; // fp32 [B, H, N]
  int B, H, N;
  int init;              // 1: the accumulator takes the part
};

template <typename T, int D>
__global__ void __launch_bounds__(256) lse_merge_kernel(MergeArgs a) {
  constexpr int TPR = D / 8;
  const int64_t rows = (int64_t)a.B * a.H * a.N;
  const int64_t row = (int64_t)blockIdx.x * (256 / TPR) + threadIdx.x / TPR;
  const int cg = threadIdx.x % TPR;
  if (row >= rows) return;
  const int n = (int)(row % a.N);
  const int64_t bh = row / a.N;
  const int h = (int)(bh % a.H), b = (int)(bh / a.H);
  float f[8];
  unpack8<T>(ldg16(reinterpret_cast<const T*>(a.part) + (int64_t)b * a.sb + (int64_t)h * a.sh +
                   (int64_t)n * a.sn + cg * 8),
             f);
  const float lp = a.part_lse[row];
  float4* acc = reinterpret_cast<float4*>(a.acc + row * D + cg * 8);
  if (a.init) {
    // a part whose row saw no key (lse -inf) has weight 0 whatever it holds
    const float z = lp == -INFINITY ? 0.f : 1.f;
    acc[0] = make_float4(z * f[0], z * f[1], z * f[2], z * f[3]);
    acc[1] = make_float4(z * f[4], z * f[5], z * f[6], z * f[7]);
    if (cg == 0) a.acc_lse[row] = lp;
    return;
  }
  const float la = a.acc_lse[row];
  const float m = fmaxf(la, lp);
  if (m == -INFINITY) return;                        // no key in either: stays 0 / -inf
  // the lanes of this row (they all take the same path) have read the old
  // LSE before its owner overwrites it
  const unsigned lane = threadIdx.x & 31u;
  const unsigned row_mask = ((TPR == 32 ? 0u : (1u << TPR)) - 1u) << (lane / TPR * TPR);
  const float wa = la == -INFINITY ? 0.f : expf(la - m);
  const float wp = lp == -INFINITY ? 0.f : expf(lp - m);
  const float inv = 1.f / (wa + wp);
  const float ca = wa * inv, cp = wp * inv;
  const float4 x0 = acc[0], x1 = acc[1];
  acc[0] = make_float4(ca * x0.x + cp * f[0], ca * x0.y + cp * f[1], ca * x0.z + cp * f[2],
                       ca * x0.w + cp * f[3]);
  acc[1] = make_float4(ca * x1.x + cp * f[4], ca * x1.y + cp * f[5], ca * x1.z + cp * f[6],
                       ca * x1.w + cp * f[7]);
  __syncwarp(row_mask);
  if (cg == 0) a.acc_lse[row] = m + logf(wa + wp);
}

// The merged result in the caller's dtype and layout.
template <typename T, int D>
__global__ void __launch_bounds__(256) lse_merge_finalize_kernel(const float* __restrict__ acc,
                                                                 void* out, int64_t sb, int64_t sh,
                                                                 int64_t sn, int B, int H, int N) {
  constexpr int TPR = D / 8;
  const int64_t rows = (int64_t)B * H * N;
  const int64_t row = (int64_t)blockIdx.x * (256 / TPR) + threadIdx.x / TPR;
  const int cg = threadIdx.x % TPR;
  if (row >= rows) return;
  const int n = (int)(row % N);
  const int64_t bh = row / N;
  const int h = (int)(bh % H), b = (int)(bh / H);
  const float4 x0 = reinterpret_cast<const float4*>(acc + row * D + cg * 8)[0];
  const float4 x1 = reinterpret_cast<const float4*>(acc + row * D + cg * 8)[1];
  uint32_t w[4];
  w[0] = pack2<T>(x0.x, x0.y);
  w[1] = pack2<T>(x0.z, x0.w);
  w[2] = pack2<T>(x1.x, x1.y);
  w[3] = pack2<T>(x1.z, x1.w);
  *reinterpret_cast<uint4*>(reinterpret_cast<T*>(out) + (int64_t)b * sb + (int64_t)h * sh +
                            (int64_t)n * sn + cg * 8) = make_uint4(w[0], w[1], w[2], w[3]);
}

}  // namespace sage
