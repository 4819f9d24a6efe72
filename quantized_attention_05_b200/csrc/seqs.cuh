// seqs.cuh -- the sequences of a call: batch entries of a dense call, or the
// packed sequences of a variable-length one (thu-ml/sageattention llms.txt,
// "sageattn_varlen": packed q/k/v with cumulative length arrays
// cu_seqlens_q/k).  Every sequence is its own problem: its own K mean,
// 128-token quantisation blocks starting at its first token, V channel
// scales and bottom-right causal alignment.
//
// Quantised layouts are the same in both cases: sequence s occupies, per
// head, pad128(len) rows starting at row H * cqp(s) + h * pad128(len),
// where cqp is the cumulative padded length.  For a dense call (all lengths
// N) that is exactly [B, H, N_pad, D].
#pragma once

#include <cstdint>

namespace sage {

// One sequence: lengths, first token in the (packed) inputs, first padded
// token in the quantised arrays.
struct SeqView {
  int nq, nk;
  int64_t cq, ck;
  int64_t cqp, ckp;
};

// Table entry layout written by seq_table_kernel: 8 int32 per sequence.
constexpr int SEQ_STRIDE = 8;

// `seqs` is null for a dense call (sequence s = batch entry s).
__device__ __forceinline__ SeqView seq_view(const int* seqs, int s, int Nq, int Nk) {
  SeqView v;
  if (seqs) {
    const int* e = seqs + SEQ_STRIDE * s;
    v.cq = e[0];
    v.nq = e[1];
    v.ck = e[2];
    v.nk = e[3];
    v.cqp = e[4];
    v.ckp = e[5];
  } else {
    v.nq = Nq;
    v.nk = Nk;
    v.cq = (int64_t)s * Nq;
    v.ck = (int64_t)s * Nk;
    v.cqp = (int64_t)s * ((Nq + 127) / 128 * 128);
    v.ckp = (int64_t)s * ((Nk + 127) / 128 * 128);
  }
  return v;
}

// One warp: the sanitised sequence table from the caller's cu_seqlens.
// Offsets are clamped to [0, total], lengths to [0, max_seqlen] and to the
// tokens left after the offset, so no later kernel can leave the packed
// inputs or the quantised arrays whatever the arrays hold; the padded
// offsets are the running sums of the padded (clamped) lengths.
__global__ void __launch_bounds__(32) seq_table_kernel(const int32_t* __restrict__ cu_q,
                                                       const int32_t* __restrict__ cu_k, int nseq,
                                                       int total_q, int total_k, int max_q,
                                                       int max_k, int* __restrict__ table) {
  const int lane = threadIdx.x;
  int run_q = 0, run_k = 0;
  for (int base = 0; base < nseq; base += 32) {
    const int s = base + lane;
    int cq = 0, nq = 0, ck = 0, nk = 0;
    if (s < nseq) {
      const int q0 = cu_q[s], q1 = cu_q[s + 1], k0 = cu_k[s], k1 = cu_k[s + 1];
      cq = min(max(q0, 0), total_q);
      ck = min(max(k0, 0), total_k);
      nq = min(min(max(q1 - q0, 0), max_q), total_q - cq);
      nk = min(min(max(k1 - k0, 0), max_k), total_k - ck);
    }
    const int pq = (nq + 127) / 128 * 128, pk = (nk + 127) / 128 * 128;
    // inclusive warp scans of the padded lengths
    int iq = pq, ik = pk;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int tq = __shfl_up_sync(0xffffffffu, iq, o);
      const int tk = __shfl_up_sync(0xffffffffu, ik, o);
      if (lane >= o) {
        iq += tq;
        ik += tk;
      }
    }
    if (s < nseq) {
      int* e = table + SEQ_STRIDE * s;
      e[0] = cq;
      e[1] = nq;
      e[2] = ck;
      e[3] = nk;
      e[4] = run_q + iq - pq;
      e[5] = run_k + ik - pk;
      e[6] = 0;
      e[7] = 0;
    }
    run_q += __shfl_sync(0xffffffffu, iq, 31);
    run_k += __shfl_sync(0xffffffffu, ik, 31);
  }
}

}  // namespace sage
