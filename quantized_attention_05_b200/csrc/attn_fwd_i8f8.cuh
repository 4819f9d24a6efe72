// attn_fwd_i8f8.cuh -- fused INT8-QK / FP8-PV attention forward for sm_100a
// (thu-ml/sageattention llms.txt: "sageattn_qk_int8_pv_fp8_cuda",
// "sageattn_qk_int8_pv_fp8_cuda_sm90": INT8 Q/K with per-block scales,
// per-channel FP8 V, PV accumulated in FP32, causal mask, LSE; "sageattn":
// GQA and sm_scale; the Triton kernel's boolean mask).
//
// One CTA owns two 128-row Q tiles of one (batch, Q head) and streams the
// 128-key K/V tiles of its KV head:
//   warp 8      TMA producer: Q tiles once, then K and V tiles (V in
//               [token, channel] order, read MN-major by the PV MMA) into a
//               3-stage ring;
//   warps 9, 10 MMA issuers, one thread each, for Q tile 0 and Q tile 1:
//               S_i = 1.5*2^23 (one f16 MMA) + Q_i K^T with tcgen05 kind::i8
//               into TMEM (int32, exact, read back as a float), O_i += P_i V
//               with kind::f8f6f4 (E4M3 x E4M3 -> FP32 in TMEM); each issues
//               the next tile's QK^T of its Q tile as soon as that tile's S
//               has been read, so the tensor pipe runs while softmax works,
//               and the two threads' waits and commits overlap each other's
//               MMAs;
//   warps 0..7  two softmax warpgroups, one per Q tile, one thread per row:
//               tcgen05.ld of the int32 scores, dequantisation by
//               q_scale*k_scale*sm_scale*log2(e), masking, online softmax
//               with exp2, P -> E4M3 (pre-scaled by 448) into shared
//               memory in the 128-byte-swizzled K-major layout of the MMA,
//               O rescaled in TMEM when the running max moves, and the
//               epilogue (O * vscale / l -> bf16/fp16, LSE).
// TMEM: 512 columns = 2 x (S 128 columns + O D columns, padded to 256).
// Every wait on a barrier is bounded (sage_ptx.cuh).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sage_ptx.cuh"
#include "seqs.cuh"

namespace sage {

constexpr int ATT_BM = 128, ATT_BN = 128;
constexpr int ATT_STAGES = 3;
constexpr int ATT_ISSUERS = 2;      // MMA-issuing threads: warps 9 and 10, one per Q tile
constexpr int ATT_THREADS = 384;   // 3 warpgroups: 2 softmax, 1 TMA/MMA (+1 idle warp)
// Register split between the warpgroups (setmaxnreg): the TMA/MMA warpgroup
// keeps ATT_REGS_LOW per thread, the softmax warpgroups grow to
// ATT_REGS_HIGH.  The sum must not exceed what the block is launched with
// (384 threads x the kernel's compiled register count); the host checks it.
// 208 / 88 compiles without spills (224 / 56 spilled a few words and ran
// 1.5 % slower on B200).
constexpr int ATT_REGS_LOW = 88;
constexpr int ATT_REGS_HIGH = 208;
constexpr int ATT_MAX_NKT = 2048;   // keys <= 262144
constexpr float LOG2_448 = 8.807354922057604f;
constexpr float LN2_F = 0.6931471805599453f;
constexpr float LOG2E_F = 1.4426950408889634f;

struct AttnArgs {
  const float* q_scale;
  const float* k_scale;
  const float* v_scale;
  const float* qdk;
  void* out;
  int64_t out_sb, out_sh, out_sn;
  int out_fp16;
  float* lse;
  const uint8_t* tile_class;       // [Bm, Hm, nqt, nkt] or null
  const void* mask;                // bool bytes or fp32 (mask_kind), element strides
  int64_t m_sb, m_sh, m_sq;
  int m_bcast_b, m_bcast_h, mask_vec16;
  int mask_kind;                   // 0: boolean, 1: fp32 added to the scaled scores
  int B, Hq, Hkv, G, Nq, Nk, Nqp, Nkp, nqt, nkt, nqp;
  int causal, return_lse, causal_off;
  float c0;                        // sm_scale * log2(e)
  float sm_scale;
  // B sequences; `seqs` (device table, see seqs.cuh) for a packed
  // variable-length call, null for a dense one; max_nqp bounds the Q-tile
  // pairs of any sequence (the grid is sized by it).
  const int* seqs;
  int max_nqp;
};

// The sequence a CTA works on: its sizes and where its head's rows start in
// the quantised arrays, the scales, q.kmean / LSE and the output.
struct CtaSeq {
  int Nq, Nk, nqt, nkt, Nqp, Nkp, causal_off;
  int64_t qrow0, krow0;   // q8 row, k8/v8 row of token 0
  int64_t qs0, ks0;       // q_scale, k_scale index of block 0
  int64_t tok0;           // q_dot_kmean / lse index of token 0
  int64_t out0;           // out element offset of token 0
};

__device__ __forceinline__ CtaSeq cta_seq(const AttnArgs& a, int s, int h, int g) {
  const SeqView v = seq_view(a.seqs, s, a.Nq, a.Nk);
  CtaSeq c;
  c.Nq = v.nq;
  c.Nk = v.nk;
  c.nqt = (v.nq + ATT_BM - 1) / ATT_BM;
  c.nkt = (v.nk + ATT_BN - 1) / ATT_BN;
  c.Nqp = c.nqt * ATT_BM;
  c.Nkp = c.nkt * ATT_BN;
  c.causal_off = v.nk - v.nq;
  c.qrow0 = (int64_t)a.Hq * v.cqp + (int64_t)h * c.Nqp;
  c.krow0 = (int64_t)a.Hkv * v.ckp + (int64_t)g * c.Nkp;
  c.qs0 = (int64_t)a.Hq * (v.cqp / ATT_BM) + (int64_t)h * c.nqt;
  c.ks0 = (int64_t)a.Hkv * (v.ckp / ATT_BN) + (int64_t)g * c.nkt;
  c.tok0 = (int64_t)a.Hq * v.cq + (int64_t)h * v.nq;
  c.out0 = (a.seqs ? v.cq * a.out_sn : (int64_t)s * a.out_sb) + (int64_t)h * a.out_sh;
  return c;
}

template <int D>
struct AttnLayout {
  static constexpr int Q_BYTES = ATT_BM * D;
  static constexpr int K_BYTES = ATT_BN * D;
  static constexpr int V_BYTES = ATT_BN * D;
  static constexpr int P_BYTES = ATT_BM * ATT_BN;
  static constexpr int QK_SWIZZLE = D;            // bytes per Q/K row: 128 or 64
  static constexpr int QK_SBO = 8 * D;            // 8-row group stride
  // V tile: 128 token rows of D bytes, read MN-major by the PV MMA (one
  // swizzle atom across D, 8-row groups QK_SBO apart); one MMA consumes 32
  // tokens, i.e. 32 rows.
  static constexpr int V_KSTEP = 32 * D;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + ATT_STAGES * K_BYTES;
  static constexpr int OFF_P = OFF_V + ATT_STAGES * V_BYTES;   // [warpgroup][buffer]
  static constexpr int OFF_INIT = OFF_P + 4 * P_BYTES;   // f16 A (4 KB) and B (4 KB) of the S init
  static constexpr int OFF_BAR = OFF_INIT + 8192;
  // q_full, kv_full[S], kv_empty[S], s_full[2], s_free[2], p_full[2][2],
  // o_ready[2][2], mma_done, wg0_started
  static constexpr int NBAR = 1 + 2 * ATT_STAGES + 2 + 2 + 4 + 4 + 1 + 1;
  static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
  static constexpr int OFF_VS = (OFF_TMEM + 16 + 15) / 16 * 16;
  static constexpr int OFF_NLIST = OFF_VS + D * 4;
  static constexpr int OFF_LIST = OFF_NLIST + 16;
  // the list of visible key tiles, then their K scales
  static constexpr size_t bytes(int nkt) { return 1024 + OFF_LIST + (size_t)nkt * 8; }
};
// the longest key list must fit the 227 KB of shared memory a CTA can have
static_assert(AttnLayout<128>::bytes(ATT_MAX_NKT) <= 232448, "attention smem");
static_assert(AttnLayout<64>::bytes(ATT_MAX_NKT) <= 232448, "attention smem");

// Exponentials: every one on MUFU ex2.  An FMA-pipe polynomial for one pair
// in 8 (or 4) gained at most 1 % on B200 and moved enough E4M3 roundings of
// P to break the parity bound on short rows; a threshold on rescaling O
// (keeping a stale max until it is exceeded by a margin) gained 7 % but
// quantises P against another reference than the exact running max, which
// broke the parity bound on small cases too.
// int32 score S as the float 1.5*2^23 + S (exact for |S| < 2^22): the QK^T
// MMA accumulates the int32 S onto the bit pattern of 1.5*2^23 (0x4B400000),
// which an f16 MMA (512 x 1536 summed over K = 16) writes into S first.
constexpr float MAGIC_F = 12582912.0f;

// Write one thread's row of 128 E4M3 probabilities (32 packed words) into a
// 128x128-byte K-major tile with the 128-byte swizzle: 16-byte chunk c of
// row r lives at r*128 + ((c ^ (r % 8)) * 16).  Tile base 1024-aligned.
__device__ __forceinline__ void store_p_row(uint8_t* tile, int r, const uint32_t* pk) {
  uint8_t* row = tile + r * 128;
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) << 4)) =
        make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
}

// Flags of key tile kt for Q tile qt (0 if nothing in it is visible):
// bit 0 visible, bit 2 needs per-element masking, bit 4 reads the boolean
// mask; shifted left by `wg` (0 or 1).
__device__ __forceinline__ uint32_t tile_flags(const AttnArgs& a, const CtaSeq& cs, int b, int h,
                                               int qt, int wg, int kt) {
  const int row_lo = qt * ATT_BM;
  if (row_lo >= cs.Nq) return 0;
  const int row_hi = min(row_lo + ATT_BM - 1, cs.Nq - 1);
  const int key_lo = kt * ATT_BN, key_hi = key_lo + ATT_BN - 1;
  if (key_lo >= cs.Nk) return 0;
  if (a.causal && key_lo > row_hi + cs.causal_off) return 0;
  bool need = key_hi >= cs.Nk || (a.causal && key_hi > row_lo + cs.causal_off);
  bool part = false;
  if (a.tile_class) {
    const int bm = a.m_bcast_b ? 0 : b, hm = a.m_bcast_h ? 0 : h;
    const int Hm = a.m_bcast_h ? 1 : a.Hq;
    const uint8_t cls = a.tile_class[(((int64_t)bm * Hm + hm) * a.nqt + qt) * a.nkt + kt];
    if (cls == 0) return 0;
    part = cls == 2;
  }
  const uint32_t f = 1u | ((need || part) ? 4u : 0u) | (part ? 16u : 0u);
  return f << wg;
}

__device__ __forceinline__ void decode_work(const AttnArgs& a, int bid, int& qp, int& b, int& h) {
  if (a.causal || a.seqs) {  // longest rows first
    const int per = a.B * a.Hq;
    qp = a.max_nqp - 1 - bid / per;
    const int r = bid % per;
    b = r / a.Hq;
    h = r % a.Hq;
  } else {         // Q heads sharing a KV head run side by side (K/V reuse in L2)
    const int j = bid % a.G;
    int t = bid / a.G;
    qp = t % a.nqp;
    t /= a.nqp;
    const int g = t % a.Hkv;
    b = t / a.Hkv;
    h = g * a.G + j;
  }
}

template <typename OutT>
__device__ __forceinline__ uint32_t pack2(float lo, float hi);
template <>
__device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
template <>
__device__ __forceinline__ uint32_t pack2<__half>(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int D, typename OutT>
__device__ __forceinline__ void store_out_chunk(const AttnArgs& a, OutT* orow, int cb,
                                                const uint32_t* o, const float* s_vs, float inv_l) {
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float x0 = __uint_as_float(o[2 * i]) * s_vs[cb + 2 * i] * inv_l;
    const float x1 = __uint_as_float(o[2 * i + 1]) * s_vs[cb + 2 * i + 1] * inv_l;
    w[i] = pack2<OutT>(x0, x1);
  }
  uint4* dst = reinterpret_cast<uint4*>(orow + cb);
#pragma unroll
  for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
}

// Visibility of the 128 keys of tile kt for one row (bit j of vis[j / 32]):
// key length, causal limit and, for mixed mask tiles, the boolean mask.
__device__ __forceinline__ void tile_visibility(const AttnArgs& a, const CtaSeq& cs, int kt,
                                                int row, bool part, const uint8_t* mrow,
                                                uint32_t* vis) {
  const int key0 = kt * ATT_BN;
  int jmax = min(ATT_BN - 1, cs.Nk - 1 - key0);
  if (a.causal) jmax = min(jmax, row + cs.causal_off - key0);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const int hi = jmax - 32 * w;  // keep bits 0..hi
    vis[w] = hi >= 31 ? ~0u : (hi < 0 ? 0u : ((2u << hi) - 1u));
  }
  if (part && mrow) {
    const uint8_t* mk = mrow + key0;
    if (a.mask_vec16 && key0 + ATT_BN <= cs.Nk) {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint4 mv = __ldg(reinterpret_cast<const uint4*>(mk) + q);
        const uint32_t wds[4] = {mv.x, mv.y, mv.z, mv.w};
        uint32_t bits = 0;
#pragma unroll
        for (int t = 0; t < 16; ++t)
          bits |= (((wds[t >> 2] >> (8 * (t & 3))) & 0xFFu) ? 1u : 0u) << t;
        vis[q >> 1] &= ~(((~bits) & 0xFFFFu) << (16 * (q & 1)));
      }
    } else {
      // word index unrolled, so vis stays in registers
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        uint32_t bits = vis[w];
        for (int t = 0; t < 32; ++t)
          if (key0 + 32 * w + t < cs.Nk && mk[32 * w + t] == 0) bits &= ~(1u << t);
        vis[w] = bits;
      }
    }
  }
}

// Exponentials, E4M3 P into the swizzled shared-memory tile, and the row sum
// of one 128-key tile.  sr holds 1.5*2^23 + S as float bits (0 for hidden
// keys when NEED); p = 2^(S*c + bias) in fp32, P = E4M3(p) (bias includes
// log2(448) and minus the running max), row sum of the unquantised p.
// BIASED: sr already holds the scaled score plus the mask's bias (log2
// units, -inf for hidden keys) as float bits; p = 2^(sr + bias).
template <bool NEED, bool BIASED = false>
__device__ __forceinline__ float exp_tile(const uint32_t* sr, const uint32_t* vis, float c,
                                          float bias, uint8_t* ptile, int rt) {
  const uint64_t c2 = f2_pack(c, c), b2 = f2_pack(bias, bias);
  const uint64_t nm2 = f2_pack(-MAGIC_F, -MAGIC_F);
  uint64_t acc = f2_pack(0.f, 0.f);
  uint8_t* prow = ptile + rt * 128;
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) {
    uint32_t pw[8];
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
      float pp[4];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int j = ch * 32 + 2 * (i + u);
        const uint64_t y =
            BIASED ? f2_add(f2_pack(__uint_as_float(sr[j]), __uint_as_float(sr[j + 1])), b2)
                   : f2_fma(f2_add(f2_pack(__uint_as_float(sr[j]), __uint_as_float(sr[j + 1])), nm2),
                            c2, b2);
        float y0, y1;
        f2_unpack(y, y0, y1);
        uint64_t p = f2_pack(ex2_approx(y0), ex2_approx(y1));
        if (NEED) {
          float p0, p1;
          f2_unpack(p, p0, p1);
          if (!((vis[j >> 5] >> (j & 31)) & 1u)) p0 = 0.f;
          if (!((vis[j >> 5] >> ((j + 1) & 31)) & 1u)) p1 = 0.f;
          p = f2_pack(p0, p1);
        }
        acc = f2_add(acc, p);
        f2_unpack(p, pp[2 * u], pp[2 * u + 1]);
      }
      pw[i >> 1] = cvt_e4m3x4(pp[0], pp[1], pp[2], pp[3]);
    }
    // 16-byte chunks 2ch and 2ch+1 of the row, 128-byte swizzle
    *reinterpret_cast<uint4*>(prow + (((2 * ch) ^ (rt & 7)) << 4)) =
        make_uint4(pw[0], pw[1], pw[2], pw[3]);
    *reinterpret_cast<uint4*>(prow + (((2 * ch + 1) ^ (rt & 7)) << 4)) =
        make_uint4(pw[4], pw[5], pw[6], pw[7]);
  }
  float a0, a1;
  f2_unpack(acc, a0, a1);
  return a0 + a1;
}

// FMASK: the instantiation for a float mask (its biased softmax path is
// compiled only there, so the kernel without it keeps its code size).
template <int D, bool FMASK>
__global__ void __launch_bounds__(ATT_THREADS, 1)
    attn_fwd_i8f8_kernel(const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, AttnArgs a) {
  using L = AttnLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sK = smem + L::OFF_K;
  uint8_t* sV = smem + L::OFF_V;
  uint8_t* sP = smem + L::OFF_P;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint8_t* sInit = smem + L::OFF_INIT;
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + ATT_STAGES;
  uint64_t* s_full = kv_empty + ATT_STAGES;   // [wg]
  uint64_t* s_free = s_full + 2;              // [wg]
  uint64_t* p_full = s_free + 2;              // [wg * 2 + buffer]
  uint64_t* o_ready = p_full + 4;             // [wg * 2 + buffer]
  uint64_t* mma_done = o_ready + 4;
  uint64_t* wg0_started = mma_done + 1;    // Q tile 0's first P tile is published
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_TMEM);
  float* s_vs = reinterpret_cast<float*>(smem + L::OFF_VS);
  int* s_nlist = reinterpret_cast<int*>(smem + L::OFF_NLIST);
  uint32_t* s_list = reinterpret_cast<uint32_t*>(smem + L::OFF_LIST);
  float* s_ks = reinterpret_cast<float*>(s_list + a.nkt);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int qp, b, h;
  decode_work(a, blockIdx.x, qp, b, h);
  const int g = h / a.G;
  const int bhk = b * a.Hkv + g;
  const CtaSeq cs = cta_seq(a, b, h, g);
  // the softmax warps read the sequence view from shared memory when they
  // need it (fewer registers held through their loop)
  __shared__ CtaSeq s_cs;
  const int qt0 = 2 * qp;
  // a variable-length call sizes the grid by its longest sequence: CTAs
  // beyond this sequence's tiles leave before any setup
  if (qt0 >= cs.nqt) return;
  const bool has1 = qt0 + 1 < cs.nqt;

  // ------------------------------------------------------------ setup
  if (warp == 0) {
    int count = 0;
    uint32_t orf = 0;
    for (int base = 0; base < cs.nkt; base += 32) {
      const int kt = base + lane;
      uint32_t f = 0;
      if (kt < cs.nkt) {
        f = tile_flags(a, cs, b, h, qt0, 0, kt);
        if (has1) f |= tile_flags(a, cs, b, h, qt0 + 1, 1, kt);
      }
      const unsigned bal = __ballot_sync(0xffffffffu, (f & 3u) != 0);
      if (f & 3u) {
        const int pos = count + __popc(bal & ((1u << lane) - 1u));
        s_list[pos] = ((uint32_t)kt << 8) | f;
        s_ks[pos] = a.k_scale[cs.ks0 + kt];
      }
      count += __popc(bal);
      orf |= f;
    }
    orf = __reduce_or_sync(0xffffffffu, orf);
    if (lane == 0) {
      s_nlist[0] = count;
      s_nlist[1] = (int)orf;
    }
  } else if (warp == 1 && lane == 0) {
    s_cs = cs;
    mbar_init(q_full, 1);
    for (int s = 0; s < ATT_STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], ATT_ISSUERS);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&p_full[i], 128);
      mbar_init(&o_ready[i], 1);
    }
    mbar_init(mma_done, ATT_ISSUERS);
    mbar_init(wg0_started, 128);
    fence_mbar_init();
  } else if (warp == 9) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  } else if (warp == 8 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  for (int c = threadIdx.x; c < D; c += blockDim.x) s_vs[c] = a.v_scale[(int64_t)bhk * D + c];
  // operands of the S init: f16 512.0 (0x6000) everywhere in A, 1536.0
  // (0x6600) in B; K = 16 products of 786432 sum exactly to 1.5*2^23
  for (int i = threadIdx.x; i < 2048; i += blockDim.x)
    reinterpret_cast<uint32_t*>(sInit)[i] = i < 1024 ? 0x60006000u : 0x66006600u;
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int ntile = s_nlist[0];
  const uint32_t orf = (uint32_t)s_nlist[1];

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(ATT_REGS_LOW));
    if (warp == 8) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      const bool act0 = orf & 1u, act1 = (orf >> 1) & 1u;
      mbar_arrive_expect_tx(q_full, (uint32_t)((act0 ? L::Q_BYTES : 0) + (act1 ? L::Q_BYTES : 0)));
      if (act0) tma_load_2d(sQ, &tmQ, q_full, 0, (int)(cs.qrow0 + qt0 * ATT_BM));
      if (act1) tma_load_2d(sQ + L::Q_BYTES, &tmQ, q_full, 0, (int)(cs.qrow0 + (qt0 + 1) * ATT_BM));
      int issued = 0;
      for (int idx = 0; idx < ntile; ++idx) {
        const int st = idx % ATT_STAGES, rd = idx / ATT_STAGES;
        if (idx >= ATT_STAGES && !mbar_wait(&kv_empty[st], (rd - 1) & 1, SITE_KV_EMPTY)) break;
        const int kt = (int)(s_list[idx] >> 8);
        mbar_arrive_expect_tx(&kv_full[st], (uint32_t)(L::K_BYTES + L::V_BYTES));
        tma_load_2d(sK + st * L::K_BYTES, &tmK, &kv_full[st], 0, (int)(cs.krow0 + kt * ATT_BN));
        tma_load_2d(sV + st * L::V_BYTES, &tmV, &kv_full[st], 0, (int)(cs.krow0 + kt * ATT_BN));
        ++issued;
      }
      // every copy issued above lands before the CTA's shared memory is
      // released, also when a wait gave up (otherwise already the case: the
      // issuers wait for every tile)
      mbar_drain(q_full, 0);
      for (int st = 0; st < ATT_STAGES && st < issued; ++st) {
        const int last = st + (issued - 1 - st) / ATT_STAGES * ATT_STAGES;
        mbar_drain(&kv_full[st], (last / ATT_STAGES) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 9 || warp == 10) {
    // ---------------------------------------------------------- MMA issuers
    if (lane == 0) {
      constexpr uint32_t IDESC_QK = instr_desc(kDS32, kS8, kS8, ATT_BM, ATT_BN);
      constexpr uint32_t IDESC_INIT = instr_desc(kDF32, 0u, 0u, ATT_BM, ATT_BN);
      const uint64_t dInitA = smem_desc(smem_u32(sInit), 256, 32);
      const uint64_t dInitB = smem_desc(smem_u32(sInit) + 4096, 256, 32);
      constexpr uint32_t IDESC_PV = instr_desc(kDF32, kE4M3, kE4M3, ATT_BM, D) | kBMajorMN;
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aP = smem_u32(sP);
      // One issuing thread per Q tile (warp 9: Q tile 0, warp 10: Q tile 1).
      // A thread is held by each tcgen05.mma for about its execution time,
      // so the waits and commits of one thread (~50-100 clocks each) leave
      // the tensor pipe idle unless the other thread's MMAs fill it.  Per
      // visible list position e the thread issues QK(e), then PV of its
      // previous visible position, each gated by one bounded wait; it then
      // releases, in list order, every K/V stage it is done with by a
      // commit (which arrives only after its MMAs reading the stage have
      // completed).  A stage is refilled once both threads have released it
      // (kv_empty counts 2).  Before releasing position p a thread waits
      // until p's tile has arrived: otherwise a thread with nothing to read
      // (a position its Q tile does not see, or no Q tile at all) would
      // arrive for p and p + 3 before the other thread released p, and the
      // stage would be refilled while still being read.
      const int i = warp - 9;
      uint32_t nqk = 0u, npv = 0u;
      int rel = 0;   // next list position this thread releases
      auto release_to = [&](int last) -> bool {
        for (; rel <= last; ++rel) {
          if (!mbar_wait(&kv_full[rel % ATT_STAGES], (rel / ATT_STAGES) & 1, SITE_KV_FULL))
            return false;
          tc_commit(&kv_empty[rel % ATT_STAGES]);
        }
        return true;
      };
      auto issue_pv = [&](int ep) -> bool {
        if (!mbar_wait(&p_full[i * 2 + (npv & 1u)], (npv >> 1) & 1u, SITE_P_FULL)) return false;
        tc_fence_after();
        const uint32_t tO = tmem + (uint32_t)(i * 256 + 128);
        const uint32_t pa = aP + (i * 2 + (npv & 1u)) * L::P_BYTES;
        const uint32_t va = aV + (ep % ATT_STAGES) * L::V_BYTES;
#pragma unroll
        for (int kk = 0; kk < ATT_BN / 32; ++kk)
          mma_f8f6f4(tO, smem_desc(pa + 32 * kk, 1024, 128),
                     smem_desc(va + L::V_KSTEP * kk, L::QK_SBO, L::QK_SWIZZLE), IDESC_PV,
                     (npv > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&o_ready[i * 2 + (npv & 1u)]);
        ++npv;
        return release_to(ep);
      };
      bool ok = mbar_wait(q_full, 0, SITE_Q_FULL);
      tc_fence_after();
      int ep = -1;   // previous visible position
      for (int e = 0; ok && e < ntile; ++e) {
        if (!((s_list[e] >> i) & 1u)) continue;
        ok = mbar_wait(&kv_full[e % ATT_STAGES], (e / ATT_STAGES) & 1, SITE_KV_FULL) &&
             mbar_wait(&s_free[i], nqk & 1u, SITE_S_FREE);
        if (!ok) break;
        tc_fence_after();
        const uint32_t tS = tmem + (uint32_t)(i * 256);
        const uint32_t qa = aQ + i * L::Q_BYTES, ka = aK + (e % ATT_STAGES) * L::K_BYTES;
        mma_f16(tS, dInitA, dInitB, IDESC_INIT, 0u);
#pragma unroll
        for (int k = 0; k < D / 32; ++k)
          mma_i8(tS, smem_desc(qa + 32 * k, L::QK_SBO, L::QK_SWIZZLE),
                 smem_desc(ka + 32 * k, L::QK_SBO, L::QK_SWIZZLE), IDESC_QK, 1u);
        tc_commit(&s_full[i]);
        ++nqk;
        if (ep >= 0) ok = issue_pv(ep);
        ep = e;
      }
      if (ok && ep >= 0) ok = issue_pv(ep);
      // positions after this Q tile's last one (or all, if it has none)
      if (ok) ok = release_to(ntile - 1);
      // every MMA issued above completes before the CTA tears down TMEM
      tc_commit(mma_done);
      // (a wait that gives up because another one failed is followed by the
      // drain: the MMAs still finish before TMEM is freed)
      if (!mbar_wait(mma_done, 0, SITE_MMA_DONE)) mbar_drain(mma_done, 0);
    }
    __syncwarp();
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(ATT_REGS_HIGH));
    // ---------------------------------------------------------- softmax WGs
    const CtaSeq& cs = s_cs;
    const int wg = warp >> 2;
    const int rt = threadIdx.x & 127;
    const int qt = qt0 + wg;
    const int row = qt * ATT_BM + rt;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + (uint32_t)(wg * 256);
    const uint32_t tO = tS + 128;
    const bool tile_exists = qt < cs.nqt;
    const float cq = tile_exists ? a.q_scale[cs.qs0 + qt] * a.c0 : 0.f;
    const uint8_t* mrow = nullptr;           // this row of the mask (bytes or floats)
    if (a.mask && row < cs.Nq) {
      const int bm = a.m_bcast_b ? 0 : b, hm = a.m_bcast_h ? 0 : h;
      const int64_t el = (int64_t)bm * a.m_sb + (int64_t)hm * a.m_sh + (int64_t)row * a.m_sq;
      mrow = reinterpret_cast<const uint8_t*>(a.mask) + el * (a.mask_kind ? 4 : 1);
    }
    // S starts free; each QK^T is preceded by an f16 MMA that sets S to
    // 1.5*2^23, so the int32 sum on top reads as the float 1.5*2^23 + S.
    mbar_arrive(&s_free[wg]);
    // Q tile 1's warpgroup starts once Q tile 0's has published its first P
    // tile (when it has one; a barrier of its own, completed once): the two
    // warpgroups' exponential phases then start half a tile apart instead of
    // contending for MUFU from the first tile on (causal GQA workload at B=4:
    // 7.18 -> 7.09 ms; the masked LLM workload 1.14 -> 1.10 ms).
    bool ok = true;
    if (wg == 1 && (orf & 1u))
      ok = __all_sync(0xffffffffu, mbar_wait(wg0_started, 0, SITE_P_FULL));
    float m_ref = -INFINITY, l = 0.f;
    uint32_t n = 0;
    for (int idx = 0; ok && idx < ntile; ++idx) {
      const uint32_t e = s_list[idx];
      if (!((e >> wg) & 1u)) continue;
      const int kt = (int)(e >> 8);
      const bool need = (e >> (2 + wg)) & 1u;
      const bool part = (e >> (4 + wg)) & 1u;
      const float c = cq * s_ks[idx];
      const uint32_t buf = n & 1u;
      uint8_t* ptile = sP + (wg * 2 + buf) * L::P_BYTES;
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[wg], n & 1, SITE_S_FULL));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[128];
      SAGE_TMEM_LD128(tS, sr);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&s_free[wg]);
      // the P buffer this tile writes was read by PV(n-2): test it now (its
      // latency overlaps the row max), wait below only if it was not done
      const bool pbuf_free =
          n < 2 || mbar_test(&o_ready[wg * 2 + buf], ((n - 2) >> 1) & 1);

      // sr holds 1.5*2^23 + S as float bits; hidden keys -> 0.0 (below every score)
      uint32_t vis[4] = {~0u, ~0u, ~0u, ~0u};
      const bool biased = FMASK && part;
      if (need) {
        tile_visibility(a, cs, kt, row, part && !FMASK, mrow, vis);
        if (!biased) {
#pragma unroll
          for (int j = 0; j < 128; ++j)
            if (!((vis[j >> 5] >> (j & 31)) & 1u)) sr[j] = 0u;
        }
      }
      float mt;   // tile max of the scaled scores (-inf if this row sees no key here)
      if (FMASK && biased) {
        // float mask: sr <- S * c + bias * log2(e) (-inf for hidden keys),
        // in 32-key chunks of 16-byte bias loads
        const float* brow = mrow ? reinterpret_cast<const float*>(mrow) + kt * ATT_BN : nullptr;
        float bm0 = -INFINITY, bm1 = -INFINITY;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          float bb[32];
          const int key0 = kt * ATT_BN + ch * 32;
          if (brow && key0 + 32 <= cs.Nk && (reinterpret_cast<uintptr_t>(brow) & 15u) == 0) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 f = __ldg(reinterpret_cast<const float4*>(brow + ch * 32) + i);
              bb[4 * i] = f.x; bb[4 * i + 1] = f.y; bb[4 * i + 2] = f.z; bb[4 * i + 3] = f.w;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              bb[i] = (brow && key0 + i < cs.Nk) ? __ldg(brow + ch * 32 + i) : -INFINITY;
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int j = ch * 32 + i;
            const float t = ((vis[j >> 5] >> (j & 31)) & 1u)
                                ? fmaf(__uint_as_float(sr[j]) - MAGIC_F, c, bb[i] * LOG2E_F)
                                : -INFINITY;
            sr[j] = __float_as_uint(t);
            if (i & 1) bm1 = fmaxf(bm1, t); else bm0 = fmaxf(bm0, t);
          }
        }
        mt = fmaxf(bm0, bm1);
      } else {
        float m0 = __uint_as_float(sr[0]), m1 = __uint_as_float(sr[1]);
        float m2 = __uint_as_float(sr[2]), m3 = __uint_as_float(sr[3]);
#pragma unroll
        for (int j = 4; j < 128; j += 8) {
          m0 = max3f(m0, __uint_as_float(sr[j]), __uint_as_float(sr[j + 1]));
          m1 = max3f(m1, __uint_as_float(sr[j + 2]), __uint_as_float(sr[j + 3]));
          m2 = max3f(m2, __uint_as_float(sr[j + 4]), __uint_as_float(sr[j + 5]));
          m3 = max3f(m3, __uint_as_float(sr[j + 6]), __uint_as_float(sr[j + 7]));
        }
        const float mx = max3f(m0, m1, fmaxf(m2, m3));
        mt = mx >= 4194304.f ? (mx - MAGIC_F) * c : -INFINITY;
      }
      const float m_new = fmaxf(m_ref, mt);
      const float m_use = m_new == -INFINITY ? 0.f : m_new;
      const float alpha = m_new == m_ref ? 1.f : ex2_approx(m_ref - m_use);
      const float bias = LOG2_448 - m_use;

      // the P buffer being overwritten was read by PV(n-2); O is touched only
      // once PV(n-1) has completed
      if (!__all_sync(0xffffffffu, pbuf_free)) {
        ok = __all_sync(0xffffffffu, mbar_wait(&o_ready[wg * 2 + buf], ((n - 2) >> 1) & 1,
                                                SITE_O_READY));
        if (!ok) break;
      }
      float rs;
      if constexpr (FMASK) {
        rs = biased ? exp_tile<true, true>(sr, vis, c, bias, ptile, rt)
                    : need ? exp_tile<true>(sr, vis, c, bias, ptile, rt)
                           : exp_tile<false>(sr, vis, c, bias, ptile, rt);
      } else {
        rs = need ? exp_tile<true>(sr, vis, c, bias, ptile, rt)
                  : exp_tile<false>(sr, vis, c, bias, ptile, rt);
      }
      if (n > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        const uint32_t pb = (n - 1) & 1u;
        ok = __all_sync(0xffffffffu, mbar_wait(&o_ready[wg * 2 + pb], ((n - 1) >> 1) & 1,
                                                SITE_O_READY));
        if (!ok) break;
        tc_fence_after();
        const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
        for (int cb = 0; cb < D; cb += 32) {
          uint32_t o[32];
          SAGE_TMEM_LD32(tO + cb, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            float x0, x1;
            f2_unpack(f2_mul(f2_pack(__uint_as_float(o[i]), __uint_as_float(o[i + 1])), a2), x0, x1);
            o[i] = __float_as_uint(x0);
            o[i + 1] = __float_as_uint(x1);
          }
          SAGE_TMEM_ST32(tO + cb, o);
        }
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[wg * 2 + buf]);
      if (wg == 0 && n == 0) mbar_arrive(wg0_started);
      l = l * alpha + rs;
      m_ref = m_new;
      ++n;
    }
    if (ok && n > 0) {
      const uint32_t pb = (n - 1) & 1u;
      ok = __all_sync(0xffffffffu,
                      mbar_wait(&o_ready[wg * 2 + pb], ((n - 1) >> 1) & 1, SITE_O_READY));
      tc_fence_after();
    }
    if (tile_exists) {
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      const bool live = ok && n > 0;
      char* obase = reinterpret_cast<char*>(a.out) + (cs.out0 + (int64_t)row * a.out_sn) * 2;
#pragma unroll
      for (int cb = 0; cb < D; cb += 32) {
        uint32_t o[32];
        if (live) {
          SAGE_TMEM_LD32(tO + cb, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
        if (row < cs.Nq) {
          if (a.out_fp16)
            store_out_chunk<D, __half>(a, reinterpret_cast<__half*>(obase), cb, o, s_vs, inv_l);
          else
            store_out_chunk<D, __nv_bfloat16>(a, reinterpret_cast<__nv_bfloat16*>(obase), cb, o,
                                              s_vs, inv_l);
        }
      }
      if (a.return_lse && row < cs.Nq) {
        float v = -INFINITY;
        if (l > 0.f)
          v = (m_ref + log2f(l) - LOG2_448) * LN2_F + a.sm_scale * a.qdk[cs.tok0 + row];
        a.lse[cs.tok0 + row] = v;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------ mask classes
// One CTA per (mask batch/head, q tile, k tile): 0 = nothing visible,
// 1 = everything visible, 2 = mixed.  Only rows < Nq and keys < Nk count.
// For a float mask: 0 = every entry -inf, 1 = every entry 0 (no bias),
// 2 = otherwise.  Strides in elements.
__global__ void __launch_bounds__(256) mask_classify_kernel(const void* __restrict__ mask,
                                                            int kind, int64_t sb, int64_t sh,
                                                            int64_t sq, int Hm, int Nq, int Nk,
                                                            int nqt, int nkt,
                                                            uint8_t* __restrict__ cls) {
  const int kt = blockIdx.x, qt = blockIdx.y, bhm = blockIdx.z;
  const int bm = bhm / Hm, hm = bhm % Hm;
  const int64_t base = (int64_t)bm * sb + (int64_t)hm * sh;
  int any = 0, all = 1;
  for (int idx = threadIdx.x; idx < ATT_BM * ATT_BN; idx += blockDim.x) {
    const int r = qt * ATT_BM + idx / ATT_BN, c = kt * ATT_BN + idx % ATT_BN;
    if (r < Nq && c < Nk) {
      const int64_t e = base + (int64_t)r * sq + c;
      if (kind == 0) {
        const int v = static_cast<const uint8_t*>(mask)[e] != 0;
        any |= v;
        all &= v;
      } else {
        const float x = static_cast<const float*>(mask)[e];
        any |= x != -INFINITY;
        all &= x == 0.f;
      }
    }
  }
  any = __syncthreads_or(any);
  all = __syncthreads_and(all);
  if (threadIdx.x == 0) cls[((int64_t)bhm * nqt + qt) * nkt + kt] = any ? (all ? 1 : 2) : 0;
}

// ------------------------------------------------------------ test kernels
// One 128x128 int32 tile of Q K^T through the same TMA maps, descriptors
// and kind::i8 MMA chain as the attention kernel.
template <int D>
__global__ void __launch_bounds__(128, 1)
    debug_qk_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    int qrow, int krow, int32_t* __restrict__ tile) {
  using L = AttnLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sQ = smem;
  uint8_t* sK = smem + L::Q_BYTES;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::Q_BYTES + L::K_BYTES);
  uint32_t* slot = reinterpret_cast<uint32_t*>(bar + 2);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 32) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&bar[0], L::Q_BYTES + L::K_BYTES);
    tma_load_2d(sQ, &tmQ, &bar[0], 0, qrow);
    tma_load_2d(sK, &tmK, &bar[0], 0, krow);
    if (mbar_wait(&bar[0], 0, SITE_DEBUG)) {
      tc_fence_after();
      constexpr uint32_t IDESC = instr_desc(kDS32, kS8, kS8, ATT_BM, ATT_BN);
#pragma unroll
      for (int k = 0; k < D / 32; ++k)
        mma_i8(tmem, smem_desc(smem_u32(sQ) + 32 * k, L::QK_SBO, L::QK_SWIZZLE),
               smem_desc(smem_u32(sK) + 32 * k, L::QK_SBO, L::QK_SWIZZLE), IDESC, k > 0 ? 1u : 0u);
    } else {
      mbar_drain(&bar[0], 0);   // the copies land before shared memory is released
    }
    tc_commit(&bar[1]);
  }
  __syncwarp();
  const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar[1], 0, SITE_DEBUG));
  tc_fence_after();
  const int r = threadIdx.x;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
#pragma unroll
  for (int cb = 0; cb < 128; cb += 32) {
    uint32_t v[32];
    SAGE_TMEM_LD32(tmem + lane_base + cb, v);
    tmem_wait_ld();
    if (ok)
      for (int i = 0; i < 32; ++i) tile[r * 128 + cb + i] = (int32_t)v[i];
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    if (!ok) mbar_drain(&bar[1], 0);   // the MMAs finish before TMEM is freed
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// One P (threads -> swizzled smem) times V^T (TMA) tile, FP32 result.
template <int D>
__global__ void __launch_bounds__(128, 1)
    debug_pv_kernel(const __grid_constant__ CUtensorMap tmV, int vrow, int vcol,
                    const uint8_t* __restrict__ p, float* __restrict__ acc) {
  using L = AttnLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sP = smem;
  uint8_t* sV = smem + L::P_BYTES;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::P_BYTES + L::V_BYTES);
  uint32_t* slot = reinterpret_cast<uint32_t*>(bar + 2);
  const int warp = threadIdx.x >> 5;
  const int r = threadIdx.x;
  if (threadIdx.x == 32) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(slot, 128);
    tmem_relinquish();
  }
  uint32_t pk[32];
  for (int i = 0; i < 32; ++i) pk[i] = __ldg(reinterpret_cast<const uint32_t*>(p + r * 128) + i);
  store_p_row(sP, r, pk);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&bar[0], L::V_BYTES);
    tma_load_2d(sV, &tmV, &bar[0], vcol, vrow);
    if (mbar_wait(&bar[0], 0, SITE_DEBUG)) {
      tc_fence_after();
      constexpr uint32_t IDESC = instr_desc(kDF32, kE4M3, kE4M3, ATT_BM, D) | kBMajorMN;
#pragma unroll
      for (int k = 0; k < ATT_BN / 32; ++k)
        mma_f8f6f4(tmem, smem_desc(smem_u32(sP) + 32 * k, 1024, 128),
                   smem_desc(smem_u32(sV) + L::V_KSTEP * k, L::QK_SBO, L::QK_SWIZZLE), IDESC,
                   k > 0 ? 1u : 0u);
    } else {
      mbar_drain(&bar[0], 0);   // the copy lands before shared memory is released
    }
    tc_commit(&bar[1]);
  }
  __syncwarp();
  const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar[1], 0, SITE_DEBUG));
  tc_fence_after();
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
#pragma unroll
  for (int cb = 0; cb < D; cb += 32) {
    uint32_t v[32];
    SAGE_TMEM_LD32(tmem + lane_base + cb, v);
    tmem_wait_ld();
    if (ok)
      for (int i = 0; i < 32; ++i) acc[r * D + cb + i] = __uint_as_float(v[i]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    if (!ok) mbar_drain(&bar[1], 0);   // the MMAs finish before TMEM is freed
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// A single thread waits on a barrier that nothing arrives on.
__global__ void debug_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_wait(&bar, 0, SITE_DEBUG, limit_ns);
  }
}

}  // namespace sage
