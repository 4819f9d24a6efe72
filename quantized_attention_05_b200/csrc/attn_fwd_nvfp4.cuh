// attn_fwd_nvfp4.cuh -- NVFP4 attention forward for sm_100a
// ("flashinfer.nvfp4_attention_sm120_fwd": pre-quantised FP4 Q/K/V with
// per-vector FP8 scale factors, qk_correction with one row per 128-token Q
// block, unpadded_k_len masking, optional LSE; "sageattn3_blackwell": FP4
// microscaling for Q/K and V).
//
// One CTA owns two 128-row Q tiles of one (batch, Q head) and streams the
// 128-key tiles of its KV head:
//   warp 8   producer: TMA for the packed Q, K and V^T tiles into a
//            4-stage ring, and the scale factors staged in shared memory in
//            the layout tcgen05.cp expects (for every 64-element K block a
//            512-byte block: row r's four scale factors as one 32-bit word
//            at 16*(r%32) + 4*(r/32)), read from global memory one tile ahead;
//   warp 11  the qk_correction row of each Q tile for the stage's key tile
//            as bf16 hi + lo, the B operand of one bf16 MMA that adds it to
//            S (also read one tile ahead);
//   warps 9, 10  MMA issuers, one thread each: warp 9 every QK^T
//            (tcgen05.cp of the K scale factors into TMEM, tcgen05.mma
//            kind::mxf4nvf4 with 16-element E4M3 block scales into the one S
//            accumulator the Q tiles take turns on, then S += qk_correction
//            by a kind::f16 MMA onto the same fp32 accumulator), warp 10
//            every PV (V and P scale factors, O_t += P_t V into TMEM, fp32);
//   warps 0-7  two softmax warpgroups, one per Q tile, one thread per row:
//            the 128 scores of a tile (the correction already in S), masking,
//            the exact running max, exp2, P' = 2688 * p quantised per 16 keys
//            to E2M1 with an E4M3 scale (written in the 64-byte-swizzled
//            K-major layout of the MMA), O rescaled in TMEM when the running
//            max moves; epilogue O / l and LSE.
// TMEM: S 128 columns, O 2 x 128 columns, scale factors 40 columns.  An S
// buffer per Q tile (as in the INT8 kernel) would leave no columns for the
// scale factors; with one shared S buffer a Q tile's next QK^T waits only
// until the other tile has read S, which the softmax of a tile outlasts.
#pragma once

#include "attn_fwd_i8f8.cuh"
#include "quantize_nvfp4.cuh"

namespace sage {

constexpr int NV_THREADS = 384;   // 3 warpgroups: 2 softmax, 1 producers/MMA
constexpr int NV_PRODUCER_WARP = 8, NV_QK_WARP = 9, NV_PV_WARP = 10, NV_CORR_WARP = 11;
constexpr int NV_STAGES = 4;      // K/V ring depth
// Register split (setmaxnreg): the producer/MMA warpgroup keeps NV_REGS_LOW
// per thread, the softmax warpgroups grow to NV_REGS_HIGH; the host checks
// that the sum fits the launch's register file.
constexpr int NV_REGS_LOW = 56;
constexpr int NV_REGS_HIGH = 224;
constexpr float LOG2_2688 = 11.392317422778761f;   // log2(448 * 6)

struct NvAttnArgs {
  const uint8_t* q_sf;
  const uint8_t* k_sf;
  const uint8_t* v_sf_t;
  const float* corr;
  const float* qdk;
  void* out;
  int64_t out_sb, out_sh, out_sn;
  int out_fp16;
  float* lse;
  int B, Hq, Hkv, G, Nq, Nk, Nqp, Nkp, nqt, nkt, nqp, L;
  int causal, return_lse, causal_off;
  float c0;       // sm_scale * log2(e)
  float sm_scale;
};

template <int D>
struct NvLayout {
  static constexpr int ROWB = D / 2;            // bytes per packed Q/K row
  static constexpr int Q_BYTES = 128 * ROWB;
  static constexpr int K_BYTES = 128 * ROWB;
  static constexpr int KSTRIDE = (K_BYTES + 1023) / 1024 * 1024;
  static constexpr int V_BYTES = D * 64;        // V^T tile: D rows x 128 keys
  static constexpr int P_BYTES = 128 * 64;      // P tile: 128 rows x 128 keys
  static constexpr int KB_QK = D / 64;          // 64-element K blocks of QK^T
  static constexpr int SF_BLK = 512;
  static constexpr int QK_SWIZZLE = ROWB;       // 64 or 32 bytes
  static constexpr int QK_SBO = 8 * ROWB;
  static constexpr int OFF_Q = 0;               // [Q tile]
  static constexpr int OFF_K = (2 * Q_BYTES + 1023) / 1024 * 1024;
  static constexpr int OFF_V = OFF_K + NV_STAGES * KSTRIDE;
  static constexpr int OFF_P = OFF_V + NV_STAGES * V_BYTES;     // [Q tile][buffer]
  static constexpr int OFF_QSF = OFF_P + 4 * P_BYTES;           // [Q tile][K block]
  static constexpr int OFF_KSF = OFF_QSF + 2 * KB_QK * SF_BLK;  // [stage][K block]
  static constexpr int OFF_VSF = OFF_KSF + NV_STAGES * KB_QK * SF_BLK;   // [stage][key block]
  static constexpr int OFF_PSF = OFF_VSF + NV_STAGES * 2 * SF_BLK;       // [Q tile][buffer][key block]
  // qk_correction row of each stage and Q tile as the B operand of one bf16
  // MMA (128 keys x K = 16, 32-byte rows: (hi, lo, 0, ...) in one 16-byte
  // chunk, zeros in the other), and the A operand (1, 1, 0, ...) in both
  // chunks of every row: the MMA adds hi + lo of key j's correction to every
  // S row.
  static constexpr int OFF_CORR = (OFF_PSF + 4 * 2 * SF_BLK + 1023) / 1024 * 1024;  // [stage][Q tile]
  static constexpr int OFF_ONES = OFF_CORR + NV_STAGES * 2 * 4096;
  static constexpr int OFF_BAR = OFF_ONES + 4096;
  // q_full, kv_full[S], kv_empty[S], s_full[2], s_free[2], p_full[2][2],
  // o_ready[2][2], mma_done
  static constexpr int NBAR = 1 + 2 * NV_STAGES + 2 + 2 + 4 + 4 + 1;
  static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
  static constexpr int OFF_NLIST = (OFF_TMEM + 16 + 15) / 16 * 16;
  static constexpr int OFF_LIST = OFF_NLIST + 16;
  static constexpr size_t bytes(int nkt) { return 1024 + OFF_LIST + (size_t)nkt * 4; }
  // TMEM columns: one S buffer the two Q tiles take turns on, O of each Q
  // tile, then the scale factors (4 columns per 64-element block)
  static constexpr uint32_t T_S = 0, T_O = 128, T_SFQ = 384, T_SFK = T_SFQ + 8 * KB_QK,
                            T_SFV = T_SFK + 4 * KB_QK, T_SFP = T_SFV + 8;
};
static_assert(NvLayout<128>::bytes(ATT_MAX_NKT) <= 232448, "nvfp4 attention smem");
static_assert(NvLayout<128>::T_SFP + 8 <= 512, "nvfp4 attention tmem");

// Block-scaled FP4 MMA: D[tmem] (+)= (A * sfa) (B * sfb)^T, scale factors in TMEM.
__device__ __forceinline__ void mma_nvfp4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// Copy one 512-byte scale-factor block (32 rows x 16 bytes in shared memory,
// no swizzle) into 4 TMEM columns, broadcast to the four lane quarters.
__device__ __forceinline__ void sf_copy(uint32_t tmem_col, uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
  d |= (uint64_t)(128u >> 4) << 32;   // 8-row groups 128 bytes apart
  d |= (uint64_t)1u << 46;            // descriptor version
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(tmem_col), "l"(d)
               : "memory");
}

// Instruction descriptor of the block-scaled MMA: E2M1 A and B (format 1),
// E4M3 scale factors (bit 23 = 0), K-major, K = 64, N >> 3 at 17, M >> 4 at 24.
__host__ __device__ constexpr uint32_t nv_idesc(uint32_t M, uint32_t N) {
  return (1u << 7) | (1u << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

// Stage the scale factors of 128 rows (row-major, D/16 bytes each, rows from
// `src` with `row_stride` bytes) into the tcgen05.cp layout at `dst`: the
// four scale factors of a 64-element block of row r form one word at
// block*512 + 16*(r % 32) + 4*(r / 32).  Rows >= nrows become 0.
template <int NSF>
__device__ __forceinline__ void stage_sf(uint8_t* dst, const uint8_t* src, int64_t row_stride,
                                         int nrows, int lane) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = lane + 32 * i;
    uint32_t w[NSF / 4];
    if (r < nrows) {
      const uint8_t* p = src + (int64_t)r * row_stride;
#pragma unroll
      for (int b = 0; b < NSF / 4; ++b) w[b] = *reinterpret_cast<const uint32_t*>(p + 4 * b);
    } else {
#pragma unroll
      for (int b = 0; b < NSF / 4; ++b) w[b] = 0u;
    }
#pragma unroll
    for (int b = 0; b < NSF / 4; ++b)
      *reinterpret_cast<uint32_t*>(dst + b * 512 + 16 * (r & 31) + 4 * (r >> 5)) = w[b];
  }
}

// The same staging in two halves, so that a tile's global loads can be in
// flight while the producer waits for a free stage: load_sf reads one
// lane's four rows into registers, store_sf writes them in the layout above.
template <int NSF>
struct SfRegs {
  uint32_t w[4][NSF / 4];
};
template <int NSF>
__device__ __forceinline__ void load_sf(SfRegs<NSF>& r, const uint8_t* src, int64_t row_stride,
                                        int nrows, int lane) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = lane + 32 * i;
#pragma unroll
    for (int b = 0; b < NSF / 4; ++b)
      r.w[i][b] = row < nrows ? __ldg(reinterpret_cast<const uint32_t*>(src + (int64_t)row * row_stride) + b)
                              : 0u;
  }
}
template <int NSF>
__device__ __forceinline__ void store_sf(uint8_t* dst, const SfRegs<NSF>& r, int lane) {
  // the lane's rows lane + 32i are the four words of one 16-byte chunk
#pragma unroll
  for (int b = 0; b < NSF / 4; ++b)
    *reinterpret_cast<uint4*>(dst + b * 512 + 16 * lane) = make_uint4(r.w[0][b], r.w[1][b], r.w[2][b], r.w[3][b]);
}

// The 16-key vectors of one thread's row: P' = 2688 * p quantised to E2M1
// codes with an E4M3 scale per vector, written into the row of the P tile
// (64-byte-swizzled K-major: 16-byte chunk c of row r at r*64 + (c ^ ((r/2) % 4))*16)
// and its scale words; returns the sum of the unquantised p.  The scale of a
// vector depends only on its largest score: amax = the p of that score (same
// fma and ex2 as the element itself; 0 when the whole vector is hidden), sf =
// e4m3(amax / 6); the eight scales come first, so the codes wait on no long
// chain.
template <bool NEED>
__device__ __forceinline__ float nv_exp_tile(const uint32_t* sr, const uint32_t* vis,
                                             const float* vmax, float c, float bias,
                                             const float* s_inv, uint8_t* prow, int rt,
                                             uint32_t* sfw) {
  const uint64_t c2 = f2_pack(c, c), b2 = f2_pack(bias, bias);
  float inv[8], q[8];
#pragma unroll
  for (int vv = 0; vv < 8; ++vv) q[vv] = div6_rn(ex2_approx(fmaf(vmax[vv], c, bias)));
  // the eight scale codes, four per conversion statement, already in the
  // byte order of the scale-factor words
  sfw[0] = cvt_e4m3x4(q[0], q[1], q[2], q[3]);
  sfw[1] = cvt_e4m3x4(q[4], q[5], q[6], q[7]);
#pragma unroll
  for (int vv = 0; vv < 8; ++vv) inv[vv] = s_inv[(sfw[vv >> 2] >> (8 * (vv & 3))) & 0xFFu];
  uint64_t acc = f2_pack(0.f, 0.f);
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) {
    uint32_t w[4];
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int vv = 2 * ch + h2;
      const uint64_t inv2 = f2_pack(inv[vv], inv[vv]);
      float yq[16];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int j = vv * 16 + 2 * i;
        const uint64_t y = f2_fma(f2_pack(__uint_as_float(sr[j]), __uint_as_float(sr[j + 1])), c2, b2);
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
        // P' / scale, rounded to E2M1 below
        f2_unpack(f2_mul(p, inv2), yq[2 * i], yq[2 * i + 1]);
      }
      w[2 * h2] = e2m1x8(yq);
      w[2 * h2 + 1] = e2m1x8(yq + 8);
    }
    *reinterpret_cast<uint4*>(prow + ((ch ^ ((rt >> 1) & 3)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  float a0, a1;
  f2_unpack(acc, a0, a1);
  return a0 + a1;
}

template <int D>
__global__ void __launch_bounds__(NV_THREADS, 1)
    attn_fwd_nvfp4_kernel(const __grid_constant__ CUtensorMap tmQ,
                          const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, NvAttnArgs a) {
  using L = NvLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sK = smem + L::OFF_K;
  uint8_t* sV = smem + L::OFF_V;
  uint8_t* sP = smem + L::OFF_P;
  uint8_t* sQsf = smem + L::OFF_QSF;
  uint8_t* sKsf = smem + L::OFF_KSF;
  uint8_t* sVsf = smem + L::OFF_VSF;
  uint8_t* sPsf = smem + L::OFF_PSF;
  uint8_t* sCorrB = smem + L::OFF_CORR;
  uint8_t* sOnes = smem + L::OFF_ONES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + NV_STAGES;
  uint64_t* s_full = kv_empty + NV_STAGES;   // [Q tile]
  uint64_t* s_free = s_full + 2;              // [Q tile]
  uint64_t* p_full = s_free + 2;              // [Q tile * 2 + buffer]
  uint64_t* o_ready = p_full + 4;             // [Q tile * 2 + buffer]
  uint64_t* mma_done = o_ready + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_TMEM);
  int* s_nlist = reinterpret_cast<int*>(smem + L::OFF_NLIST);
  uint32_t* s_list = reinterpret_cast<uint32_t*>(smem + L::OFF_LIST);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ float s_inv[256];   // 1 / value(E4M3 code), 0 for code 0
  __shared__ float s_one[D];     // unit value scales of the shared epilogue
  fill_e4m3_inverse(s_inv);
  for (int i = threadIdx.x; i < D; i += blockDim.x) s_one[i] = 1.f;
  // work: (b, h, pair of Q tiles); causal -> longest rows first
  int b, h, qp;
  {
    const int bid = blockIdx.x, per = a.B * a.Hq;
    if (a.causal) {
      qp = a.nqp - 1 - bid / per;
      b = (bid % per) / a.Hq;
      h = (bid % per) % a.Hq;
    } else {   // Q heads sharing a KV head run side by side (K/V reuse in L2)
      const int j = bid % a.G;
      int t = bid / a.G;
      qp = t % a.nqp;
      t /= a.nqp;
      const int g = t % a.Hkv;
      b = t / a.Hkv;
      h = g * a.G + j;
    }
  }
  const int g = h / a.G;
  const int bhq = b * a.Hq + h, bhk = b * a.Hkv + g;
  const int qt0 = 2 * qp;
  const bool has1 = qt0 + 1 < a.nqt;

  if (warp == 0) {
    // visible key tiles: bit t = Q tile t sees a key of it, bit 2 + t = Q
    // tile t needs per-element masking there
    int count = 0;
    for (int base = 0; base < a.nkt; base += 32) {
      const int kt = base + lane;
      uint32_t f = 0;
      if (kt < a.nkt) {
        const int key_lo = kt * 128, key_hi = key_lo + 127;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (t == 1 && !has1) break;
          const int row_lo = (qt0 + t) * 128, row_hi = min(row_lo + 127, a.Nq - 1);
          const bool vis = key_lo < a.L && !(a.causal && key_lo > row_hi + a.causal_off);
          const bool need = key_hi >= a.L || (a.causal && key_hi > row_lo + a.causal_off);
          if (vis) f |= (1u << t) | (need ? 4u << t : 0u);
        }
      }
      const unsigned bal = __ballot_sync(0xffffffffu, f != 0);
      if (f) s_list[count + __popc(bal & ((1u << lane) - 1u))] = ((uint32_t)kt << 8) | f;
      count += __popc(bal);
    }
    if (lane == 0) s_nlist[0] = count;
  } else if (warp == 1 && lane == 0) {
    mbar_init(q_full, 32);
    for (int s = 0; s < NV_STAGES; ++s) {
      mbar_init(&kv_full[s], 64);   // the producer's and the correction warp's lanes
      mbar_init(&kv_empty[s], 2);   // released by the QK and the PV issuer
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&p_full[i], 128);
      mbar_init(&o_ready[i], 1);
    }
    mbar_init(mma_done, 2);
    fence_mbar_init();
  } else if (warp == NV_QK_WARP) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  } else if (warp == NV_PRODUCER_WARP && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  // A operand of the correction MMA: bf16 1.0 (0x3F80) at k = 0 and 1 of
  // both 16-byte chunks of every row; the correction B tiles start zero (only
  // the first word of each row's data chunk is ever rewritten)
  for (int u = threadIdx.x; u < 256; u += blockDim.x)
    *reinterpret_cast<uint4*>(sOnes + 16 * u) = make_uint4(0x3F803F80u, 0u, 0u, 0u);
  for (int u = threadIdx.x; u < NV_STAGES * 2 * 4096 / 16; u += blockDim.x)
    reinterpret_cast<uint4*>(sCorrB)[u] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int ntile = s_nlist[0];

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(NV_REGS_LOW));
    if (warp == NV_PRODUCER_WARP) {
      // -------------------------------------------------------- producer
      const int ntq = has1 ? 2 : 1;
      for (int t = 0; t < ntq; ++t)
        stage_sf<D / 16>(sQsf + t * L::KB_QK * L::SF_BLK,
                         a.q_sf + ((int64_t)bhq * a.Nqp + (qt0 + t) * 128) * (D / 16), D / 16, 128,
                         lane);
      fence_proxy_async_smem();
      if (lane == 0) {
        mbar_arrive_expect_tx(q_full, (uint32_t)(ntq * L::Q_BYTES));
        for (int t = 0; t < ntq; ++t)
          tma_load_2d(sQ + t * L::Q_BYTES, &tmQ, q_full, 0, bhq * a.Nqp + (qt0 + t) * 128);
      } else {
        mbar_arrive(q_full);
      }
      // Per tile the lane's share of the K and V scale factors is read into
      // registers one tile ahead: the global loads of tile idx+1 are in
      // flight while the producer waits for a free stage and stores tile idx.
      SfRegs<D / 16> ksf;
      SfRegs<8> vsf;
      auto load_tile = [&](int idx) {
        const int kt = (int)(s_list[idx] >> 8);
        load_sf<D / 16>(ksf, a.k_sf + ((int64_t)bhk * a.Nkp + kt * 128) * (D / 16), D / 16, 128, lane);
        load_sf<8>(vsf, a.v_sf_t + (int64_t)bhk * D * (a.Nkp / 16) + kt * 8, a.Nkp / 16, D, lane);
      };
      if (ntile > 0) load_tile(0);
      int issued = 0;
      for (int idx = 0; idx < ntile; ++idx) {
        const int st = idx % NV_STAGES, rd = idx / NV_STAGES;
        if (idx >= NV_STAGES &&
            !__all_sync(0xffffffffu, mbar_wait(&kv_empty[st], (rd - 1) & 1, SITE_KV_EMPTY)))
          break;
        const int kt = (int)(s_list[idx] >> 8);
        store_sf<D / 16>(sKsf + st * L::KB_QK * L::SF_BLK, ksf, lane);
        store_sf<8>(sVsf + st * 2 * L::SF_BLK, vsf, lane);
        if (idx + 1 < ntile) load_tile(idx + 1);
        fence_proxy_async_smem();
        if (lane == 0) {
          mbar_arrive_expect_tx(&kv_full[st], (uint32_t)(L::K_BYTES + L::V_BYTES));
          tma_load_2d(sK + st * L::KSTRIDE, &tmK, &kv_full[st], 0, bhk * a.Nkp + kt * 128);
          tma_load_2d(sV + st * L::V_BYTES, &tmV, &kv_full[st], kt * 64, bhk * D);
        } else {
          mbar_arrive(&kv_full[st]);
        }
        ++issued;
      }
      // every copy issued above lands before the CTA's shared memory is
      // released, also when a wait gave up (otherwise already the case: the
      // issuers wait for every tile)
      if (lane == 0) {
        mbar_drain(q_full, 0);
        for (int st = 0; st < NV_STAGES && st < issued; ++st) {
          const int last = st + (issued - 1 - st) / NV_STAGES * NV_STAGES;
          mbar_drain(&kv_full[st], (last / NV_STAGES) & 1);
        }
      }
      __syncwarp();
    } else if (warp == NV_CORR_WARP) {
      // -------------------------------------------------------- correction rows
      // The qk_correction rows of the stage's key tile for the Q tiles that
      // see it, as the B operand of the correction MMA; read one tile ahead
      // like the scale factors.  Lane l handles keys l, l + 32, l + 64,
      // l + 96 (coalesced loads; its 4-byte stores at 32-byte row strides
      // hit eight banks per eight rows).
      float cv[2][4];
      const float* corr0 = a.corr + ((int64_t)bhq * a.nqt + qt0) * a.Nkp;
      auto load_tile = [&](int idx) {
        const uint32_t e = s_list[idx];
        const int kt = (int)(e >> 8);
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int i = 0; i < 4; ++i)
            cv[t][i] = ((e >> t) & 1u) ? __ldg(corr0 + (int64_t)t * a.Nkp + kt * 128 + lane + 32 * i) : 0.f;
      };
      if (ntile > 0) load_tile(0);
      for (int idx = 0; idx < ntile; ++idx) {
        const int st = idx % NV_STAGES, rd = idx / NV_STAGES;
        if (idx >= NV_STAGES &&
            !__all_sync(0xffffffffu, mbar_wait(&kv_empty[st], (rd - 1) & 1, SITE_KV_EMPTY)))
          break;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          // the correction of key j as bf16 hi + lo (|x - hi - lo| <= 2^-18 |x|),
          // the first word of row j's data chunk in the B tile (the rest of
          // the tile stays zero from the setup)
          uint8_t* tile = sCorrB + (st * 2 + t) * 4096;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int j = lane + 32 * i;
            const float x = cv[t][i];
            const __nv_bfloat16 hi = __float2bfloat16_rn(x);
            const __nv_bfloat16 lo = __float2bfloat16_rn(__fsub_rn(x, __bfloat162float(hi)));
            const uint32_t w =
                (uint32_t)__bfloat16_as_ushort(hi) | ((uint32_t)__bfloat16_as_ushort(lo) << 16);
            const int sw = (j >> 2) & 1;   // 32-byte swizzle: chunk c of row j at (c ^ sw) * 16
            *reinterpret_cast<uint32_t*>(tile + j * 32 + (sw << 4)) = w;
          }
        }
        if (idx + 1 < ntile) load_tile(idx + 1);
        fence_proxy_async_smem();
        mbar_arrive(&kv_full[st]);
      }
      __syncwarp();
    } else if (warp == NV_QK_WARP || warp == NV_PV_WARP) {
      // -------------------------------------------------------- MMA issuers
      // Two issuing threads: warp 9 issues every QK^T (K scale factors,
      // block-scaled FP4 MMAs, the qk_correction MMA) for both Q tiles in
      // list order, warp 10 every PV (V and P scale factors, block-scaled
      // FP4 MMAs).  Each tcgen05.mma or tcgen05.cp holds its thread for
      // about its execution time and each wait or commit costs tens of
      // clocks; two threads overlap one side's waits with the other's MMAs.
      // The Q tiles take turns on the one S buffer: a QK^T waits until the
      // previous user of S has read it.  tcgen05 operations of one thread
      // run in issue order, so a scale-factor copy never overtakes the MMA
      // that reads the previous contents of its columns.  A K/V stage is
      // released once both threads have committed on it.
      if (lane == 0) {
        constexpr uint32_t ID_QK = nv_idesc(128, 128);
        constexpr uint32_t ID_PV = nv_idesc(128, D);
        const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aP = smem_u32(sP);
        bool ok = true;
        if (warp == NV_QK_WARP) {
          ok = mbar_wait(q_full, 0, SITE_Q_FULL);
          tc_fence_after();
          for (int t = 0; t < (has1 ? 2 : 1); ++t)
#pragma unroll
            for (int kb = 0; kb < L::KB_QK; ++kb)
              sf_copy(tmem + L::T_SFQ + 4 * (t * L::KB_QK + kb),
                      smem_u32(sQsf) + (t * L::KB_QK + kb) * L::SF_BLK);
          int prev = -1;           // Q tile of the previous user of S
          uint32_t nuse[2] = {0u, 0u};
          for (int idx = 0; ok && idx < ntile; ++idx) {
            const int st = idx % NV_STAGES;
            const uint32_t f = s_list[idx];
            if (!mbar_wait(&kv_full[st], (idx / NV_STAGES) & 1, SITE_KV_FULL)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int kb = 0; kb < L::KB_QK; ++kb)
              sf_copy(tmem + L::T_SFK + 4 * kb, smem_u32(sKsf) + (st * L::KB_QK + kb) * L::SF_BLK);
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              if (!((f >> t) & 1u)) continue;
              const uint32_t np = prev == 1 ? nuse[1] : nuse[0];   // (nuse stays in registers)
              if (prev >= 0 && !mbar_wait(&s_free[prev], (np - 1u) & 1u, SITE_S_FREE)) {
                ok = false;
                break;
              }
              tc_fence_after();
#pragma unroll
              for (int kb = 0; kb < L::KB_QK; ++kb)
                mma_nvfp4(tmem + L::T_S, smem_desc(aQ + t * L::Q_BYTES + 32 * kb, L::QK_SBO, L::QK_SWIZZLE),
                          smem_desc(aK + st * L::KSTRIDE + 32 * kb, L::QK_SBO, L::QK_SWIZZLE), ID_QK,
                          tmem + L::T_SFQ + 4 * (t * L::KB_QK + kb), tmem + L::T_SFK + 4 * kb,
                          kb > 0 ? 1u : 0u);
              // S += qk_correction of each key (one bf16 MMA onto the fp32 scores)
              mma_f16(tmem + L::T_S, smem_desc(smem_u32(sOnes), 256, 32),
                      smem_desc(smem_u32(sCorrB) + (st * 2 + t) * 4096, 256, 32),
                      instr_desc(kDF32, 1u, 1u, 128, 128), 1u);
              tc_commit(&s_full[t]);
              prev = t;
              ++nuse[t];
            }
            if (!ok) break;
            tc_commit(&kv_empty[st]);
          }
        } else {
          uint32_t npv[2] = {0u, 0u};
          for (int idx = 0; ok && idx < ntile; ++idx) {
            const int st = idx % NV_STAGES;
            const uint32_t f = s_list[idx];
            if (!mbar_wait(&kv_full[st], (idx / NV_STAGES) & 1, SITE_KV_FULL)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int kb = 0; kb < 2; ++kb)
              sf_copy(tmem + L::T_SFV + 4 * kb, smem_u32(sVsf) + (st * 2 + kb) * L::SF_BLK);
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              if (!((f >> t) & 1u)) continue;
              const uint32_t pb = t * 2 + (npv[t] & 1u);
              if (!mbar_wait(&p_full[pb], (npv[t] >> 1) & 1u, SITE_P_FULL)) {
                ok = false;
                break;
              }
              tc_fence_after();
#pragma unroll
              for (int kb = 0; kb < 2; ++kb)
                sf_copy(tmem + L::T_SFP + 4 * kb, smem_u32(sPsf) + (pb * 2 + kb) * L::SF_BLK);
#pragma unroll
              for (int kb = 0; kb < 2; ++kb)
                mma_nvfp4(tmem + L::T_O + 128 * t, smem_desc(aP + pb * L::P_BYTES + 32 * kb, 512, 64),
                          smem_desc(aV + st * L::V_BYTES + 32 * kb, 512, 64), ID_PV,
                          tmem + L::T_SFP + 4 * kb, tmem + L::T_SFV + 4 * kb,
                          (npv[t] > 0 || kb > 0) ? 1u : 0u);
              tc_commit(&o_ready[pb]);
              ++npv[t];
            }
            if (!ok) break;
            tc_commit(&kv_empty[st]);
          }
        }
        // every MMA issued above completes before the CTA tears down TMEM
        tc_commit(mma_done);
        // (a wait that gives up because another one failed is followed by the
        // drain: the MMAs still finish before TMEM is freed)
        if (!mbar_wait(mma_done, 0, SITE_MMA_DONE)) mbar_drain(mma_done, 0);
      }
      __syncwarp();
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(NV_REGS_HIGH));
    // ---------------------------------------------------------- softmax
    const int t = warp >> 2;                  // Q tile of this warpgroup
    const int rt = threadIdx.x & 127;
    const int row = (qt0 + t) * 128 + rt;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + L::T_S;
    const uint32_t tO = tmem + lane_base + L::T_O + 128 * t;
    const bool tile_exists = qt0 + t < a.nqt;
    const float c = a.c0;
    float m_ref = -INFINITY, l = 0.f;
    uint32_t n = 0;
    bool ok = true;
    for (int idx = 0; idx < ntile; ++idx) {
      const uint32_t e = s_list[idx];
      if (!((e >> t) & 1u)) continue;
      const int kt = (int)(e >> 8);
      const bool need = (e >> (2 + t)) & 1u;
      const uint32_t buf = n & 1u, pb = t * 2 + buf;
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[t], n & 1u, SITE_S_FULL));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[128];
      SAGE_TMEM_LD128(tS, sr);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&s_free[t]);
      // the P buffer this tile writes was read by PV(n-2): test it now (its
      // latency overlaps the row max), wait below only if it was not done
      const bool pbuf_free = n < 2 || mbar_test(&o_ready[pb], ((n - 2) >> 1) & 1);
      // S already holds the scores plus qk_correction (added by the MMA)
      uint32_t vis[4] = {~0u, ~0u, ~0u, ~0u};
      if (need) {
        const int key0 = kt * 128;
        int jmax = min(127, a.L - 1 - key0);
        if (a.causal) jmax = min(jmax, row + a.causal_off - key0);
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const int hi = jmax - 32 * w;
          vis[w] = hi >= 31 ? ~0u : (hi < 0 ? 0u : ((2u << hi) - 1u));
        }
#pragma unroll
        for (int j = 0; j < 128; ++j)
          if (!((vis[j >> 5] >> (j & 31)) & 1u)) sr[j] = __float_as_uint(-INFINITY);
      }
      // maxima of the eight 16-key vectors (they also give each vector's P'
      // amax: p is increasing in the score), then of the row
      float vmax[8];
#pragma unroll
      for (int vv = 0; vv < 8; ++vv) {
        const float* x = reinterpret_cast<const float*>(sr) + 16 * vv;
        const float t0 = max3f(x[0], x[1], x[2]), t1 = max3f(x[3], x[4], x[5]);
        const float t2 = max3f(x[6], x[7], x[8]), t3 = max3f(x[9], x[10], x[11]);
        const float t4 = max3f(x[12], x[13], x[14]);
        vmax[vv] = max3f(max3f(t0, t1, t2), max3f(t3, t4, x[15]), -INFINITY);
      }
      const float mx = max3f(max3f(vmax[0], vmax[1], vmax[2]), max3f(vmax[3], vmax[4], vmax[5]),
                             fmaxf(vmax[6], vmax[7]));
      const float mt = mx == -INFINITY ? -INFINITY : mx * c;
      const float m_new = fmaxf(m_ref, mt);
      const float m_use = m_new == -INFINITY ? 0.f : m_new;
      const float alpha = ex2_approx(m_ref - m_use);
      const float bias = LOG2_2688 - m_use;

      if (!__all_sync(0xffffffffu, pbuf_free)) {
        ok = __all_sync(0xffffffffu, mbar_wait(&o_ready[pb], ((n - 2) >> 1) & 1, SITE_O_READY));
        if (!ok) break;
      }
      uint8_t* prow = sP + pb * L::P_BYTES + rt * 64;
      uint32_t sfw[2];
      const float rs = need ? nv_exp_tile<true>(sr, vis, vmax, c, bias, s_inv, prow, rt, sfw)
                            : nv_exp_tile<false>(sr, vis, vmax, c, bias, s_inv, prow, rt, sfw);
      uint8_t* psf = sPsf + pb * 2 * L::SF_BLK + 16 * (rt & 31) + 4 * (rt >> 5);
      *reinterpret_cast<uint32_t*>(psf) = sfw[0];
      *reinterpret_cast<uint32_t*>(psf + L::SF_BLK) = sfw[1];
      if (n > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        const uint32_t po = t * 2 + ((n - 1) & 1u);
        ok = __all_sync(0xffffffffu, mbar_wait(&o_ready[po], ((n - 1) >> 1) & 1, SITE_O_READY));
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
      mbar_arrive(&p_full[pb]);
      l = l * alpha + rs;
      m_ref = m_new;
      ++n;
    }
    if (ok && n > 0) {
      const uint32_t po = t * 2 + ((n - 1) & 1u);
      ok = __all_sync(0xffffffffu, mbar_wait(&o_ready[po], ((n - 1) >> 1) & 1, SITE_O_READY));
      tc_fence_after();
    }
    if (tile_exists) {
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      const bool live = ok && n > 0;
      char* obase = reinterpret_cast<char*>(a.out) +
                    ((int64_t)b * a.out_sb + (int64_t)h * a.out_sh + (int64_t)row * a.out_sn) * 2;
      AttnArgs unused{};
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
        if (row < a.Nq) {
          if (a.out_fp16)
            store_out_chunk<D, __half>(unused, reinterpret_cast<__half*>(obase), cb, o, s_one, inv_l);
          else
            store_out_chunk<D, __nv_bfloat16>(unused, reinterpret_cast<__nv_bfloat16*>(obase), cb, o,
                                              s_one, inv_l);
        }
      }
      if (a.return_lse && row < a.Nq) {
        float v = -INFINITY;
        if (l > 0.f)
          v = (m_ref + log2f(l) - LOG2_2688) * LN2_F + a.sm_scale * a.qdk[(int64_t)bhq * a.Nq + row];
        a.lse[(int64_t)bhq * a.Nq + row] = v;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == NV_QK_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace sage
