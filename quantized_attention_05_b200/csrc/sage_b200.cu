// sage_b200.cu -- the C ABI of include/sage_b200.h: argument validation,
// workspace layout, TMA descriptors, kernel launches, and the chunked
// copy/compute pipeline of the host-buffer calls.  Built as one
// translation unit with the kernel headers (device state such as the status
// word lives here once).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <mutex>

#include "sage_b200.h"
#include "sage_ptx.cuh"
#include "seqs.cuh"
#include "quantize_i8f8.cuh"
#include "attn_fwd_i8f8.cuh"
#include "quantize_nvfp4.cuh"
#include "attn_fwd_nvfp4.cuh"
#include "merge.cuh"
#include "pipe_schedule.h"

using namespace sage;

namespace {

constexpr int kSMs = 148;

int64_t pad128(int64_t n) { return (n + 127) / 128 * 128; }
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool log_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("SAGE_LOG");
    return e && e[0] == '1';
  }();
  return on;
}

// ---------------------------------------------------------------- checks
bool valid_dims(int64_t B, int64_t H, int64_t N, int64_t D) {
  return B >= 1 && H >= 1 && N >= 1 && D >= 1 && B <= (1 << 16) && H <= (1 << 12);
}

sage_status check_tensor(const sage_tensor* t) {
  if (!t || !t->ptr) return SAGE_ERR_INVALID_ARG;
  if (t->dtype != SAGE_BF16 && t->dtype != SAGE_FP16) return SAGE_ERR_INVALID_ARG;
  if (!valid_dims(t->B, t->H, t->N, t->D)) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(t->ptr)) return SAGE_ERR_INVALID_ARG;
  if (t->sn < t->D || t->sn % 8 || t->sh % 8 || t->sb % 8 || t->sh < 0 || t->sb < 0)
    return SAGE_ERR_INVALID_ARG;
  if (t->D != 64 && t->D != 128) return SAGE_ERR_UNSUPPORTED;
  if (t->N > 128 * ATT_MAX_NKT) return SAGE_ERR_UNSUPPORTED;
  return SAGE_OK;
}

sage_status check_qkv_shapes(int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq, int64_t Nk,
                             int64_t D) {
  if (!valid_dims(B, Hq, Nq, D) || !valid_dims(B, Hkv, Nk, D)) return SAGE_ERR_INVALID_ARG;
  if (Hq % Hkv) return SAGE_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return SAGE_ERR_UNSUPPORTED;
  if (Nq > 128 * ATT_MAX_NKT || Nk > 128 * ATT_MAX_NKT) return SAGE_ERR_UNSUPPORTED;
  // TMA row coordinates are int32
  if (B * Hq * pad128(Nq) >= (int64_t(1) << 31) || B * Hkv * pad128(Nk) >= (int64_t(1) << 31) ||
      B * Hkv * D >= (int64_t(1) << 31))
    return SAGE_ERR_UNSUPPORTED;
  return SAGE_OK;
}

// The (batch entry, head) pairs of one launch form a grid's y or z extent,
// which is at most 65535.
constexpr int64_t kMaxGridYZ = 65535;

sage_status check_qkv(const sage_qkv_i8f8* z, bool need_qdk) {
  if (!z) return SAGE_ERR_INVALID_ARG;
  sage_status st = check_qkv_shapes(z->B, z->Hq, z->Hkv, z->Nq, z->Nk, z->D);
  if (st != SAGE_OK) return st;
  if (z->B * z->Hq > kMaxGridYZ) return SAGE_ERR_UNSUPPORTED;
  if (!z->q || !z->q_scale || !z->k || !z->k_scale || !z->k_mean || !z->v || !z->v_scale)
    return SAGE_ERR_INVALID_ARG;
  if (need_qdk && !z->q_dot_kmean) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(z->q) || !aligned16(z->k) || !aligned16(z->v)) return SAGE_ERR_INVALID_ARG;
  return SAGE_OK;
}

sage_status check_mask(const sage_mask* m, int64_t B, int64_t Hq, int64_t Nq, int64_t Nk) {
  if (!m) return SAGE_OK;
  if (!m->ptr) return SAGE_ERR_INVALID_ARG;
  if (m->kind != SAGE_MASK_BOOL && m->kind != SAGE_MASK_FLOAT) return SAGE_ERR_INVALID_ARG;
  if (m->kind == SAGE_MASK_FLOAT && (reinterpret_cast<uintptr_t>(m->ptr) & 3u))
    return SAGE_ERR_INVALID_ARG;
  if (!(m->B == 1 || m->B == B) || !(m->H == 1 || m->H == Hq)) return SAGE_ERR_INVALID_ARG;
  if (m->Nq != Nq || m->Nk != Nk) return SAGE_ERR_INVALID_ARG;
  if (m->sq < Nk || (m->B > 1 && m->sb < 0) || (m->H > 1 && m->sh < 0)) return SAGE_ERR_INVALID_ARG;
  return SAGE_OK;
}

size_t mask_class_bytes(const sage_mask* m, int64_t Nq, int64_t Nk) {
  if (!m) return 0;
  return align256((size_t)m->B * m->H * (pad128(Nq) / 128) * (pad128(Nk) / 128));
}

// ---------------------------------------------------------------- pass A plan
struct QuantPlan {
  int splits, split_tokens;
  size_t part_bytes;  // hi + lo + amax
};

QuantPlan quant_plan(int64_t B, int64_t Hkv, int64_t Nk, int64_t D) {
  const int64_t bh = B * Hkv;
  const int64_t max_split = std::max<int64_t>(1, (Nk + 255) / 256);
  const int64_t want = std::max<int64_t>(1, (8 * kSMs + bh - 1) / bh);
  int64_t s = std::min(want, max_split);
  int64_t t = ((Nk + s - 1) / s + 31) / 32 * 32;
  s = (Nk + t - 1) / t;
  QuantPlan p;
  p.splits = (int)s;
  p.split_tokens = (int)t;
  const size_t n = (size_t)bh * s * D;
  p.part_bytes = align256(n * 8) * 2 + align256(n * 4) + align256((size_t)bh * D * 4);
  return p;
}

// ---------------------------------------------------------------- TMA maps
PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D byte tensor [outer][inner] with rows `row_bytes` apart, box
// [box_outer][box_inner].
bool make_tmap_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                  uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                  CUtensorMapSwizzle sw) {
  auto enc = tmap_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

CUtensorMapSwizzle qk_swizzle(int64_t D) {
  return D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
}

bool make_qkv_tmaps(const sage_qkv_i8f8* z, CUtensorMap* tq, CUtensorMap* tk, CUtensorMap* tv) {
  const int64_t Nqp = pad128(z->Nq), Nkp = pad128(z->Nk), D = z->D;
  return make_tmap_u8(tq, z->q, D, z->B * z->Hq * Nqp, D, (uint32_t)D, 128, qk_swizzle(D)) &&
         make_tmap_u8(tk, z->k, D, z->B * z->Hkv * Nkp, D, (uint32_t)D, 128, qk_swizzle(D)) &&
         make_tmap_u8(tv, z->v, D, z->B * z->Hkv * Nkp, D, (uint32_t)D, 128, qk_swizzle(D));
}

// Dynamic shared memory opt-in, once per device and kernel.
template <typename K>
bool ensure_smem(K kernel, size_t bytes, std::atomic<uint32_t>* flags) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 32) return false;
  const uint32_t bit = 1u << dev;
  if (flags->load(std::memory_order_acquire) & bit) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
      cudaSuccess)
    return false;
  flags->fetch_or(bit, std::memory_order_acq_rel);
  return true;
}

sage_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

// ---------------------------------------------------------------- quantise
// Pass A, stats and pass B for B sequences (dense batch entries or the rows
// of a sequence table); the grids are sized by the longest sequence.
sage_status launch_quantize(const QuantArgs& a, const QuantPlan& plan, int64_t D, bool fp16,
                            cudaStream_t stream) {
  const dim3 gridA(plan.splits, a.B * a.Hkv);
  const int64_t nblocks = (int64_t)a.B * a.Hq * a.max_nqt + 2 * (int64_t)a.B * a.Hkv * a.max_nkt;
  if (nblocks >= (int64_t(1) << 31)) return SAGE_ERR_UNSUPPORTED;
  if (log_enabled())
    std::fprintf(stderr, "[sage] quantize B=%d Hq=%d Hkv=%d Nq=%d Nk=%d D=%lld splits=%d x %d, blocks=%lld\n",
                 a.B, a.Hq, a.Hkv, a.Nq, a.Nk, (long long)D, plan.splits, plan.split_tokens,
                 (long long)nblocks);
  const int nb = (int)nblocks;
  if (D == 128) {
    if (fp16) {
      kmean_vamax_partial_kernel<__half, 128><<<gridA, QUANT_THREADS, 0, stream>>>(a);
      kv_stats_kernel<128><<<a.B * a.Hkv, 128, 0, stream>>>(a);
      quant_blocks_kernel<__half, 128><<<nb, QUANT_THREADS, 0, stream>>>(a);
    } else {
      kmean_vamax_partial_kernel<__nv_bfloat16, 128><<<gridA, QUANT_THREADS, 0, stream>>>(a);
      kv_stats_kernel<128><<<a.B * a.Hkv, 128, 0, stream>>>(a);
      quant_blocks_kernel<__nv_bfloat16, 128><<<nb, QUANT_THREADS, 0, stream>>>(a);
    }
  } else {
    if (fp16) {
      kmean_vamax_partial_kernel<__half, 64><<<gridA, QUANT_THREADS, 0, stream>>>(a);
      kv_stats_kernel<64><<<a.B * a.Hkv, 64, 0, stream>>>(a);
      quant_blocks_kernel<__half, 64><<<nb, QUANT_THREADS, 0, stream>>>(a);
    } else {
      kmean_vamax_partial_kernel<__nv_bfloat16, 64><<<gridA, QUANT_THREADS, 0, stream>>>(a);
      kv_stats_kernel<64><<<a.B * a.Hkv, 64, 0, stream>>>(a);
      quant_blocks_kernel<__nv_bfloat16, 64><<<nb, QUANT_THREADS, 0, stream>>>(a);
    }
  }
  return launch_status();
}

sage_status run_quantize(const sage_tensor* q, const sage_tensor* k, const sage_tensor* v,
                         int smooth_k, const sage_qkv_i8f8* out, void* ws, size_t ws_bytes,
                         cudaStream_t stream) {
  sage_status st;
  if ((st = check_tensor(q)) || (st = check_tensor(k)) || (st = check_tensor(v))) return st;
  if (!out) return SAGE_ERR_INVALID_ARG;
  if (q->dtype != k->dtype || q->dtype != v->dtype) return SAGE_ERR_INVALID_ARG;
  if (k->B != q->B || v->B != q->B || k->H != v->H || k->N != v->N || k->D != q->D ||
      v->D != q->D)
    return SAGE_ERR_INVALID_ARG;
  if ((st = check_qkv(out, false))) return st;
  if (out->B != q->B || out->Hq != q->H || out->Hkv != k->H || out->Nq != q->N ||
      out->Nk != k->N || out->D != q->D)
    return SAGE_ERR_INVALID_ARG;
  const QuantPlan plan = quant_plan(k->B, k->H, k->N, k->D);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SAGE_ERR_INVALID_ARG;
  if (ws_bytes < plan.part_bytes) return SAGE_ERR_WORKSPACE;

  QuantArgs a{};
  a.q = q->ptr;
  a.k = k->ptr;
  a.v = v->ptr;
  a.q_sb = q->sb; a.q_sh = q->sh; a.q_sn = q->sn;
  a.k_sb = k->sb; a.k_sh = k->sh; a.k_sn = k->sn;
  a.v_sb = v->sb; a.v_sh = v->sh; a.v_sn = v->sn;
  a.B = (int)q->B; a.Hq = (int)q->H; a.Hkv = (int)k->H; a.G = a.Hq / a.Hkv;
  a.Nq = (int)q->N; a.Nk = (int)k->N;
  a.Nqp = (int)pad128(q->N); a.Nkp = (int)pad128(k->N);
  a.nqt = a.Nqp / 128; a.nkt = a.Nkp / 128;
  a.smooth_k = smooth_k ? 1 : 0;
  a.splits = plan.splits;
  a.split_tokens = plan.split_tokens;
  const size_t n = (size_t)a.B * a.Hkv * plan.splits * q->D;
  char* w = static_cast<char*>(ws);
  a.part_hi = reinterpret_cast<double*>(w);
  a.part_lo = reinterpret_cast<double*>(w + align256(n * 8));
  a.part_amax = reinterpret_cast<float*>(w + 2 * align256(n * 8));
  a.va = reinterpret_cast<float*>(w + 2 * align256(n * 8) + align256(n * 4));
  a.q8 = out->q; a.q_scale = out->q_scale; a.k8 = out->k; a.k_scale = out->k_scale;
  a.k_mean = out->k_mean; a.v8 = out->v; a.v_scale = out->v_scale; a.qdk = out->q_dot_kmean;
  a.kv_limit = a.Nk;
  a.seqs = nullptr;
  a.max_nqt = a.nqt;
  a.max_nkt = a.nkt;

  return launch_quantize(a, plan, q->D, q->dtype == SAGE_FP16, stream);
}

// ---------------------------------------------------------------- attention
std::atomic<uint32_t> g_smem_set_64{0}, g_smem_set_128{0}, g_smem_set_64f{0}, g_smem_set_128f{0};

sage_status launch_attention(const AttnArgs& a, int64_t D, const CUtensorMap& tq,
                             const CUtensorMap& tk, const CUtensorMap& tv, int64_t grid,
                             cudaStream_t stream) {
  if (grid >= (int64_t(1) << 31)) return SAGE_ERR_UNSUPPORTED;
  const bool fmask = a.mask && a.mask_kind == SAGE_MASK_FLOAT;
  auto kernel = D == 128 ? (fmask ? attn_fwd_i8f8_kernel<128, true> : attn_fwd_i8f8_kernel<128, false>)
                         : (fmask ? attn_fwd_i8f8_kernel<64, true> : attn_fwd_i8f8_kernel<64, false>);
  std::atomic<uint32_t>* flag = D == 128 ? (fmask ? &g_smem_set_128f : &g_smem_set_128)
                                         : (fmask ? &g_smem_set_64f : &g_smem_set_64);
  // the kernel redistributes registers between its warpgroups; that is only
  // safe if the launch provides at least the sum of their shares
  {
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return SAGE_ERR_CUDA;
    if (128 * ATT_REGS_LOW + 256 * ATT_REGS_HIGH > ATT_THREADS * fa.numRegs)
      return SAGE_ERR_UNSUPPORTED;
  }
  const size_t smem = D == 128 ? AttnLayout<128>::bytes(a.nkt) : AttnLayout<64>::bytes(a.nkt);
  const size_t smem_max = D == 128 ? AttnLayout<128>::bytes(ATT_MAX_NKT) : AttnLayout<64>::bytes(ATT_MAX_NKT);
  if (!ensure_smem(kernel, smem_max, flag)) return SAGE_ERR_CUDA;
  kernel<<<(unsigned)grid, ATT_THREADS, smem, stream>>>(tq, tk, tv, a);
  return launch_status();
}

sage_status run_attention(const sage_qkv_i8f8* z, int causal, float sm_scale, int return_lse,
                          const sage_mask* mask, void* out, int32_t out_dtype, int64_t out_sb,
                          int64_t out_sh, int64_t out_sn, float* lse, void* ws, size_t ws_bytes,
                          cudaStream_t stream) {
  sage_status st;
  if ((st = check_qkv(z, return_lse != 0))) return st;
  if (!out || !aligned16(out)) return SAGE_ERR_INVALID_ARG;
  if (out_dtype != SAGE_BF16 && out_dtype != SAGE_FP16) return SAGE_ERR_INVALID_ARG;
  if (out_sn < z->D || out_sn % 8 || out_sh % 8 || out_sb % 8 || out_sh < 0 || out_sb < 0)
    return SAGE_ERR_INVALID_ARG;
  if ((return_lse != 0) != (lse != nullptr)) return SAGE_ERR_INVALID_ARG;
  if (!std::isfinite(sm_scale)) return SAGE_ERR_INVALID_ARG;
  if ((st = check_mask(mask, z->B, z->Hq, z->Nq, z->Nk))) return st;
  const size_t need = mask_class_bytes(mask, z->Nq, z->Nk);
  if (need && (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u))) return SAGE_ERR_INVALID_ARG;
  if (ws_bytes < need) return SAGE_ERR_WORKSPACE;

  AttnArgs a{};
  a.q_scale = z->q_scale; a.k_scale = z->k_scale; a.v_scale = z->v_scale; a.qdk = z->q_dot_kmean;
  a.out = out; a.out_sb = out_sb; a.out_sh = out_sh; a.out_sn = out_sn;
  a.out_fp16 = out_dtype == SAGE_FP16;
  a.lse = lse;
  a.B = (int)z->B; a.Hq = (int)z->Hq; a.Hkv = (int)z->Hkv; a.G = a.Hq / a.Hkv;
  a.Nq = (int)z->Nq; a.Nk = (int)z->Nk;
  a.Nqp = (int)pad128(z->Nq); a.Nkp = (int)pad128(z->Nk);
  a.nqt = a.Nqp / 128; a.nkt = a.Nkp / 128; a.nqp = (a.nqt + 1) / 2;
  a.causal = causal ? 1 : 0;
  a.return_lse = return_lse ? 1 : 0;
  a.causal_off = a.Nk - a.Nq;
  a.seqs = nullptr;
  a.max_nqp = a.nqp;
  const float s = sm_scale > 0.f ? sm_scale : 1.0f / std::sqrt((float)z->D);
  a.sm_scale = s;
  a.c0 = (float)((double)s * 1.4426950408889634);
  if (mask) {
    a.mask = mask->ptr;
    a.mask_kind = mask->kind;
    a.m_sb = mask->sb; a.m_sh = mask->sh; a.m_sq = mask->sq;
    a.m_bcast_b = mask->B == 1; a.m_bcast_h = mask->H == 1;
    a.mask_vec16 = mask->kind == SAGE_MASK_BOOL && aligned16(mask->ptr) && mask->sq % 16 == 0 &&
                   (mask->B == 1 || mask->sb % 16 == 0) && (mask->H == 1 || mask->sh % 16 == 0);
    uint8_t* cls = static_cast<uint8_t*>(ws);
    a.tile_class = cls;
    const int Hm = (int)mask->H;
    mask_classify_kernel<<<dim3(a.nkt, a.nqt, (unsigned)(mask->B * mask->H)), 256, 0, stream>>>(
        mask->ptr, mask->kind, mask->B == 1 ? 0 : mask->sb, mask->H == 1 ? 0 : mask->sh, mask->sq,
        Hm, a.Nq, a.Nk, a.nqt, a.nkt, cls);
    if ((st = launch_status())) return st;
  }
  CUtensorMap tq, tk, tv;
  if (!make_qkv_tmaps(z, &tq, &tk, &tv)) return SAGE_ERR_CUDA;
  const int grid = a.nqp * a.B * a.Hq;
  if (log_enabled())
    std::fprintf(stderr, "[sage] attn B=%d Hq=%d Hkv=%d Nq=%d Nk=%d D=%lld causal=%d grid=%d\n", a.B,
                 a.Hq, a.Hkv, a.Nq, a.Nk, (long long)z->D, a.causal, grid);
  return launch_attention(a, z->D, tq, tk, tv, grid, stream);
}

// ---------------------------------------------------------------- NVFP4 quantise
struct NvPlan {
  QuantPlan k, q;
  size_t k_bytes, q_bytes, qm_bytes, total;
};
NvPlan nv_plan(int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq, int64_t Nk, int64_t D) {
  NvPlan p;
  p.k = quant_plan(B, Hkv, Nk, D);
  p.q = quant_plan(B, Hq, Nq, D);
  const int64_t nqt = pad128(Nq) / 128;
  // per-block means need one split per 128-token block; the global mean uses
  // the reduction plan.  Size for the larger of the two.
  const int64_t qs = std::max<int64_t>(p.q.splits, nqt);
  p.k_bytes = 2 * align256((size_t)B * Hkv * p.k.splits * D * 8);
  p.q_bytes = 2 * align256((size_t)B * Hq * qs * D * 8);
  // the Q means as bf16 hi and lo parts, the correction MMA's B operand
  p.qm_bytes = 2 * align256((size_t)B * Hq * nqt * D * 2);
  p.total = p.k_bytes + p.q_bytes + p.qm_bytes;
  return p;
}

sage_status check_nvfp4(const sage_qkv_nvfp4* z, bool need_qdk) {
  if (!z) return SAGE_ERR_INVALID_ARG;
  sage_status st = check_qkv_shapes(z->B, z->Hq, z->Hkv, z->Nq, z->Nk, z->D);
  if (st != SAGE_OK) return st;
  if (z->B * z->Hq > kMaxGridYZ) return SAGE_ERR_UNSUPPORTED;
  if (!z->q || !z->q_sf || !z->k || !z->k_sf || !z->v_t || !z->v_sf_t || !z->qk_correction ||
      !z->q_mean || !z->k_mean)
    return SAGE_ERR_INVALID_ARG;
  if (need_qdk && !z->q_dot_kmean) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(z->q) || !aligned16(z->k) || !aligned16(z->v_t) || !aligned16(z->qk_correction) ||
      !aligned16(z->q_mean))
    return SAGE_ERR_INVALID_ARG;
  if (z->unpadded_k_len < 1 || z->unpadded_k_len > z->Nk) return SAGE_ERR_INVALID_ARG;
  return SAGE_OK;
}

// one opt-in flag per instantiation of the correction kernel
template <typename T, int D>
std::atomic<uint32_t>& corr_smem_flag() {
  static std::atomic<uint32_t> flag{0};
  return flag;
}

sage_status run_quantize_nvfp4(const sage_tensor* q, const sage_tensor* k, const sage_tensor* v,
                               int per_block_mean, int64_t unpadded_k_len,
                               const sage_qkv_nvfp4* out, void* ws, size_t ws_bytes,
                               cudaStream_t stream) {
  sage_status st;
  if ((st = check_tensor(q)) || (st = check_tensor(k)) || (st = check_tensor(v))) return st;
  if (q->dtype != k->dtype || q->dtype != v->dtype) return SAGE_ERR_INVALID_ARG;
  if (k->B != q->B || v->B != q->B || k->H != v->H || k->N != v->N || k->D != q->D ||
      v->D != q->D)
    return SAGE_ERR_INVALID_ARG;
  const int64_t L = unpadded_k_len <= 0 ? k->N : unpadded_k_len;
  if (L > k->N) return SAGE_ERR_INVALID_ARG;
  if ((st = check_nvfp4(out, false))) return st;
  if (out->B != q->B || out->Hq != q->H || out->Hkv != k->H || out->Nq != q->N ||
      out->Nk != k->N || out->D != q->D || out->unpadded_k_len != L ||
      (out->per_block_mean != 0) != (per_block_mean != 0))
    return SAGE_ERR_INVALID_ARG;
  const NvPlan plan = nv_plan(q->B, q->H, k->H, q->N, k->N, q->D);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SAGE_ERR_INVALID_ARG;
  if (ws_bytes < plan.total) return SAGE_ERR_WORKSPACE;

  NvQuantArgs a{};
  a.q = q->ptr; a.k = k->ptr; a.v = v->ptr;
  a.q_sb = q->sb; a.q_sh = q->sh; a.q_sn = q->sn;
  a.k_sb = k->sb; a.k_sh = k->sh; a.k_sn = k->sn;
  a.v_sb = v->sb; a.v_sh = v->sh; a.v_sn = v->sn;
  a.B = (int)q->B; a.Hq = (int)q->H; a.Hkv = (int)k->H; a.G = a.Hq / a.Hkv;
  a.Nq = (int)q->N; a.Nk = (int)k->N;
  a.Nqp = (int)pad128(q->N); a.Nkp = (int)pad128(k->N);
  a.nqt = a.Nqp / 128; a.nkt = a.Nkp / 128;
  a.L = (int)L;
  a.per_block_mean = per_block_mean ? 1 : 0;
  // K sums over the first L tokens
  const QuantPlan kp = quant_plan(q->B, k->H, L, q->D);
  a.k_splits = kp.splits; a.k_split_tokens = kp.split_tokens;
  if (a.per_block_mean) {
    a.q_splits = a.nqt; a.q_split_tokens = 128;
  } else {
    a.q_splits = plan.q.splits; a.q_split_tokens = plan.q.split_tokens;
  }
  char* w = static_cast<char*>(ws);
  const size_t kn = (size_t)a.B * a.Hkv * plan.k.splits * q->D;
  const size_t qn = (size_t)a.B * a.Hq * std::max(plan.q.splits, a.nqt) * q->D;
  a.k_hi = reinterpret_cast<double*>(w);
  a.k_lo = reinterpret_cast<double*>(w + align256(kn * 8));
  a.q_hi = reinterpret_cast<double*>(w + plan.k_bytes);
  a.q_lo = reinterpret_cast<double*>(w + plan.k_bytes + align256(qn * 8));
  const size_t qmn = (size_t)a.B * a.Hq * a.nqt * q->D;
  a.qm_bhi = reinterpret_cast<uint16_t*>(w + plan.k_bytes + plan.q_bytes);
  a.qm_blo = reinterpret_cast<uint16_t*>(w + plan.k_bytes + plan.q_bytes + align256(qmn * 2));
  a.q4 = out->q; a.q_sf = out->q_sf; a.k4 = out->k; a.k_sf = out->k_sf;
  a.v4t = out->v_t; a.v_sf_t = out->v_sf_t; a.corr = out->qk_correction;
  a.q_mean = out->q_mean; a.k_mean = out->k_mean; a.qdk = out->q_dot_kmean;

  const bool fp16 = q->dtype == SAGE_FP16;
  const int nblocks = a.B * a.Hq * a.nqt + 2 * a.B * a.Hkv * a.nkt;
  const dim3 gk(a.k_splits, a.B * a.Hkv), gq(a.q_splits, a.B * a.Hq), gc(a.nkt, a.B * a.Hkv);
  const size_t corr_smem = q->D == 128 ? NvCorrLayout<128>::BYTES : NvCorrLayout<64>::BYTES;
#define SAGE_NV_LAUNCH(T, D)                                                                     \
  do {                                                                                           \
    nv_colsum_kernel<T, D><<<gk, QUANT_THREADS, 0, stream>>>(a.k, a.k_sb, a.k_sh, a.k_sn, a.Hkv, \
                                                             a.L, a.k_splits, a.k_split_tokens,  \
                                                             a.k_hi, a.k_lo);                    \
    if (!a.per_block_mean)                                                                       \
      nv_colsum_kernel<T, D><<<gq, QUANT_THREADS, 0, stream>>>(a.q, a.q_sb, a.q_sh, a.q_sn, a.Hq, \
                                                               a.Nq, a.q_splits, a.q_split_tokens, \
                                                               a.q_hi, a.q_lo);                  \
    nv_means_kernel<D><<<a.B * a.Hkv + (a.per_block_mean ? 0 : a.B * a.Hq * ((a.nqt + NVM_QBLOCKS - 1) / NVM_QBLOCKS)), \
                         D, 0, stream>>>(a);                                                     \
    nv_quant_kernel<T, D><<<nblocks, QUANT_THREADS, 0, stream>>>(a);                             \
    if (!ensure_smem(nv_corr_kernel<T, D>, corr_smem, &corr_smem_flag<T, D>()))                  \
      return SAGE_ERR_CUDA;                                                                      \
    nv_corr_kernel<T, D><<<gc, NVC_THREADS, corr_smem, stream>>>(a);                             \
  } while (0)
  if (q->D == 128) {
    if (fp16) SAGE_NV_LAUNCH(__half, 128); else SAGE_NV_LAUNCH(__nv_bfloat16, 128);
  } else {
    if (fp16) SAGE_NV_LAUNCH(__half, 64); else SAGE_NV_LAUNCH(__nv_bfloat16, 64);
  }
#undef SAGE_NV_LAUNCH
  return launch_status();
}

// ---------------------------------------------------------------- NVFP4 attention
std::atomic<uint32_t> g_smem_nv64{0}, g_smem_nv128{0};

sage_status run_attention_nvfp4(const sage_qkv_nvfp4* z, float sm_scale, int causal,
                                int per_block_mean, int return_lse, void* out, int32_t out_dtype,
                                int64_t out_sb, int64_t out_sh, int64_t out_sn, float* lse,
                                cudaStream_t stream) {
  sage_status st;
  if ((st = check_nvfp4(z, return_lse != 0))) return st;
  if ((per_block_mean != 0) != (z->per_block_mean != 0)) return SAGE_ERR_INVALID_ARG;
  if (!out || !aligned16(out)) return SAGE_ERR_INVALID_ARG;
  if (out_dtype != SAGE_BF16 && out_dtype != SAGE_FP16) return SAGE_ERR_INVALID_ARG;
  if (out_sn < z->D || out_sn % 8 || out_sh % 8 || out_sb % 8 || out_sh < 0 || out_sb < 0)
    return SAGE_ERR_INVALID_ARG;
  if ((return_lse != 0) != (lse != nullptr)) return SAGE_ERR_INVALID_ARG;
  if (!std::isfinite(sm_scale)) return SAGE_ERR_INVALID_ARG;
  NvAttnArgs a{};
  a.q_sf = z->q_sf; a.k_sf = z->k_sf; a.v_sf_t = z->v_sf_t; a.corr = z->qk_correction;
  a.qdk = z->q_dot_kmean;
  a.out = out; a.out_sb = out_sb; a.out_sh = out_sh; a.out_sn = out_sn;
  a.out_fp16 = out_dtype == SAGE_FP16;
  a.lse = lse;
  a.B = (int)z->B; a.Hq = (int)z->Hq; a.Hkv = (int)z->Hkv; a.G = a.Hq / a.Hkv;
  a.Nq = (int)z->Nq; a.Nk = (int)z->Nk;
  a.Nqp = (int)pad128(z->Nq); a.Nkp = (int)pad128(z->Nk);
  a.nqt = a.Nqp / 128; a.nkt = a.Nkp / 128;
  a.nqp = (a.nqt + 1) / 2;
  a.L = (int)z->unpadded_k_len;
  a.causal = causal ? 1 : 0;
  a.return_lse = return_lse ? 1 : 0;
  a.causal_off = a.Nk - a.Nq;
  const float s = sm_scale > 0.f ? sm_scale : 1.0f / std::sqrt((float)z->D);
  a.sm_scale = s;
  a.c0 = (float)((double)s * 1.4426950408889634);
  const int64_t D = z->D;
  const CUtensorMapSwizzle sw = D == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_u8(&tq, z->q, D / 2, z->B * z->Hq * a.Nqp, D / 2, (uint32_t)(D / 2), 128, sw) ||
      !make_tmap_u8(&tk, z->k, D / 2, z->B * z->Hkv * a.Nkp, D / 2, (uint32_t)(D / 2), 128, sw) ||
      !make_tmap_u8(&tv, z->v_t, a.Nkp / 2, z->B * z->Hkv * D, a.Nkp / 2, 64, (uint32_t)D,
                    CU_TENSOR_MAP_SWIZZLE_64B))
    return SAGE_ERR_CUDA;
  const int grid = a.B * a.Hq * a.nqp;
  auto kernel = D == 128 ? attn_fwd_nvfp4_kernel<128> : attn_fwd_nvfp4_kernel<64>;
  // the kernel redistributes registers between its warpgroups; that is only
  // safe if the launch provides at least the sum of their shares
  {
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return SAGE_ERR_CUDA;
    if (128 * NV_REGS_LOW + 256 * NV_REGS_HIGH > NV_THREADS * fa.numRegs) return SAGE_ERR_UNSUPPORTED;
  }
  const size_t smem = D == 128 ? NvLayout<128>::bytes(a.nkt) : NvLayout<64>::bytes(a.nkt);
  const size_t smem_max = D == 128 ? NvLayout<128>::bytes(ATT_MAX_NKT) : NvLayout<64>::bytes(ATT_MAX_NKT);
  if (!ensure_smem(kernel, smem_max, D == 128 ? &g_smem_nv128 : &g_smem_nv64)) return SAGE_ERR_CUDA;
  kernel<<<grid, NV_THREADS, smem, stream>>>(tq, tk, tv, a);
  return launch_status();
}

// Carve the fused call's workspace: quantised Q/K/V, then the quantiser's
// partials, then the mask classes.
struct FusedLayout {
  size_t q8, qs, k8, ks, km, v8, vs, qdk, part, cls, total;
};
FusedLayout fused_layout(int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq, int64_t Nk, int64_t D,
                         const sage_mask* mask) {
  const int64_t Nqp = pad128(Nq), Nkp = pad128(Nk);
  FusedLayout f{};
  size_t o = 0;
  f.q8 = o; o += align256((size_t)B * Hq * Nqp * D);
  f.qs = o; o += align256((size_t)B * Hq * (Nqp / 128) * 4);
  f.k8 = o; o += align256((size_t)B * Hkv * Nkp * D);
  f.ks = o; o += align256((size_t)B * Hkv * (Nkp / 128) * 4);
  f.km = o; o += align256((size_t)B * Hkv * D * 4);
  f.v8 = o; o += align256((size_t)B * Hkv * D * Nkp);
  f.vs = o; o += align256((size_t)B * Hkv * D * 4);
  f.qdk = o; o += align256((size_t)B * Hq * Nq * 4);
  f.part = o; o += quant_plan(B, Hkv, Nk, D).part_bytes;
  f.cls = o; o += mask_class_bytes(mask, Nq, Nk);
  f.total = o;
  return f;
}

std::atomic<uint32_t> g_smem_dbg_qk{0}, g_smem_dbg_pv{0};

// ---------------------------------------------------------------- varlen
// Workspace of a variable-length call: the sequence table, then the
// quantised arrays sized for the worst padding (every sequence wastes up to
// 127 rows per head), the quantiser's reductions and q.kmean.
struct VarlenLayout {
  size_t table, q8, qs, k8, ks, km, v8, vs, qdk, part, total;
  int64_t rows_q, rows_k;   // row capacity of q8 and of k8 / v8
};

VarlenLayout varlen_layout(int64_t nseq, int64_t Hq, int64_t Hkv, int64_t total_q,
                           int64_t total_k, int64_t max_k, int64_t D, bool with_qdk) {
  VarlenLayout f{};
  f.rows_q = Hq * (total_q + 128 * nseq);
  f.rows_k = Hkv * (total_k + 128 * nseq);
  size_t o = 0;
  f.table = o; o += align256((size_t)nseq * SEQ_STRIDE * 4);
  f.q8 = o; o += align256((size_t)f.rows_q * D);
  f.qs = o; o += align256((size_t)(f.rows_q / 128) * 4);
  f.k8 = o; o += align256((size_t)f.rows_k * D);
  f.ks = o; o += align256((size_t)(f.rows_k / 128) * 4);
  f.km = o; o += align256((size_t)nseq * Hkv * D * 4);
  f.v8 = o; o += align256((size_t)f.rows_k * D);
  f.vs = o; o += align256((size_t)nseq * Hkv * D * 4);
  f.qdk = o; o += with_qdk ? align256((size_t)Hq * total_q * 4) : 0;
  f.part = o; o += quant_plan(nseq, Hkv, max_k, D).part_bytes;
  f.total = o;
  return f;
}

// A packed [total, H, D] tensor of a variable-length call (B = 1).
sage_status check_packed(const sage_tensor* t) {
  if (!t || !t->ptr) return SAGE_ERR_INVALID_ARG;
  if (t->dtype != SAGE_BF16 && t->dtype != SAGE_FP16) return SAGE_ERR_INVALID_ARG;
  if (t->B != 1 || t->H < 1 || t->H > (1 << 12) || t->N < 1 || t->N >= (int64_t(1) << 30))
    return SAGE_ERR_INVALID_ARG;
  if (!aligned16(t->ptr)) return SAGE_ERR_INVALID_ARG;
  if (t->sn < t->D || t->sn % 8 || t->sh % 8 || t->sh < 0) return SAGE_ERR_INVALID_ARG;
  if (t->D != 64 && t->D != 128) return SAGE_ERR_UNSUPPORTED;
  return SAGE_OK;
}

// ---------------------------------------------------------------- fused path
// Quantise into the workspace laid out by `f` (at `w`), then attend.
sage_status run_fused(const sage_tensor* q, const sage_tensor* k, const sage_tensor* v, int causal,
                      float sm_scale, int return_lse, int smooth_k, const sage_mask* mask,
                      void* out, int64_t out_sb, int64_t out_sh, int64_t out_sn, float* lse,
                      const FusedLayout& f, char* w, cudaStream_t stream) {
  sage_status st;
  sage_qkv_i8f8 z{};
  z.q = reinterpret_cast<int8_t*>(w + f.q8);
  z.q_scale = reinterpret_cast<float*>(w + f.qs);
  z.k = reinterpret_cast<int8_t*>(w + f.k8);
  z.k_scale = reinterpret_cast<float*>(w + f.ks);
  z.k_mean = reinterpret_cast<float*>(w + f.km);
  z.v = reinterpret_cast<uint8_t*>(w + f.v8);
  z.v_scale = reinterpret_cast<float*>(w + f.vs);
  z.q_dot_kmean = return_lse ? reinterpret_cast<float*>(w + f.qdk) : nullptr;
  z.B = q->B; z.Hq = q->H; z.Hkv = k->H; z.Nq = q->N; z.Nk = k->N; z.D = q->D;
  if ((st = run_quantize(q, k, v, smooth_k, &z, w + f.part, f.cls - f.part, stream))) return st;
  return run_attention(&z, causal, sm_scale, return_lse, mask, out, q->dtype, out_sb, out_sh,
                       out_sn, lse, w + f.cls, f.total - f.cls, stream);
}

// ---------------------------------------------------------------- host pipeline
// sage_attn_fwd_host streams a problem held in host memory through the GPU in
// chunks of (batch entry, KV head) groups.  Every group is a problem of its
// own (its K mean, its V channel scales, the 128-token blocks of its Q heads),
// so a chunk computed alone gives the bits the whole call gives.  Chunk c
// passes through three streams:
//   copy-in stream:  Q/K/V of chunk c into input slot c % kPipeSlots;
//   caller's stream: quantise + attend chunk c into output slot c % kPipeSlots;
//   copy-out stream: output slot to the host out / lse;
// so the copy in of a later chunk, the kernels of chunk c and the copy out of
// an earlier chunk overlap (the host link carries both directions at once).
constexpr int kPipeSlots = 3;
constexpr int kPipeRing = kPipeSlots + 1;            // events of one kind in flight
// automatic chunk: about this many bytes of inputs (measured on B200 with
// pinned host memory: INT8 causal GQA 16K is fastest at ~100 MB chunks,
// NVFP4 16K at ~25 MB, whose kernels per chunk are shorter)
constexpr size_t kPipeChunkI8 = size_t(100) << 20;
constexpr size_t kPipeChunkNv = size_t(25) << 20;
constexpr int kPipeMaxDevices = 64;

// Staging order of heads [h0, h0 + nh) of one batch entry: token-major
// ([N, nh, D]) when the caller's tensor keeps all heads of a token together
// in one row (head stride D, token stride at least H * D: the NHD layout),
// else head-major ([nh, N, D]).
bool token_major(int64_t H, int64_t D, int64_t sh, int64_t sn) {
  return H > 1 && sh == D && sn >= H * D;
}
struct Stage {
  int64_t sh, sn;
};
Stage stage_of(bool tm, int64_t N, int64_t nh, int64_t D) {
  return tm ? Stage{D, nh * D} : Stage{N * D, D};
}

// Heads [h0, h0 + nh) of batch entry b between the caller's strided tensor
// (host side) and its contiguous staging copy (device side).
cudaError_t copy_heads(char* dev, char* host, bool tm, int64_t sb, int64_t sh, int64_t sn,
                       int64_t b, int64_t h0, int64_t nh, int64_t N, int64_t D, size_t es,
                       bool to_dev, cudaStream_t s) {
  char* hb = host + (b * sb + h0 * sh) * (int64_t)es;
  auto copy2d = [&](char* d, char* h, size_t width, size_t dpitch, size_t hpitch, size_t rows) {
    return to_dev ? cudaMemcpy2DAsync(d, dpitch, h, hpitch, width, rows, cudaMemcpyDefault, s)
                  : cudaMemcpy2DAsync(h, hpitch, d, dpitch, width, rows, cudaMemcpyDefault, s);
  };
  if (tm)  // token-major: one 2-D copy, a row per token
    return copy2d(dev, hb, nh * D * es, nh * D * es, sn * es, N);
  if (sn == D && sh == N * D)  // the chunk's heads are one contiguous range
    return copy2d(dev, hb, nh * N * D * es, nh * N * D * es, nh * N * D * es, 1);
  for (int64_t i = 0; i < nh; ++i) {
    const cudaError_t e =
        copy2d(dev + i * N * D * (int64_t)es, hb + i * sh * (int64_t)es, D * es, D * es, sn * es, N);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// The caller's mask restricted to heads [h0, h0 + nh) of batch entry b.
sage_mask chunk_mask(const sage_mask& m, int64_t b, int64_t h0, int64_t nh) {
  sage_mask c = m;
  const int64_t el = (m.B > 1 ? b * m.sb : 0) + (m.H > 1 ? h0 * m.sh : 0);
  c.ptr = static_cast<const char*>(m.ptr) + el * (m.kind == SAGE_MASK_FLOAT ? 4 : 1);
  c.B = 1;
  c.H = m.H > 1 ? nh : 1;
  return c;
}

struct PipeLayout {
  int64_t gpc;                 // KV-head groups per chunk (at most)
  bool edge;                   // one-group first and last chunks (pipe_chunk_groups)
  size_t q, k, v, o, l, slot;  // offsets in a slot, slot bytes
  size_t fused, total;         // one chunk's quantise + attend workspace
};

// Staging slots for chunks of `chunk_groups` KV-head groups (0: automatic,
// with one-group first and last chunks) and, after them, the largest
// per-chunk quantise + attend workspace that `chunk_ws(ng)` reports for the
// chunk sizes the schedule uses.
template <typename ChunkWs>
PipeLayout pipe_layout(int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq, int64_t Nk, int64_t D,
                       int64_t chunk_groups, size_t auto_bytes, ChunkWs chunk_ws) {
  const int64_t G = Hq / Hkv;
  const size_t per_group = (size_t)(G * Nq + 2 * Nk) * D * 2;
  int64_t gpc = chunk_groups > 0
                    ? chunk_groups
                    : std::max<int64_t>(1, (int64_t)((auto_bytes + per_group / 2) / per_group));
  gpc = std::min(gpc, Hkv);
  PipeLayout p{};
  p.gpc = gpc;
  p.edge = chunk_groups == 0 && gpc > 1 && B * Hkv > 2;
  size_t o = 0;
  p.q = o; o += align256((size_t)gpc * G * Nq * D * 2);
  p.k = o; o += align256((size_t)gpc * Nk * D * 2);
  p.v = o; o += align256((size_t)gpc * Nk * D * 2);
  p.o = o; o += align256((size_t)gpc * G * Nq * D * 2);
  p.l = o; o += align256((size_t)gpc * G * Nq * 4);
  p.slot = o;
  p.fused = kPipeSlots * p.slot;
  // every chunk size of the schedule: the first, a middle and the last batch
  // entry cover every case pipe_chunk_groups distinguishes
  size_t fw = 0;
  for (const int64_t b : {int64_t(0), std::min<int64_t>(1, B - 1), B - 1})
    for (int64_t g0 = 0, ng = 0; g0 < Hkv; g0 += ng) {
      ng = pipe_chunk_groups(b, g0, B, Hkv, gpc, p.edge);
      fw = std::max(fw, chunk_ws(ng));
    }
  p.total = p.fused + fw;
  return p;
}

// The INT8/FP8 path's per-chunk workspace (sage_attn_fwd's layout for one chunk).
size_t i8_chunk_ws(int64_t G, int64_t Nq, int64_t Nk, int64_t D, const sage_mask* mask,
                   int64_t ng) {
  sage_mask cm{};
  if (mask) cm = chunk_mask(*mask, 0, 0, ng * G);
  return fused_layout(1, ng * G, ng, Nq, Nk, D, mask ? &cm : nullptr).total;
}

// The NVFP4 path's per-chunk workspace: the quantised arrays of one chunk
// (sage_qkv_nvfp4 of B = 1, nh Q heads, ng KV heads) and the quantiser's sums.
struct NvChunkLayout {
  size_t q4, qsf, k4, ksf, vt, vsft, corr, qm, km, qdk, part, total;
};
NvChunkLayout nv_chunk_layout(int64_t nh, int64_t ng, int64_t Nq, int64_t Nk, int64_t D) {
  const int64_t Nqp = pad128(Nq), Nkp = pad128(Nk), nqt = Nqp / 128;
  NvChunkLayout f{};
  size_t o = 0;
  f.q4 = o; o += align256((size_t)nh * Nqp * D / 2);
  f.qsf = o; o += align256((size_t)nh * Nqp * D / 16);
  f.k4 = o; o += align256((size_t)ng * Nkp * D / 2);
  f.ksf = o; o += align256((size_t)ng * Nkp * D / 16);
  f.vt = o; o += align256((size_t)ng * D * Nkp / 2);
  f.vsft = o; o += align256((size_t)ng * D * Nkp / 16);
  f.corr = o; o += align256((size_t)nh * nqt * Nkp * 4);
  f.qm = o; o += align256((size_t)nh * nqt * D * 4);
  f.km = o; o += align256((size_t)ng * D * 4);
  f.qdk = o; o += align256((size_t)nh * Nq * 4);
  f.part = o; o += nv_plan(1, nh, ng, Nq, Nk, D).total;
  f.total = o;
  return f;
}

// Copy streams and events, created once per device on first use.
struct PipeStreams {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, join_in = nullptr, join_out = nullptr;
  cudaEvent_t copied[kPipeRing], computed[kPipeRing], drained[kPipeRing];
};
std::mutex g_pipe_mu;  // held while a call enqueues (the events are shared)
PipeStreams g_pipe[kPipeMaxDevices];

sage_status pipe_streams(PipeStreams** res) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kPipeMaxDevices)
    return SAGE_ERR_CUDA;
  PipeStreams& p = g_pipe[dev];
  if (!p.in) {
    PipeStreams n;
    bool ok = cudaStreamCreateWithFlags(&n.in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&n.out, cudaStreamNonBlocking) == cudaSuccess;
    cudaEvent_t* evs[] = {&n.start, &n.join_in, &n.join_out};
    for (cudaEvent_t* e : evs)
      ok = ok && cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; i < kPipeRing; ++i)
      ok = ok && cudaEventCreateWithFlags(&n.copied[i], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&n.computed[i], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&n.drained[i], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) return SAGE_ERR_CUDA;  // a failed creation leaks what it made; it does not recur
    p = n;
  }
  *res = &p;
  return SAGE_OK;
}

// `compute(b, h0, g0, cq, ck, cv, out_slot, out_sh, out_sn, lse_slot)`
// enqueues the quantise + attend of one chunk (heads h0.. of batch entry b,
// KV heads g0..) on `stream`, reading the staged cq/ck/cv and writing the
// staged output (strides in elements) and LSE, with its workspace at
// w + p.fused.
template <typename Compute>
sage_status run_host_pipeline(const sage_tensor* q, const sage_tensor* k, const sage_tensor* v,
                              int return_lse, void* out, int64_t out_sb, int64_t out_sh,
                              int64_t out_sn, float* lse, const PipeLayout& p, char* w,
                              cudaStream_t stream, Compute compute) {
  std::lock_guard<std::mutex> lock(g_pipe_mu);
  PipeStreams* ps = nullptr;
  sage_status st = pipe_streams(&ps);
  if (st) return st;
  const int64_t B = q->B, Hq = q->H, Hkv = k->H, Nq = q->N, Nk = k->N, D = q->D;
  const int64_t G = Hq / Hkv;
  const size_t es = 2;
  char* hq = static_cast<char*>(const_cast<void*>(q->ptr));
  char* hk = static_cast<char*>(const_cast<void*>(k->ptr));
  char* hv = static_cast<char*>(const_cast<void*>(v->ptr));
  char* ho = static_cast<char*>(out);
  const bool tq = token_major(Hq, D, q->sh, q->sn), tk = token_major(Hkv, D, k->sh, k->sn),
             tv = token_major(Hkv, D, v->sh, v->sn), to = token_major(Hq, D, out_sh, out_sn);
  bool ok = cudaEventRecord(ps->start, stream) == cudaSuccess &&
            cudaStreamWaitEvent(ps->in, ps->start, 0) == cudaSuccess &&
            cudaStreamWaitEvent(ps->out, ps->start, 0) == cudaSuccess;
  int64_t c = 0;
  for (int64_t b = 0; ok && b < B; ++b) {
    for (int64_t g0 = 0, ng = 0; ok && g0 < Hkv; g0 += ng, ++c) {
      ng = pipe_chunk_groups(b, g0, B, Hkv, p.gpc, p.edge);
      const int64_t nh = ng * G, h0 = g0 * G;
      const int r = (int)(c % kPipeRing);
      char* sl = w + (c % kPipeSlots) * p.slot;
      // copy in, once the chunk that last used this slot has been computed
      if (c >= kPipeSlots)
        ok = cudaStreamWaitEvent(ps->in, ps->computed[(c - kPipeSlots) % kPipeRing], 0) ==
             cudaSuccess;
      ok = ok && copy_heads(sl + p.q, hq, tq, q->sb, q->sh, q->sn, b, h0, nh, Nq, D, es, true,
                            ps->in) == cudaSuccess;
      ok = ok && copy_heads(sl + p.k, hk, tk, k->sb, k->sh, k->sn, b, g0, ng, Nk, D, es, true,
                            ps->in) == cudaSuccess;
      ok = ok && copy_heads(sl + p.v, hv, tv, v->sb, v->sh, v->sn, b, g0, ng, Nk, D, es, true,
                            ps->in) == cudaSuccess;
      ok = ok && cudaEventRecord(ps->copied[r], ps->in) == cudaSuccess;
      // quantise + attend, once the output slot has been drained
      ok = ok && cudaStreamWaitEvent(stream, ps->copied[r], 0) == cudaSuccess;
      if (ok && c >= kPipeSlots)
        ok = cudaStreamWaitEvent(stream, ps->drained[(c - kPipeSlots) % kPipeRing], 0) ==
             cudaSuccess;
      if (!ok) break;
      const Stage sq = stage_of(tq, Nq, nh, D), sk = stage_of(tk, Nk, ng, D),
                  sv = stage_of(tv, Nk, ng, D), so = stage_of(to, Nq, nh, D);
      const sage_tensor cq{sl + p.q, q->dtype, 1, nh, Nq, D, nh * Nq * D, sq.sh, sq.sn};
      const sage_tensor ck{sl + p.k, k->dtype, 1, ng, Nk, D, ng * Nk * D, sk.sh, sk.sn};
      const sage_tensor cv{sl + p.v, v->dtype, 1, ng, Nk, D, ng * Nk * D, sv.sh, sv.sn};
      st = compute(b, h0, g0, cq, ck, cv, sl + p.o, so.sh, so.sn,
                   return_lse ? reinterpret_cast<float*>(sl + p.l) : nullptr);
      if (st) break;
      ok = cudaEventRecord(ps->computed[r], stream) == cudaSuccess;
      // copy out
      ok = ok && cudaStreamWaitEvent(ps->out, ps->computed[r], 0) == cudaSuccess;
      ok = ok && copy_heads(sl + p.o, ho, to, out_sb, out_sh, out_sn, b, h0, nh, Nq, D, es, false,
                            ps->out) == cudaSuccess;
      if (ok && return_lse)
        ok = cudaMemcpyAsync(lse + (b * Hq + h0) * Nq, sl + p.l, (size_t)nh * Nq * 4,
                             cudaMemcpyDefault, ps->out) == cudaSuccess;
      ok = ok && cudaEventRecord(ps->drained[r], ps->out) == cudaSuccess;
    }
  }
  // the caller's stream continues only after everything enqueued on the copy
  // streams, whatever happened above
  const bool joined = cudaEventRecord(ps->join_in, ps->in) == cudaSuccess &&
                      cudaEventRecord(ps->join_out, ps->out) == cudaSuccess &&
                      cudaStreamWaitEvent(stream, ps->join_in, 0) == cudaSuccess &&
                      cudaStreamWaitEvent(stream, ps->join_out, 0) == cudaSuccess;
  if (st) return st;
  return ok && joined ? SAGE_OK : SAGE_ERR_CUDA;
}

// A whole-path call without queries (q->B == 0 or q->N == 0) has no output to
// compute.  Returns true for such a call, with *st set to SAGE_OK when its
// sizes are consistent (q, k, v of one dtype, matching batch, head counts
// with Hq % Hkv == 0, k and v of one length, D 64 or 128) and to the error
// otherwise.  Pointers are not looked at: an empty tensor has no storage.
// Nothing is launched or enqueued for it.
bool empty_call(const sage_tensor* q, const sage_tensor* k, const sage_tensor* v,
                sage_status* st) {
  if (!q || !k || !v || (q->B != 0 && q->N != 0)) return false;
  *st = SAGE_ERR_INVALID_ARG;
  for (const sage_tensor* t : {q, k, v}) {
    if (t->dtype != SAGE_BF16 && t->dtype != SAGE_FP16) return true;
    if (t->B < 0 || t->B > (1 << 16) || t->H < 1 || t->H > (1 << 12) || t->N < 0 || t->D < 1)
      return true;
  }
  if (k->dtype != q->dtype || v->dtype != q->dtype || k->B != q->B || v->B != q->B ||
      v->H != k->H || v->N != k->N || k->D != q->D || v->D != q->D || q->H % k->H)
    return true;
  *st = q->D == 64 || q->D == 128 ? SAGE_OK : SAGE_ERR_UNSUPPORTED;
  return true;
}

// Arguments of the host-resident calls' outputs: out (host, q's logical
// shape, element strides, 16-byte aligned rows), lse (host, when asked for),
// a non-negative chunk size.
sage_status check_host_out(const sage_tensor* q, const void* out, int64_t out_sb, int64_t out_sh,
                           int64_t out_sn, int return_lse, const float* lse, int64_t chunk_groups) {
  if (!out || chunk_groups < 0 || (return_lse && !lse)) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(out) || out_sn < q->D || out_sn % 8 || out_sh % 8 || out_sb % 8 || out_sh < 0 ||
      out_sb < 0)
    return SAGE_ERR_INVALID_ARG;
  return SAGE_OK;
}

}  // namespace

// =================================================================== C ABI
extern "C" {

const char* sage_status_str(sage_status s) {
  switch (s) {
    case SAGE_OK: return "ok";
    case SAGE_ERR_INVALID_ARG: return "invalid argument";
    case SAGE_ERR_UNSUPPORTED: return "unsupported configuration";
    case SAGE_ERR_WORKSPACE: return "workspace too small";
    case SAGE_ERR_CUDA: return "CUDA error";
    case SAGE_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

const char* sage_version(void) { return "sage_b200 0.1 (sm_100a)"; }

sage_status sage_get_device_status(sage_stream_t stream, uint32_t* site) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return SAGE_ERR_CUDA;
  uint32_t v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return SAGE_ERR_CUDA;
  if (v && cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return SAGE_ERR_CUDA;
  if (site) *site = v;
  return v ? SAGE_ERR_TIMEOUT : SAGE_OK;
}

size_t sage_quantize_workspace_bytes(int64_t B, int64_t Hkv, int64_t Nk, int64_t D) {
  if (!valid_dims(B, Hkv, Nk, D)) return 0;
  return quant_plan(B, Hkv, Nk, D).part_bytes;
}

sage_status sage_quantize_qkv(const sage_tensor* q, const sage_tensor* k, const sage_tensor* v,
                              int smooth_k, const sage_qkv_i8f8* out, void* ws, size_t ws_bytes,
                              sage_stream_t stream) {
  return run_quantize(q, k, v, smooth_k, out, ws, ws_bytes, stream);
}

size_t sage_attn_quantized_workspace_bytes(const sage_qkv_i8f8* z, const sage_mask* mask) {
  if (!z) return 0;
  return mask_class_bytes(mask, z->Nq, z->Nk);
}

sage_status sage_attn_fwd_quantized(const sage_qkv_i8f8* qkv, int causal, float sm_scale,
                                    int return_lse, const sage_mask* mask, void* out,
                                    int32_t out_dtype, int64_t out_sb, int64_t out_sh,
                                    int64_t out_sn, float* lse, void* ws, size_t ws_bytes,
                                    sage_stream_t stream) {
  return run_attention(qkv, causal, sm_scale, return_lse, mask, out, out_dtype, out_sb, out_sh,
                       out_sn, lse, ws, ws_bytes, stream);
}

size_t sage_attn_fwd_workspace_bytes(int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq, int64_t Nk,
                                     int64_t D, const sage_mask* mask) {
  if (!valid_dims(B, Hq, Nq, D) || !valid_dims(B, Hkv, Nk, D)) return 0;
  return fused_layout(B, Hq, Hkv, Nq, Nk, D, mask).total;
}

sage_status sage_attn_fwd(const sage_tensor* q, const sage_tensor* k, const sage_tensor* v,
                          int causal, float sm_scale, int num_kv_heads, int return_lse,
                          int smooth_k, const sage_mask* mask, void* out, int64_t out_sb,
                          int64_t out_sh, int64_t out_sn, float* lse, void* ws, size_t ws_bytes,
                          sage_stream_t stream) {
  sage_status st;
  if (empty_call(q, k, v, &st)) return st ? st : num_kv_heads == k->H ? SAGE_OK : SAGE_ERR_INVALID_ARG;
  if ((st = check_tensor(q)) || (st = check_tensor(k)) || (st = check_tensor(v))) return st;
  if (num_kv_heads != k->H) return SAGE_ERR_INVALID_ARG;
  if ((st = check_qkv_shapes(q->B, q->H, k->H, q->N, k->N, q->D))) return st;
  if (q->B * q->H > kMaxGridYZ) return SAGE_ERR_UNSUPPORTED;
  if ((st = check_mask(mask, q->B, q->H, q->N, k->N))) return st;
  const FusedLayout f = fused_layout(q->B, q->H, k->H, q->N, k->N, q->D, mask);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SAGE_ERR_INVALID_ARG;
  if (ws_bytes < f.total) return SAGE_ERR_WORKSPACE;
  return run_fused(q, k, v, causal, sm_scale, return_lse, smooth_k, mask, out, out_sb, out_sh,
                   out_sn, lse, f, static_cast<char*>(ws), stream);
}

size_t sage_attn_fwd_host_workspace_bytes(int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq,
                                          int64_t Nk, int64_t D, const sage_mask* mask,
                                          int64_t chunk_groups) {
  if (!valid_dims(B, Hq, Nq, D) || !valid_dims(B, Hkv, Nk, D) || Hq % Hkv || chunk_groups < 0)
    return 0;
  const int64_t G = Hq / Hkv;
  return pipe_layout(B, Hq, Hkv, Nq, Nk, D, chunk_groups, kPipeChunkI8,
                     [&](int64_t ng) { return i8_chunk_ws(G, Nq, Nk, D, mask, ng); })
      .total;
}

sage_status sage_attn_fwd_host(const sage_tensor* q, const sage_tensor* k, const sage_tensor* v,
                               int causal, float sm_scale, int num_kv_heads, int return_lse,
                               int smooth_k, const sage_mask* mask, void* out, int64_t out_sb,
                               int64_t out_sh, int64_t out_sn, float* lse, int64_t chunk_groups,
                               void* ws, size_t ws_bytes, sage_stream_t stream) {
  sage_status st;
  if (empty_call(q, k, v, &st)) return st ? st : num_kv_heads == k->H ? SAGE_OK : SAGE_ERR_INVALID_ARG;
  if ((st = check_tensor(q)) || (st = check_tensor(k)) || (st = check_tensor(v))) return st;
  if (num_kv_heads != k->H || k->dtype != q->dtype || v->dtype != q->dtype)
    return SAGE_ERR_INVALID_ARG;
  if (k->B != q->B || v->B != q->B || v->H != k->H || v->N != k->N || k->D != q->D ||
      v->D != q->D)
    return SAGE_ERR_INVALID_ARG;
  if ((st = check_qkv_shapes(q->B, q->H, k->H, q->N, k->N, q->D))) return st;
  if ((st = check_mask(mask, q->B, q->H, q->N, k->N))) return st;
  if ((st = check_host_out(q, out, out_sb, out_sh, out_sn, return_lse, lse, chunk_groups))) return st;
  const int64_t Nq = q->N, Nk = k->N, D = q->D, G = q->H / k->H;
  const PipeLayout p = pipe_layout(q->B, q->H, k->H, Nq, Nk, D, chunk_groups, kPipeChunkI8,
                                   [&](int64_t ng) { return i8_chunk_ws(G, Nq, Nk, D, mask, ng); });
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SAGE_ERR_INVALID_ARG;
  if (ws_bytes < p.total) return SAGE_ERR_WORKSPACE;
  char* fw = static_cast<char*>(ws) + p.fused;
  return run_host_pipeline(
      q, k, v, return_lse, out, out_sb, out_sh, out_sn, lse, p, static_cast<char*>(ws), stream,
      [&](int64_t b, int64_t h0, int64_t, const sage_tensor& cq, const sage_tensor& ck,
          const sage_tensor& cv, char* o, int64_t o_sh, int64_t o_sn, float* l) {
        sage_mask cm{};
        if (mask) cm = chunk_mask(*mask, b, h0, cq.H);
        const FusedLayout f = fused_layout(1, cq.H, ck.H, Nq, Nk, D, mask ? &cm : nullptr);
        return run_fused(&cq, &ck, &cv, causal, sm_scale, return_lse, smooth_k,
                         mask ? &cm : nullptr, o, cq.H * Nq * D, o_sh, o_sn, l, f, fw, stream);
      });
}

size_t sage_attn_fwd_nvfp4_host_workspace_bytes(int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq,
                                                int64_t Nk, int64_t D, int64_t chunk_groups) {
  if (!valid_dims(B, Hq, Nq, D) || !valid_dims(B, Hkv, Nk, D) || Hq % Hkv || chunk_groups < 0)
    return 0;
  const int64_t G = Hq / Hkv;
  return pipe_layout(B, Hq, Hkv, Nq, Nk, D, chunk_groups, kPipeChunkNv,
                     [&](int64_t ng) { return nv_chunk_layout(ng * G, ng, Nq, Nk, D).total; })
      .total;
}

sage_status sage_attn_fwd_nvfp4_host(const sage_tensor* q, const sage_tensor* k,
                                     const sage_tensor* v, float sm_scale, int causal,
                                     int per_block_mean, int64_t unpadded_k_len, int return_lse,
                                     void* out, int64_t out_sb, int64_t out_sh, int64_t out_sn,
                                     float* lse, int64_t chunk_groups, void* ws, size_t ws_bytes,
                                     sage_stream_t stream) {
  sage_status st;
  if (empty_call(q, k, v, &st)) return st ? st : unpadded_k_len <= k->N ? SAGE_OK : SAGE_ERR_INVALID_ARG;
  if ((st = check_tensor(q)) || (st = check_tensor(k)) || (st = check_tensor(v))) return st;
  if (k->dtype != q->dtype || v->dtype != q->dtype) return SAGE_ERR_INVALID_ARG;
  if (k->B != q->B || v->B != q->B || v->H != k->H || v->N != k->N || k->D != q->D ||
      v->D != q->D)
    return SAGE_ERR_INVALID_ARG;
  if ((st = check_qkv_shapes(q->B, q->H, k->H, q->N, k->N, q->D))) return st;
  const int64_t L = unpadded_k_len <= 0 ? k->N : unpadded_k_len;
  if (L > k->N) return SAGE_ERR_INVALID_ARG;
  if ((st = check_host_out(q, out, out_sb, out_sh, out_sn, return_lse, lse, chunk_groups))) return st;
  const int64_t Nq = q->N, Nk = k->N, D = q->D, G = q->H / k->H;
  const PipeLayout p = pipe_layout(q->B, q->H, k->H, Nq, Nk, D, chunk_groups, kPipeChunkNv,
                                   [&](int64_t ng) { return nv_chunk_layout(ng * G, ng, Nq, Nk, D).total; });
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SAGE_ERR_INVALID_ARG;
  if (ws_bytes < p.total) return SAGE_ERR_WORKSPACE;
  char* fw = static_cast<char*>(ws) + p.fused;
  return run_host_pipeline(
      q, k, v, return_lse, out, out_sb, out_sh, out_sn, lse, p, static_cast<char*>(ws), stream,
      [&](int64_t, int64_t, int64_t, const sage_tensor& cq, const sage_tensor& ck,
          const sage_tensor& cv, char* o, int64_t o_sh, int64_t o_sn, float* l) {
        const NvChunkLayout f = nv_chunk_layout(cq.H, ck.H, Nq, Nk, D);
        sage_qkv_nvfp4 z{};
        z.q = reinterpret_cast<uint8_t*>(fw + f.q4);
        z.q_sf = reinterpret_cast<uint8_t*>(fw + f.qsf);
        z.k = reinterpret_cast<uint8_t*>(fw + f.k4);
        z.k_sf = reinterpret_cast<uint8_t*>(fw + f.ksf);
        z.v_t = reinterpret_cast<uint8_t*>(fw + f.vt);
        z.v_sf_t = reinterpret_cast<uint8_t*>(fw + f.vsft);
        z.qk_correction = reinterpret_cast<float*>(fw + f.corr);
        z.q_mean = reinterpret_cast<float*>(fw + f.qm);
        z.k_mean = reinterpret_cast<float*>(fw + f.km);
        z.q_dot_kmean = return_lse ? reinterpret_cast<float*>(fw + f.qdk) : nullptr;
        z.B = 1; z.Hq = cq.H; z.Hkv = ck.H; z.Nq = Nq; z.Nk = Nk; z.D = D;
        z.unpadded_k_len = L;
        z.per_block_mean = per_block_mean ? 1 : 0;
        sage_status s2 = run_quantize_nvfp4(&cq, &ck, &cv, per_block_mean, L, &z, fw + f.part,
                                            f.total - f.part, stream);
        if (s2) return s2;
        return run_attention_nvfp4(&z, sm_scale, causal, per_block_mean, return_lse, o, q->dtype,
                                   cq.H * Nq * D, o_sh, o_sn, l, stream);
      });
}

size_t sage_quantize_nvfp4_workspace_bytes(int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq,
                                           int64_t Nk, int64_t D) {
  if (!valid_dims(B, Hq, Nq, D) || !valid_dims(B, Hkv, Nk, D)) return 0;
  return nv_plan(B, Hq, Hkv, Nq, Nk, D).total;
}

sage_status sage_quantize_qkv_nvfp4(const sage_tensor* q, const sage_tensor* k,
                                    const sage_tensor* v, int per_block_mean,
                                    int64_t unpadded_k_len, const sage_qkv_nvfp4* out, void* ws,
                                    size_t ws_bytes, sage_stream_t stream) {
  return run_quantize_nvfp4(q, k, v, per_block_mean, unpadded_k_len, out, ws, ws_bytes, stream);
}

sage_status sage_attn_fwd_nvfp4(const sage_qkv_nvfp4* qkv, float sm_scale, int causal,
                                int per_block_mean, int return_lse, void* out, int32_t out_dtype,
                                int64_t out_sb, int64_t out_sh, int64_t out_sn, float* lse,
                                sage_stream_t stream) {
  return run_attention_nvfp4(qkv, sm_scale, causal, per_block_mean, return_lse, out, out_dtype,
                             out_sb, out_sh, out_sn, lse, stream);
}

sage_status sage_debug_qk_int32(const sage_qkv_i8f8* z, int64_t b, int64_t h, int64_t qblk,
                                int64_t kblk, int32_t* tile, sage_stream_t stream) {
  sage_status st;
  if ((st = check_qkv(z, false))) return st;
  if (!tile || b < 0 || b >= z->B || h < 0 || h >= z->Hq || qblk < 0 ||
      qblk >= pad128(z->Nq) / 128 || kblk < 0 || kblk >= pad128(z->Nk) / 128)
    return SAGE_ERR_INVALID_ARG;
  CUtensorMap tq, tk, tv;
  if (!make_qkv_tmaps(z, &tq, &tk, &tv)) return SAGE_ERR_CUDA;
  const int64_t g = h / (z->Hq / z->Hkv);
  const int qrow = (int)((b * z->Hq + h) * pad128(z->Nq) + qblk * 128);
  const int krow = (int)((b * z->Hkv + g) * pad128(z->Nk) + kblk * 128);
  if (z->D == 128) {
    const size_t smem = 1024 + AttnLayout<128>::Q_BYTES + AttnLayout<128>::K_BYTES + 64;
    if (!ensure_smem(debug_qk_kernel<128>, smem, &g_smem_dbg_qk)) return SAGE_ERR_CUDA;
    debug_qk_kernel<128><<<1, 128, smem, stream>>>(tq, tk, qrow, krow, tile);
  } else {
    const size_t smem = 1024 + AttnLayout<64>::Q_BYTES + AttnLayout<64>::K_BYTES + 64;
    debug_qk_kernel<64><<<1, 128, smem, stream>>>(tq, tk, qrow, krow, tile);
  }
  return launch_status();
}

sage_status sage_debug_pv_fp32(const sage_qkv_i8f8* z, const uint8_t* p, int64_t b, int64_t h_kv,
                               int64_t kblk, float* acc, sage_stream_t stream) {
  sage_status st;
  if ((st = check_qkv(z, false))) return st;
  if (!p || !acc || !aligned16(p) || b < 0 || b >= z->B || h_kv < 0 || h_kv >= z->Hkv ||
      kblk < 0 || kblk >= pad128(z->Nk) / 128)
    return SAGE_ERR_INVALID_ARG;
  CUtensorMap tq, tk, tv;
  if (!make_qkv_tmaps(z, &tq, &tk, &tv)) return SAGE_ERR_CUDA;
  const int vrow = (int)((b * z->Hkv + h_kv) * pad128(z->Nk) + kblk * 128);
  const int vcol = 0;
  if (z->D == 128) {
    const size_t smem = 1024 + AttnLayout<128>::P_BYTES + AttnLayout<128>::V_BYTES + 64;
    if (!ensure_smem(debug_pv_kernel<128>, smem, &g_smem_dbg_pv)) return SAGE_ERR_CUDA;
    debug_pv_kernel<128><<<1, 128, smem, stream>>>(tv, vrow, vcol, p, acc);
  } else {
    const size_t smem = 1024 + AttnLayout<64>::P_BYTES + AttnLayout<64>::V_BYTES + 64;
    debug_pv_kernel<64><<<1, 128, smem, stream>>>(tv, vrow, vcol, p, acc);
  }
  return launch_status();
}

sage_status sage_debug_wait_timeout(uint32_t timeout_us, sage_stream_t stream) {
  if (timeout_us == 0 || timeout_us > 10000000u) return SAGE_ERR_INVALID_ARG;
  debug_wait_kernel<<<1, 32, 0, stream>>>((uint64_t)timeout_us * 1000ull);
  return launch_status();
}

// ------------------------------------------------- variable length
size_t sage_attn_fwd_varlen_workspace_bytes(int64_t nseq, int64_t Hq, int64_t Hkv,
                                            int64_t total_q, int64_t total_k,
                                            int64_t max_seqlen_q, int64_t max_seqlen_k,
                                            int64_t D, int return_lse) {
  (void)max_seqlen_q;
  if (nseq < 1 || Hq < 1 || Hkv < 1 || total_q < 1 || total_k < 1 || max_seqlen_k < 1 ||
      (D != 64 && D != 128))
    return 0;
  return varlen_layout(nseq, Hq, Hkv, total_q, total_k, max_seqlen_k, D, return_lse != 0).total;
}

sage_status sage_attn_fwd_varlen(const sage_tensor* q, const sage_tensor* k, const sage_tensor* v,
                                 const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                 int64_t nseq, int64_t max_seqlen_q, int64_t max_seqlen_k,
                                 int causal, float sm_scale, int smooth_k, int return_lse,
                                 void* out, int64_t out_sn, int64_t out_sh, float* lse, void* ws,
                                 size_t ws_bytes, sage_stream_t stream) {
  sage_status st;
  if ((st = check_packed(q)) || (st = check_packed(k)) || (st = check_packed(v))) return st;
  if (q->dtype != k->dtype || q->dtype != v->dtype) return SAGE_ERR_INVALID_ARG;
  if (k->H != v->H || k->N != v->N || k->D != q->D || v->D != q->D || q->H % k->H)
    return SAGE_ERR_INVALID_ARG;
  if (nseq < 1 || nseq > (1 << 20) || !cu_seqlens_q || !cu_seqlens_k ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u))
    return SAGE_ERR_INVALID_ARG;
  if (max_seqlen_q < 1 || max_seqlen_k < 1) return SAGE_ERR_INVALID_ARG;
  if (max_seqlen_q > 128 * ATT_MAX_NKT || max_seqlen_k > 128 * ATT_MAX_NKT)
    return SAGE_ERR_UNSUPPORTED;
  if (nseq * k->H > kMaxGridYZ) return SAGE_ERR_UNSUPPORTED;
  if (!out || !aligned16(out) || out_sn < q->D || out_sn % 8 || out_sh % 8 || out_sh < 0)
    return SAGE_ERR_INVALID_ARG;
  if ((return_lse != 0) != (lse != nullptr)) return SAGE_ERR_INVALID_ARG;
  if (!std::isfinite(sm_scale)) return SAGE_ERR_INVALID_ARG;
  const int64_t D = q->D, Hq = q->H, Hkv = k->H, total_q = q->N, total_k = k->N;
  const VarlenLayout f = varlen_layout(nseq, Hq, Hkv, total_q, total_k, max_seqlen_k, D,
                                       return_lse != 0);
  // TMA row coordinates and the LSE index are int32
  if (f.rows_q >= (int64_t(1) << 31) || f.rows_k >= (int64_t(1) << 31) ||
      Hq * total_q >= (int64_t(1) << 31))
    return SAGE_ERR_UNSUPPORTED;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SAGE_ERR_INVALID_ARG;
  if (ws_bytes < f.total) return SAGE_ERR_WORKSPACE;
  char* w = static_cast<char*>(ws);
  int* table = reinterpret_cast<int*>(w + f.table);
  seq_table_kernel<<<1, 32, 0, stream>>>(cu_seqlens_q, cu_seqlens_k, (int)nseq, (int)total_q,
                                         (int)total_k, (int)max_seqlen_q, (int)max_seqlen_k,
                                         table);
  if ((st = launch_status())) return st;

  // quantise: every sequence its own K mean, blocks and V scales
  const QuantPlan plan = quant_plan(nseq, Hkv, max_seqlen_k, D);
  QuantArgs a{};
  a.q = q->ptr; a.k = k->ptr; a.v = v->ptr;
  a.q_sh = q->sh; a.q_sn = q->sn;
  a.k_sh = k->sh; a.k_sn = k->sn;
  a.v_sh = v->sh; a.v_sn = v->sn;
  a.B = (int)nseq; a.Hq = (int)Hq; a.Hkv = (int)Hkv; a.G = a.Hq / a.Hkv;
  a.Nq = (int)max_seqlen_q; a.Nk = (int)max_seqlen_k;
  a.Nqp = (int)pad128(max_seqlen_q); a.Nkp = (int)pad128(max_seqlen_k);
  a.nqt = a.Nqp / 128; a.nkt = a.Nkp / 128;
  a.smooth_k = smooth_k ? 1 : 0;
  a.splits = plan.splits;
  a.split_tokens = plan.split_tokens;
  const size_t n = (size_t)nseq * Hkv * plan.splits * D;
  char* wp = w + f.part;
  a.part_hi = reinterpret_cast<double*>(wp);
  a.part_lo = reinterpret_cast<double*>(wp + align256(n * 8));
  a.part_amax = reinterpret_cast<float*>(wp + 2 * align256(n * 8));
  a.va = reinterpret_cast<float*>(wp + 2 * align256(n * 8) + align256(n * 4));
  a.q8 = reinterpret_cast<int8_t*>(w + f.q8);
  a.q_scale = reinterpret_cast<float*>(w + f.qs);
  a.k8 = reinterpret_cast<int8_t*>(w + f.k8);
  a.k_scale = reinterpret_cast<float*>(w + f.ks);
  a.k_mean = reinterpret_cast<float*>(w + f.km);
  a.v8 = reinterpret_cast<uint8_t*>(w + f.v8);
  a.v_scale = reinterpret_cast<float*>(w + f.vs);
  a.qdk = return_lse ? reinterpret_cast<float*>(w + f.qdk) : nullptr;
  a.kv_limit = a.Nk;
  a.seqs = table;
  a.max_nqt = a.nqt;
  a.max_nkt = a.nkt;
  if ((st = launch_quantize(a, plan, D, q->dtype == SAGE_FP16, stream))) return st;

  // attention over the quantised sequences
  CUtensorMap tq, tk, tv;
  if (!make_tmap_u8(&tq, a.q8, D, f.rows_q, D, (uint32_t)D, 128, qk_swizzle(D)) ||
      !make_tmap_u8(&tk, a.k8, D, f.rows_k, D, (uint32_t)D, 128, qk_swizzle(D)) ||
      !make_tmap_u8(&tv, a.v8, D, f.rows_k, D, (uint32_t)D, 128, qk_swizzle(D)))
    return SAGE_ERR_CUDA;
  AttnArgs b{};
  b.q_scale = a.q_scale; b.k_scale = a.k_scale; b.v_scale = a.v_scale; b.qdk = a.qdk;
  b.out = out; b.out_sh = out_sh; b.out_sn = out_sn;
  b.out_fp16 = q->dtype == SAGE_FP16;
  b.lse = lse;
  b.B = (int)nseq; b.Hq = (int)Hq; b.Hkv = (int)Hkv; b.G = b.Hq / b.Hkv;
  b.Nq = a.Nq; b.Nk = a.Nk; b.Nqp = a.Nqp; b.Nkp = a.Nkp;
  b.nqt = a.nqt; b.nkt = a.nkt; b.nqp = (b.nqt + 1) / 2;
  b.causal = causal ? 1 : 0;
  b.return_lse = return_lse ? 1 : 0;
  const float s = sm_scale > 0.f ? sm_scale : 1.0f / std::sqrt((float)D);
  b.sm_scale = s;
  b.c0 = (float)((double)s * 1.4426950408889634);
  b.seqs = table;
  b.max_nqp = b.nqp;
  const int64_t grid = (int64_t)b.max_nqp * nseq * Hq;
  if (log_enabled())
    std::fprintf(stderr, "[sage] attn varlen nseq=%lld Hq=%d Hkv=%d max_q=%d max_k=%d causal=%d grid=%lld\n",
                 (long long)nseq, b.Hq, b.Hkv, b.Nq, b.Nk, b.causal, (long long)grid);
  return launch_attention(b, D, tq, tk, tv, grid, stream);
}

// ------------------------------------------------- merge over key shards
sage_status sage_lse_merge(float* acc, float* acc_lse, const void* part, int32_t part_dtype,
                           int64_t sb, int64_t sh, int64_t sn, const float* part_lse, int64_t B,
                           int64_t H, int64_t N, int64_t D, int init, sage_stream_t stream) {
  if (D != 64 && D != 128) return SAGE_ERR_UNSUPPORTED;
  if (!valid_dims(B, H, N, D)) return SAGE_ERR_INVALID_ARG;
  if (!acc || !acc_lse || !part || !part_lse || !aligned16(acc) || !aligned16(part))
    return SAGE_ERR_INVALID_ARG;
  if (part_dtype != SAGE_BF16 && part_dtype != SAGE_FP16) return SAGE_ERR_INVALID_ARG;
  if (sn < D || sn % 8 || sh % 8 || sb % 8 || sh < 0 || sb < 0) return SAGE_ERR_INVALID_ARG;
  MergeArgs a{};
  a.acc = acc; a.acc_lse = acc_lse; a.part = part; a.sb = sb; a.sh = sh; a.sn = sn;
  a.part_lse = part_lse; a.B = (int)B; a.H = (int)H; a.N = (int)N; a.init = init ? 1 : 0;
  const int64_t rows = B * H * N;
  const int64_t blocks = (rows + (256 / (D / 8)) - 1) / (256 / (D / 8));
  if (blocks >= (int64_t(1) << 31)) return SAGE_ERR_UNSUPPORTED;
  const bool fp16 = part_dtype == SAGE_FP16;
  if (D == 128) {
    if (fp16) lse_merge_kernel<__half, 128><<<(unsigned)blocks, 256, 0, stream>>>(a);
    else lse_merge_kernel<__nv_bfloat16, 128><<<(unsigned)blocks, 256, 0, stream>>>(a);
  } else {
    if (fp16) lse_merge_kernel<__half, 64><<<(unsigned)blocks, 256, 0, stream>>>(a);
    else lse_merge_kernel<__nv_bfloat16, 64><<<(unsigned)blocks, 256, 0, stream>>>(a);
  }
  return launch_status();
}

sage_status sage_lse_merge_finalize(const float* acc, void* out, int32_t out_dtype, int64_t sb,
                                    int64_t sh, int64_t sn, int64_t B, int64_t H, int64_t N,
                                    int64_t D, sage_stream_t stream) {
  if (D != 64 && D != 128) return SAGE_ERR_UNSUPPORTED;
  if (!valid_dims(B, H, N, D) || !acc || !out || !aligned16(acc) || !aligned16(out))
    return SAGE_ERR_INVALID_ARG;
  if (out_dtype != SAGE_BF16 && out_dtype != SAGE_FP16) return SAGE_ERR_INVALID_ARG;
  if (sn < D || sn % 8 || sh % 8 || sb % 8 || sh < 0 || sb < 0) return SAGE_ERR_INVALID_ARG;
  const int64_t rows = B * H * N;
  const int64_t blocks = (rows + (256 / (D / 8)) - 1) / (256 / (D / 8));
  if (blocks >= (int64_t(1) << 31)) return SAGE_ERR_UNSUPPORTED;
  const bool fp16 = out_dtype == SAGE_FP16;
  const int b = (int)B, h = (int)H, n = (int)N;
  if (D == 128) {
    if (fp16) lse_merge_finalize_kernel<__half, 128><<<(unsigned)blocks, 256, 0, stream>>>(acc, out, sb, sh, sn, b, h, n);
    else lse_merge_finalize_kernel<__nv_bfloat16, 128><<<(unsigned)blocks, 256, 0, stream>>>(acc, out, sb, sh, sn, b, h, n);
  } else {
    if (fp16) lse_merge_finalize_kernel<__half, 64><<<(unsigned)blocks, 256, 0, stream>>>(acc, out, sb, sh, sn, b, h, n);
    else lse_merge_finalize_kernel<__nv_bfloat16, 64><<<(unsigned)blocks, 256, 0, stream>>>(acc, out, sb, sh, sn, b, h, n);
  }
  return launch_status();
}

// ------------------------------------------------- allocation-free variant
// The quantiser's scratch (per-split K sums and V maxima) in a fixed array of
// the library's own device memory, for callers that cannot allocate.  Host
// code cannot use `g_noalloc_scratch` as a pointer (in host code the name is
// a host-side stand-in); its device address is looked up once per device
// with cudaGetSymbolAddress and cached.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SAGE_NOALLOC_SCRATCH_BYTES];

static void* noalloc_scratch_ptr() {
  constexpr int kMaxDevices = 64;
  static std::atomic<void*> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  void* p = cache[dev].load(std::memory_order_acquire);
  if (p) return p;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return nullptr;
  cache[dev].store(p, std::memory_order_release);
  return p;
}

sage_status sage_quantize_qkv_noalloc(const sage_tensor* q, const sage_tensor* k,
                                      const sage_tensor* v, int smooth_k,
                                      const sage_qkv_i8f8* out, sage_stream_t stream) {
  sage_status st;
  if ((st = check_tensor(q)) || (st = check_tensor(k)) || (st = check_tensor(v))) return st;
  if (quant_plan(k->B, k->H, k->N, k->D).part_bytes > SAGE_NOALLOC_SCRATCH_BYTES)
    return SAGE_ERR_WORKSPACE;  // the fixed scratch is too small for these sizes
  void* scratch = noalloc_scratch_ptr();
  if (!scratch) return SAGE_ERR_CUDA;
  return run_quantize(q, k, v, smooth_k, out, scratch, SAGE_NOALLOC_SCRATCH_BYTES, stream);
}

}  // extern "C"
