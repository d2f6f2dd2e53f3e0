// Shared device/host helpers of the sm_100a LSRM NSA library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "lsrm_nsa.h"

namespace lsrm {

// Blocks of up to 512 tokens (the 8x8x8 volume bricks) in the forward; the backward, score routing
// and the pooled-query variant keep their own (smaller) limits.
constexpr int kMaxBlockLen = 512;

// Descriptor checks shared by every entry point (host side).
inline lsrm_status check_desc(const lsrm_nsa_desc* d) {
  if (d == nullptr) return LSRM_ERR_INVALID_ARG;
  if (d->n_tokens < 1 || d->n_blocks < 1 || d->n_blocks > d->n_tokens) return LSRM_ERR_INVALID_ARG;
  if (d->n_tokens > (int64_t)INT32_MAX) return LSRM_ERR_UNSUPPORTED;
  if (d->max_block_len < 1 || d->max_block_len > kMaxBlockLen) return LSRM_ERR_INVALID_ARG;
  if (d->n_kv_heads < 1 || d->n_q_heads < d->n_kv_heads || d->n_q_heads % d->n_kv_heads) return LSRM_ERR_INVALID_ARG;
  if (d->head_dim != 32 && d->head_dim != 64) return LSRM_ERR_UNSUPPORTED;
  if (d->top_k < 1 || d->top_k > d->n_blocks) return LSRM_ERR_INVALID_ARG;
  if (d->window < 0 || (d->window & 1)) return LSRM_ERR_INVALID_ARG;
  if (!(d->scale >= 0.0f) || isinf(d->scale)) return LSRM_ERR_INVALID_ARG;
  if (d->pooled_q != 0 && d->pooled_q != 1) return LSRM_ERR_INVALID_ARG;
  if (d->n_gates != 2 && d->n_gates != 3) return LSRM_ERR_INVALID_ARG;
  if (d->n_forced < 0 || (d->n_forced > 0 && d->forced_blocks == nullptr)) return LSRM_ERR_INVALID_ARG;
  if (d->pooled_q && (d->n_q_heads != d->n_kv_heads || d->n_gates != 2)) return LSRM_ERR_INVALID_ARG;
  if (d->pooled_q && d->top_k + d->n_forced > d->n_blocks) return LSRM_ERR_INVALID_ARG;
  return LSRM_OK;
}

// ---- device status word (first 4 bytes of the workspace) ---------------------------------------
// Kernels OR a status bit in; the host reads and clears it.  Bit i set <=> status (i+1) was raised.
__device__ __forceinline__ void raise_status(uint32_t* status, lsrm_status s) {
  if (status) atomicOr(status, 1u << ((int)s - 1));
}

// ---- workspace layout ----------------------------------------------------------------------------
struct Workspace {
  size_t status, kc32, vc32, kc16, vc16, qc32, qc16, centroids, idx, obranch, bwd;
  // pooled-query (Speed3R) path: forced-block bitmap, prefix and total, gathered forced K / V,
  // and the forced part of the selected branch per token
  size_t fbits, fpre, ftotal, kf, vf, ofrc, lfrc;
  size_t rthr;  // per (block, head) lower bound on the k-th routing logit
  // pooled keys stored non-forced first: row of each block, block of each row, and the forced
  // bitmap over rows
  size_t krow, kblk, fbits_part;
  size_t kmax;  // largest |pooled key| (float bits), the width of the exact-ranking gate
  size_t total;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// backward scratch (inside the workspace's backward region): per-row constants of every branch
// (LSE in log2 units, gate, Delta, token position in its block), fp32 selected + window parts of
// dK / dV, per-split compressed-branch partials, and the inverse routing lists
constexpr int kBwdSplits = 32;  // query splits of the compressed-key pass
struct BwdWs {
  size_t rowc, dk_tok, dv_tok, dkc, dvc, inv_count, inv_cursor, inv_start, inv_list, total;
};
inline BwdWs bwd_layout(const lsrm_nsa_desc& d, int idx_heads) {
  BwdWs w{};
  size_t o = 0;
  const size_t N = (size_t)d.n_tokens, B = (size_t)d.n_blocks, Hq = (size_t)d.n_q_heads, Hkv = (size_t)d.n_kv_heads;
  const size_t D = (size_t)d.head_dim, nl = B * (size_t)idx_heads, NG = (size_t)(d.n_gates > 0 ? d.n_gates : 0);
  const size_t K = (size_t)(d.top_k > 0 ? d.top_k : 0);
  w.rowc = o;       o = align256(o + NG * N * Hq * 16);
  w.dk_tok = o;     o = align256(o + N * Hkv * D * 4);
  w.dv_tok = o;     o = align256(o + N * Hkv * D * 4);
  w.dkc = o;        o = align256(o + (size_t)kBwdSplits * B * Hkv * D * 4);
  w.dvc = o;        o = align256(o + (size_t)kBwdSplits * B * Hkv * D * 4);
  w.inv_count = o;  o = align256(o + nl * 4);
  w.inv_cursor = o; o = align256(o + nl * 4);
  w.inv_start = o;  o = align256(o + (nl + 1) * 4);
  w.inv_list = o;   o = align256(o + nl * K * 4);
  w.total = o;
  return w;
}

// backward scratch of the pooled-query (Speed3R) layer: the pooled branch's upstream gradient
// (bf16, for the tensor cores), its LSE (log2 units) and Delta per (block, head) as float2; the pooled
// gradients dQbar, dKbar, dVbar (fp32); per (token, head) the selected branch's LSE (log2 units) and
// Delta as float2 and its upstream gradient g_slc dO (bf16); the forced part of dq (fp32); dK, dV of
// the packed forced tokens (fp32, one partial per split of the query rows) and each packed token's
// (token, block); the inverse routing lists per (block, head), the lists longer than one segment
// (their ids; per list its first segment and per segment its list) and each such segment's partial
// dK, dV (fp32, 16 rows each)
constexpr int kForcedSplits = 8;
constexpr int kListSeg = 256;  // inverse-list entries per segment of the routed dK / dV pass
struct PooledBwdWs {
  size_t gbar16, rowcb, dqbar, dkbar, dvbar, rowc, dos16, dqf, dkf, dvf, fmap;
  size_t inv_count, inv_cursor, inv_start, inv_list, n_long, long_ids, seg_count, seg_start, seg_list, seg_part;
  size_t max_segs, total;
};
inline PooledBwdWs pooled_bwd_layout(const lsrm_nsa_desc& d) {
  PooledBwdWs w{};
  size_t o = 0;
  const size_t N = (size_t)d.n_tokens, B = (size_t)d.n_blocks, H = (size_t)d.n_q_heads, D = (size_t)d.head_dim;
  const size_t nf_tok = (size_t)(d.n_forced > 0 ? d.n_forced : 0) * (size_t)d.max_block_len;
  const size_t nl = B * H, K = (size_t)(d.top_k > 0 ? d.top_k : 0);
  w.gbar16 = o;     o = align256(o + B * H * D * 2);
  w.rowcb = o;      o = align256(o + B * H * 8);
  w.dqbar = o;      o = align256(o + B * H * D * 4);
  w.dkbar = o;      o = align256(o + B * H * D * 4);
  w.dvbar = o;      o = align256(o + B * H * D * 4);
  w.rowc = o;       o = align256(o + N * H * 8);
  w.dos16 = o;      o = align256(o + N * H * D * 2);
  w.dqf = o;        o = align256(o + N * H * D * 4);
  w.dkf = o;        o = align256(o + (size_t)kForcedSplits * nf_tok * H * D * 4);
  w.dvf = o;        o = align256(o + (size_t)kForcedSplits * nf_tok * H * D * 4);
  w.fmap = o;       o = align256(o + nf_tok * 8);
  w.inv_count = o;  o = align256(o + nl * 4);
  w.inv_cursor = o; o = align256(o + nl * 4);
  w.inv_start = o;  o = align256(o + (nl + 1) * 4);
  w.inv_list = o;   o = align256(o + nl * K * 4);
  w.n_long = o;     o = align256(o + 16);
  w.long_ids = o;   o = align256(o + nl * 4);
  w.seg_count = o;  o = align256(o + nl * 4);
  w.seg_start = o;  o = align256(o + (nl + 1) * 4);
  // a list longer than kListSeg has ceil(n / kListSeg) < 2 n / kListSeg segments
  w.max_segs = 2 * nl * K / (size_t)kListSeg + 1;
  w.seg_list = o;   o = align256(o + w.max_segs * 4);
  w.seg_part = o;   o = align256(o + w.max_segs * 2 * 16 * D * 4);
  w.total = o;
  return w;
}

inline Workspace workspace_layout(const lsrm_nsa_desc& d) {
  Workspace w{};
  size_t o = 0;
  const size_t B = (size_t)d.n_blocks, Hkv = (size_t)d.n_kv_heads, Hq = (size_t)d.n_q_heads, D = (size_t)d.head_dim;
  const size_t N = (size_t)d.n_tokens;
  w.status = o;    o = align256(o + 16);
  w.kc32 = o;      o = align256(o + B * Hkv * D * 4);
  w.vc32 = o;      o = align256(o + B * Hkv * D * 4);
  w.kc16 = o;      o = align256(o + B * Hkv * D * 2);
  w.vc16 = o;      o = align256(o + B * Hkv * D * 2);
  const size_t qcn = d.pooled_q ? B * Hq * D : 0;
  w.qc32 = o;      o = align256(o + qcn * 4);
  w.qc16 = o;      o = align256(o + qcn * 2);
  w.centroids = o; o = align256(o + B * 3 * 4);
  // routing indices when the caller passes none: [B][max(Hq,Hkv)][k]
  const size_t ih = d.pooled_q ? Hq : Hkv;
  w.idx = o;       o = align256(o + B * ih * (size_t)(d.top_k > 0 ? d.top_k : 1) * 4);
  // pooled compressed-branch output [B][Hq][d] fp32 (Speed3R) + its LSE [B][Hq]
  w.obranch = o;   o = align256(o + (d.pooled_q ? B * Hq * (D + 1) * 4 : 0));
  // backward scratch, sized for per-group routing lists (the larger case)
  w.bwd = o;       o = align256(o + (d.pooled_q ? pooled_bwd_layout(d).total
                                                : bwd_layout(d, d.n_kv_heads > 0 ? d.n_kv_heads : 1).total));
  const size_t nf = d.pooled_q ? (size_t)(d.n_forced > 0 ? d.n_forced : 0) : 0;
  const size_t nf_tok = nf * (size_t)d.max_block_len;
  w.fbits = o;     o = align256(o + (d.pooled_q ? (B / 32 + 2) * 4 : 0));
  w.fpre = o;      o = align256(o + (d.pooled_q ? (nf + 1) * 4 : 0));
  w.ftotal = o;    o = align256(o + (d.pooled_q ? 16 : 0));
  w.kf = o;        o = align256(o + nf_tok * Hkv * D * 2);
  w.vf = o;        o = align256(o + nf_tok * Hkv * D * 2);
  w.ofrc = o;      o = align256(o + (d.pooled_q ? N * Hq * D * 4 : 0));
  w.lfrc = o;      o = align256(o + (d.pooled_q ? N * Hq * 4 : 0));
  w.rthr = o;      o = align256(o + (d.pooled_q ? B * Hq * 4 : 0));
  w.krow = o;      o = align256(o + (d.pooled_q ? B * 4 : 0));
  w.kblk = o;      o = align256(o + (d.pooled_q ? B * 4 : 0));
  w.fbits_part = o; o = align256(o + (d.pooled_q ? (B / 32 + 2) * 4 : 0));
  w.kmax = o;      o = align256(o + (d.pooled_q ? 16 : 0));
  w.total = o;
  return w;
}

// ---- small PTX wrappers (mma.sync bring-up path) -------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool pred) {
  const int n = pred ? 16 : 0;  // src-size 0 zero-fills the destination
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(smem)), "l"(gmem), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ void ldmatrix_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                                  uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

// D = A(16x16 bf16, row) * B(16x8 bf16, col) + C (fp32)
__device__ __forceinline__ void mma_bf16_16816(float* c, const uint32_t* a, const uint32_t* b) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;\n" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

}  // namespace lsrm
