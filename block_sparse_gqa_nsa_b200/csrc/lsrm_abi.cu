// C entry points of liblsrm_nsa.so: argument validation, workspace carving and
// kernel launches.  Every pointer is caller-owned device memory; nothing here
// allocates.  See include/lsrm_nsa.h for the contract of each call.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "lsrm_common.cuh"

namespace lsrm {
lsrm_status launch_compress(const lsrm_nsa_desc& d, const int32_t* off, const void* q, const void* k, const void* v,
                            float* kc32, void* kc, float* vc32, void* vc, float* qc32, void* qc, cudaStream_t s,
                            const int32_t* kv_row = nullptr);
lsrm_status launch_route_geometric(const lsrm_nsa_desc& d, const int32_t* off, const int32_t* coords, int32_t* cen,
                                   int32_t* idx, uint32_t* status, cudaStream_t s);
lsrm_status launch_route_camera(const lsrm_nsa_desc& d, const int32_t* off, const int32_t* coords, int32_t n_vol,
                                int32_t n_views, const int32_t* proj, int32_t tiles_x, int32_t tiles_y,
                                int32_t tile_px, const int32_t* tile_block, int32_t radius, int32_t k_vol,
                                int32_t* cen, int32_t* idx, uint32_t* status, cudaStream_t stream);
lsrm_status launch_route_score(const lsrm_nsa_desc& d, const int32_t* off, const void* q, const float* kc32,
                               int32_t* idx, float* score, uint32_t* status, cudaStream_t s);
lsrm_status launch_gate_combine(const lsrm_nsa_desc& d, const float* oc, const float* os, const float* ow,
                                const void* gates, void* out, cudaStream_t s);
lsrm_status launch_attn(const lsrm_nsa_desc& d, const int32_t* off, const void* q, const void* k, const void* v,
                        const void* kc, const void* vc, const void* gates, const int32_t* idx, int idx_heads,
                        int route_all, int branches, void* out, float* obranch, float* lse, int lse_stride,
                        int lse_first, uint32_t* status, cudaStream_t stream, void* obr = nullptr);
lsrm_status launch_mixture(const lsrm_nsa_desc& d, const int32_t* off, int32_t bx, const void* q, const void* k,
                           const void* v, const void* gates, void* out, float* lse, uint32_t* status,
                           cudaStream_t stream);
lsrm_status launch_attn_dense(int D, long long n_q, int H, const void* q, const void* kc, const void* vc,
                              long long kc_rows, int n_ckeys, const int* n_ckeys_dev, float tau, float* obranch,
                              float* lse, int32_t* topk_idx, int topk_k, const uint32_t* forced_bits,
                              float* topk_thr, uint32_t* status, cudaStream_t stream,
                              const int32_t* topk_ids = nullptr, const float* rescore_q = nullptr,
                              const float* rescore_k = nullptr, const uint32_t* rescore_kmax = nullptr);
lsrm_status launch_rownorm_max(const float* x, long long rows, uint32_t* out, cudaStream_t s);
lsrm_status launch_pooled_broadcast(const lsrm_nsa_desc& d, const int32_t* off, const float* o_blk,
                                    const float* lse_blk, float* o_cmp, float* lse, cudaStream_t s);
lsrm_status launch_speed3r_forced(const lsrm_nsa_desc& d, const int32_t* off, const void* k, const void* v,
                                  uint32_t* bits, int* pre, int* total, void* kf, void* vf, uint32_t* status,
                                  cudaStream_t s);
lsrm_status launch_key_order(const lsrm_nsa_desc& d, const uint32_t* bits, int32_t* row_of_block,
                             int32_t* block_of_row, uint32_t* bits_part, cudaStream_t s);
lsrm_status launch_speed3r_routed(const lsrm_nsa_desc& d, const int32_t* off, const void* q, const void* k,
                                  const void* v, const void* gates, const int32_t* idx, const float* o_forced,
                                  const float* lse_forced, const float* o_blk, const float* lse_blk, void* out,
                                  float* lse_out, uint32_t* status, cudaStream_t s, void* obr);
lsrm_status launch_speed3r_backward(const lsrm_nsa_desc& d, const int32_t* off, const void* q, const void* k,
                                    const void* v, const void* gates, const int32_t* idx, const float* lse,
                                    const void* obr, const void* dout, void* dq, void* dk, void* dv, void* dgates,
                                    void* ws, uint32_t* status, cudaStream_t s);
lsrm_status launch_backward(const lsrm_nsa_desc& d, const int32_t* off, const void* q, const void* k, const void* v,
                            const void* kc, const void* vc, const void* gates, const int32_t* idx, int idx_heads,
                            const float* lse, const void* dout, void* dq, void* dk, void* dv, void* dgates,
                            unsigned char* ws_bwd, uint32_t* status, cudaStream_t stream, const void* obr);
}  // namespace lsrm

using namespace lsrm;

namespace {

constexpr int BR_CMP = 1, BR_SLC = 2, BR_WIN = 4;

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

lsrm_status check_ws(const lsrm_nsa_desc* d, void* ws) {
  if (ws == nullptr || !aligned(ws, 256)) return LSRM_ERR_WORKSPACE;
  (void)d;
  return LSRM_OK;
}

template <typename T>
T* wsp(void* ws, size_t off) {
  return reinterpret_cast<T*>(reinterpret_cast<unsigned char*>(ws) + off);
}

uint32_t* status_of(void* ws) { return wsp<uint32_t>(ws, 0); }


float tau_of(const lsrm_nsa_desc& d) { return d.scale > 0 ? d.scale : 1.0f / sqrtf((float)d.head_dim); }

#define LSRM_TRY(x)                         \
  do {                                      \
    lsrm_status _s = (x);                   \
    if (_s != LSRM_OK) return _s;           \
  } while (0)

// pooled compressed branch over all B block means, per head (and, with idx, the Speed3R routing:
// top_k blocks by pooled logit outside the forced set); o_blk / lse_blk go to the workspace
lsrm_status pooled_cmp(const lsrm_nsa_desc& d, const void* qc, const void* kc, const void* vc, int32_t* idx,
                       void* ws, cudaStream_t s, const float* qc32 = nullptr, const float* kc32 = nullptr) {
  const Workspace w = workspace_layout(d);
  uint32_t* bits = wsp<uint32_t>(ws, w.fbits);
  float* o_blk = wsp<float>(ws, w.obranch);
  float* l_blk = o_blk + (size_t)d.n_blocks * d.n_q_heads * d.head_dim;
  if (idx != nullptr) {
    if (d.top_k > 64) return LSRM_ERR_UNSUPPORTED;
    if (cudaMemsetAsync(bits, 0, ((size_t)d.n_blocks / 32 + 2) * 4, s) != cudaSuccess) return LSRM_ERR_CUDA;
    if (d.n_forced > 0) {
      // bits only (the prefix/gather outputs of this call are not needed here)
      lsrm_status st = launch_speed3r_forced(d, nullptr, nullptr, nullptr, bits, nullptr, nullptr, nullptr, nullptr,
                                             status_of(ws), s);
      if (st != LSRM_OK) return st;
    }
  }
  const bool exact = idx != nullptr && qc32 != nullptr && kc32 != nullptr;
  if (exact)
    LSRM_TRY(launch_rownorm_max(kc32, (long long)d.n_blocks * d.n_kv_heads, wsp<uint32_t>(ws, w.kmax), s));
  return launch_attn_dense(d.head_dim, d.n_blocks, d.n_q_heads, qc, kc, vc, d.n_blocks, d.n_blocks, nullptr,
                           tau_of(d), o_blk, l_blk, idx, idx ? d.top_k : 0, idx ? bits : nullptr,
                           idx ? wsp<float>(ws, w.rthr) : nullptr, status_of(ws), s, nullptr,
                           exact ? qc32 : nullptr, exact ? kc32 : nullptr, exact ? wsp<uint32_t>(ws, w.kmax) : nullptr);
}


}  // namespace

extern "C" {

size_t lsrm_nsa_workspace_size(const lsrm_nsa_desc* desc) {
  if (check_desc(desc) != LSRM_OK) return 0;
  return workspace_layout(*desc).total;
}

lsrm_status lsrm_nsa_workspace_init(const lsrm_nsa_desc* desc, void* ws, size_t ws_bytes, void* stream) {
  LSRM_TRY(check_desc(desc));
  LSRM_TRY(check_ws(desc, ws));
  if (ws_bytes < workspace_layout(*desc).total) return LSRM_ERR_WORKSPACE;
  if (cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream) != cudaSuccess) return LSRM_ERR_CUDA;
  return LSRM_OK;
}

lsrm_status lsrm_nsa_compress(const lsrm_nsa_desc* desc, const int32_t* off, const void* q_or_null, const void* k,
                              const void* v, float* kc32, void* kc, float* vc32, void* vc, float* qc32_or_null,
                              void* qc_or_null, void* ws, void* stream) {
  LSRM_TRY(check_desc(desc));
  if (off == nullptr || k == nullptr || v == nullptr) return LSRM_ERR_INVALID_ARG;
  if (!aligned(k, 16) || !aligned(v, 16) || (q_or_null && !aligned(q_or_null, 16))) return LSRM_ERR_INVALID_ARG;
  (void)ws;
  return launch_compress(*desc, off, q_or_null, k, v, kc32, kc, vc32, vc, qc32_or_null, qc_or_null,
                         (cudaStream_t)stream);
}

lsrm_status lsrm_route_score_topk(const lsrm_nsa_desc* desc, const int32_t* off, const void* q, const float* kc32,
                                  int32_t* idx, float* score_or_null, void* ws, void* stream) {
  LSRM_TRY(check_desc(desc));
  LSRM_TRY(check_ws(desc, ws));
  if (off == nullptr || q == nullptr || kc32 == nullptr || idx == nullptr) return LSRM_ERR_INVALID_ARG;
  return launch_route_score(*desc, off, q, kc32, idx, score_or_null, status_of(ws), (cudaStream_t)stream);
}

lsrm_status lsrm_route_geometric(const lsrm_nsa_desc* desc, const int32_t* off, const int32_t* coords, int32_t* idx,
                                 void* ws, void* stream) {
  LSRM_TRY(check_desc(desc));
  LSRM_TRY(check_ws(desc, ws));
  if (off == nullptr || coords == nullptr || idx == nullptr) return LSRM_ERR_INVALID_ARG;
  const Workspace w = workspace_layout(*desc);
  return launch_route_geometric(*desc, off, coords, wsp<int32_t>(ws, w.centroids), idx, status_of(ws),
                                (cudaStream_t)stream);
}

lsrm_status lsrm_route_camera(const lsrm_nsa_desc* desc, const int32_t* off, const int32_t* coords,
                              int32_t n_vol_blocks, int32_t n_views, const int32_t* proj, int32_t tiles_x,
                              int32_t tiles_y, int32_t tile_px, const int32_t* tile_block, int32_t radius,
                              int32_t k_vol, int32_t* idx, void* ws, void* stream) {
  LSRM_TRY(check_desc(desc));
  LSRM_TRY(check_ws(desc, ws));
  if (off == nullptr || coords == nullptr || idx == nullptr) return LSRM_ERR_INVALID_ARG;
  const int32_t B = desc->n_blocks, k_img = desc->top_k - k_vol;
  if (n_vol_blocks < 0 || n_vol_blocks > B || k_vol < 0 || k_vol > n_vol_blocks || k_img < 0 ||
      k_img > B - n_vol_blocks)
    return LSRM_ERR_INVALID_ARG;
  if (n_views < 0 || tiles_x < 1 || tiles_y < 1 || tile_px < 1 || radius < 0) return LSRM_ERR_INVALID_ARG;
  if (n_views > 0 && (proj == nullptr || tile_block == nullptr)) return LSRM_ERR_INVALID_ARG;
  const Workspace w = workspace_layout(*desc);
  return launch_route_camera(*desc, off, coords, n_vol_blocks, n_views, proj, tiles_x, tiles_y, tile_px, tile_block,
                             radius, k_vol, wsp<int32_t>(ws, w.centroids), idx, status_of(ws), (cudaStream_t)stream);
}

lsrm_status lsrm_route_pooled_topk(const lsrm_nsa_desc* desc, const void* qc, const void* kc,
                                   const float* qc32_or_null, const float* kc32_or_null, int32_t* idx, void* ws,
                                   void* stream) {
  LSRM_TRY(check_desc(desc));
  LSRM_TRY(check_ws(desc, ws));
  if (!desc->pooled_q || qc == nullptr || kc == nullptr || idx == nullptr) return LSRM_ERR_INVALID_ARG;
  if ((qc32_or_null == nullptr) != (kc32_or_null == nullptr)) return LSRM_ERR_INVALID_ARG;
  if (!aligned(qc32_or_null, 16) || !aligned(kc32_or_null, 16)) return LSRM_ERR_INVALID_ARG;
  // the routing pass is the pooled compressed branch with its top-k; values are not needed, so the
  // keys stand in for them and the branch output stays in the workspace
  return pooled_cmp(*desc, qc, kc, kc, idx, ws, (cudaStream_t)stream, qc32_or_null, kc32_or_null);
}

lsrm_status lsrm_nsa_cmp_attn(const lsrm_nsa_desc* desc, const int32_t* off, const void* q, const void* kc,
                              const void* vc, float* o_cmp, float* lse, void* ws, void* stream) {
  LSRM_TRY(check_desc(desc));
  LSRM_TRY(check_ws(desc, ws));
  if (off == nullptr || q == nullptr || kc == nullptr || vc == nullptr || o_cmp == nullptr)
    return LSRM_ERR_INVALID_ARG;
  if (desc->pooled_q) {
    const Workspace w = workspace_layout(*desc);
    float* o_blk = wsp<float>(ws, w.obranch);
    float* l_blk = o_blk + (size_t)desc->n_blocks * desc->n_q_heads * desc->head_dim;
    LSRM_TRY(pooled_cmp(*desc, q, kc, vc, nullptr, ws, (cudaStream_t)stream));
    return launch_pooled_broadcast(*desc, off, o_blk, l_blk, o_cmp, lse, (cudaStream_t)stream);
  }
  return launch_attn(*desc, off, q, nullptr, nullptr, kc, vc, nullptr, nullptr, 1, 0, BR_CMP, nullptr, o_cmp, lse,
                     1, 0, status_of(ws), (cudaStream_t)stream);
}

lsrm_status lsrm_nsa_select_attn(const lsrm_nsa_desc* desc, const int32_t* off, const void* q, const void* k,
                                 const void* v, const int32_t* idx, int32_t idx_heads, float* o_slc, float* lse,
                                 void* ws, void* stream) {
  LSRM_TRY(check_desc(desc));
  LSRM_TRY(check_ws(desc, ws));
  if (off == nullptr || q == nullptr || k == nullptr || v == nullptr || idx == nullptr || o_slc == nullptr)
    return LSRM_ERR_INVALID_ARG;
  if (idx_heads != 1 && idx_heads != desc->n_kv_heads) return LSRM_ERR_INVALID_ARG;
  return launch_attn(*desc, off, q, k, v, nullptr, nullptr, nullptr, idx, idx_heads, 0, BR_SLC, nullptr, o_slc, lse,
                     1, 0, status_of(ws), (cudaStream_t)stream);
}

lsrm_status lsrm_nsa_window_attn(const lsrm_nsa_desc* desc, const int32_t* off, const void* q, const void* k,
                                 const void* v, float* o_win, float* lse, void* ws, void* stream) {
  LSRM_TRY(check_desc(desc));
  LSRM_TRY(check_ws(desc, ws));
  if (off == nullptr || q == nullptr || k == nullptr || v == nullptr || o_win == nullptr) return LSRM_ERR_INVALID_ARG;
  if (desc->window == 0) return LSRM_ERR_INVALID_ARG;
  return launch_attn(*desc, off, q, k, v, nullptr, nullptr, nullptr, nullptr, 1, 0, BR_WIN, nullptr, o_win, lse, 1,
                     0, status_of(ws), (cudaStream_t)stream);
}

lsrm_status lsrm_nsa_gate_combine(const lsrm_nsa_desc* desc, const float* o_cmp, const float* o_slc,
                                  const float* o_win_or_null, const void* gates, void* out, void* stream) {
  LSRM_TRY(check_desc(desc));
  if (o_cmp == nullptr || o_slc == nullptr || gates == nullptr || out == nullptr) return LSRM_ERR_INVALID_ARG;
  if (desc->n_gates == 3 && o_win_or_null == nullptr) return LSRM_ERR_INVALID_ARG;
  if (!aligned(o_cmp, 16) || !aligned(o_slc, 16) || !aligned(out, 8) ||
      (o_win_or_null && !aligned(o_win_or_null, 16)))
    return LSRM_ERR_INVALID_ARG;
  return launch_gate_combine(*desc, o_cmp, o_slc, o_win_or_null, gates, out, (cudaStream_t)stream);
}

lsrm_status lsrm_nsa_attend(const lsrm_nsa_desc* desc, const int32_t* off, const void* q, const void* k,
                            const void* v, const void* kc, const void* vc, const void* gates, const int32_t* idx,
                            int32_t idx_heads, int32_t route_all, void* out, float* lse_or_null, void* ws,
                            void* stream) {
  LSRM_TRY(check_desc(desc));
  LSRM_TRY(check_ws(desc, ws));
  if (desc->pooled_q) return LSRM_ERR_UNSUPPORTED;
  if (off == nullptr || q == nullptr || k == nullptr || v == nullptr || kc == nullptr || vc == nullptr ||
      gates == nullptr || out == nullptr || (!route_all && idx == nullptr))
    return LSRM_ERR_INVALID_ARG;
  if (idx_heads != 1 && idx_heads != desc->n_kv_heads) return LSRM_ERR_INVALID_ARG;
  if (route_all && desc->top_k != desc->n_blocks) return LSRM_ERR_INVALID_ARG;
  const int branches = BR_CMP | BR_SLC | ((desc->n_gates == 3 && desc->window > 0) ? BR_WIN : 0);
  return launch_attn(*desc, off, q, k, v, kc, vc, gates, idx, idx_heads, route_all ? 1 : 0, branches, out, nullptr,
                     lse_or_null, desc->n_gates, 0, status_of(ws), (cudaStream_t)stream);
}

lsrm_status lsrm_nsa_mixture(const lsrm_nsa_desc* desc, const int32_t* off, int32_t n_blocks_x, const void* q,
                             const void* k, const void* v, const void* gates, void* out, float* lse_or_null, void* ws,
                             void* stream) {
  LSRM_TRY(check_desc(desc));
  LSRM_TRY(check_ws(desc, ws));
  if (desc->pooled_q || desc->n_gates != 2 || desc->n_forced != 0) return LSRM_ERR_INVALID_ARG;
  if (off == nullptr || q == nullptr || k == nullptr || v == nullptr || gates == nullptr || out == nullptr)
    return LSRM_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16)) return LSRM_ERR_INVALID_ARG;
  if (n_blocks_x < 0 || n_blocks_x > desc->n_blocks) return LSRM_ERR_INVALID_ARG;
  return launch_mixture(*desc, off, n_blocks_x, q, k, v, gates, out, lse_or_null, status_of(ws), (cudaStream_t)stream);
}

lsrm_status lsrm_nsa_forward(const lsrm_nsa_desc* desc, const int32_t* off, const void* q, const void* k,
                             const void* v, const void* gates, const int32_t* coords_or_null, int32_t route_mode,
                             void* out, int32_t* idx_inout, float* lse_or_null, void* obr_or_null, void* ws,
                             void* stream) {
  LSRM_TRY(check_desc(desc));
  LSRM_TRY(check_ws(desc, ws));
  if (off == nullptr || q == nullptr || k == nullptr || v == nullptr || gates == nullptr || out == nullptr)
    return LSRM_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(obr_or_null, 16)) return LSRM_ERR_INVALID_ARG;
  const lsrm_nsa_desc& d = *desc;
  const Workspace w = workspace_layout(d);
  cudaStream_t s = (cudaStream_t)stream;
  float* kc32 = wsp<float>(ws, w.kc32);
  float* vc32 = wsp<float>(ws, w.vc32);
  void* kc16 = wsp<void>(ws, w.kc16);
  void* vc16 = wsp<void>(ws, w.vc16);
  int32_t* idx = idx_inout != nullptr ? idx_inout : wsp<int32_t>(ws, w.idx);

  if (d.pooled_q) {
    // Speed3R: pooled Q/K/V; pooled compressed branch + routing; forced part of the selected
    // branch (dense, tensor cores); routed part merged with it, plus the gated combine
    if (route_mode != LSRM_ROUTE_SCORE && route_mode != LSRM_ROUTE_GIVEN) return LSRM_ERR_INVALID_ARG;
    if (route_mode == LSRM_ROUTE_GIVEN && idx_inout == nullptr) return LSRM_ERR_INVALID_ARG;
    if (d.head_dim != 64 || d.max_block_len > 16) return LSRM_ERR_UNSUPPORTED;
    void* qc16 = wsp<void>(ws, w.qc16);
    int* ftotal = wsp<int>(ws, w.ftotal);
    LSRM_TRY(launch_speed3r_forced(d, off, k, v, wsp<uint32_t>(ws, w.fbits), wsp<int>(ws, w.fpre), ftotal,
                                   wsp<void>(ws, w.kf), wsp<void>(ws, w.vf), status_of(ws), s));
    // the pooled keys are stored non-forced first (in block order), then the forced blocks, so
    // the routing passes meet forced keys only in their last chunks; rows map back to blocks
    int32_t* row_of_block = wsp<int32_t>(ws, w.krow);
    int32_t* block_of_row = wsp<int32_t>(ws, w.kblk);
    uint32_t* bits_part = wsp<uint32_t>(ws, w.fbits_part);
    LSRM_TRY(launch_key_order(d, wsp<uint32_t>(ws, w.fbits), row_of_block, block_of_row, bits_part, s));
    const bool route = route_mode == LSRM_ROUTE_SCORE;
    if (route && d.top_k > 64) return LSRM_ERR_UNSUPPORTED;
    // the routing ranks the fp32 logits of the means: their fp32 copies (keys in row order) and
    // the largest |pooled key| feed the exact ranking of the candidates
    float* qc32 = wsp<float>(ws, w.qc32);
    LSRM_TRY(launch_compress(d, off, q, k, v, route ? kc32 : nullptr, kc16, nullptr, vc16, qc32, qc16, s,
                             row_of_block));
    uint32_t* kmax = wsp<uint32_t>(ws, w.kmax);
    if (route) LSRM_TRY(launch_rownorm_max(kc32, (long long)d.n_blocks * d.n_kv_heads, kmax, s));
    float* o_blk = wsp<float>(ws, w.obranch);
    float* l_blk = o_blk + (size_t)d.n_blocks * d.n_q_heads * d.head_dim;
    LSRM_TRY(launch_attn_dense(d.head_dim, d.n_blocks, d.n_q_heads, qc16, kc16, vc16, d.n_blocks, d.n_blocks,
                               nullptr, tau_of(d), o_blk, l_blk, route ? idx : nullptr, route ? d.top_k : 0,
                               route ? bits_part : nullptr, route ? wsp<float>(ws, w.rthr) : nullptr,
                               status_of(ws), s, route ? block_of_row : nullptr, route ? qc32 : nullptr,
                               route ? kc32 : nullptr, route ? kmax : nullptr));
    float* ofrc = wsp<float>(ws, w.ofrc);
    float* lfrc = wsp<float>(ws, w.lfrc);
    const long long cap = (long long)(d.n_forced > 0 ? d.n_forced : 1) * d.max_block_len;
    LSRM_TRY(launch_attn_dense(d.head_dim, d.n_tokens, d.n_q_heads, q, wsp<void>(ws, w.kf), wsp<void>(ws, w.vf),
                               cap, 0, ftotal, tau_of(d), ofrc, lfrc, nullptr, 0, nullptr, nullptr, status_of(ws), s));
    return launch_speed3r_routed(d, off, q, k, v, gates, idx, ofrc, lfrc, o_blk, l_blk, out, lse_or_null,
                                 status_of(ws), s, obr_or_null);
  }

  LSRM_TRY(launch_compress(d, off, nullptr, k, v, route_mode == LSRM_ROUTE_SCORE ? kc32 : nullptr, kc16, nullptr,
                           vc16, nullptr, nullptr, s));
  int idx_heads = 1, route_all = 0;
  switch (route_mode) {
    case LSRM_ROUTE_GIVEN:
      if (idx_inout == nullptr) return LSRM_ERR_INVALID_ARG;
      idx_heads = d.n_kv_heads;  // a caller-given index uses the per-group layout
      break;
    case LSRM_ROUTE_SCORE:
      idx_heads = d.n_kv_heads;
      LSRM_TRY(launch_route_score(d, off, q, kc32, idx, nullptr, status_of(ws), s));
      break;
    case LSRM_ROUTE_GEOMETRIC:
      if (coords_or_null == nullptr) return LSRM_ERR_INVALID_ARG;
      idx_heads = 1;
      LSRM_TRY(launch_route_geometric(d, off, coords_or_null, wsp<int32_t>(ws, w.centroids), idx, status_of(ws), s));
      break;
    case LSRM_ROUTE_ALL:
      if (d.top_k != d.n_blocks) return LSRM_ERR_INVALID_ARG;
      route_all = 1;
      break;
    default:
      return LSRM_ERR_INVALID_ARG;
  }
  const int branches = BR_CMP | BR_SLC | ((d.n_gates == 3 && d.window > 0) ? BR_WIN : 0);
  return launch_attn(d, off, q, k, v, kc16, vc16, gates, idx, idx_heads, route_all, branches, out, nullptr,
                     lse_or_null, d.n_gates, 0, status_of(ws), s, obr_or_null);
}

lsrm_status lsrm_nsa_backward(const lsrm_nsa_desc* desc, const int32_t* off, const void* q, const void* k,
                              const void* v, const void* gates, const int32_t* idx, int32_t idx_heads,
                              const float* lse, const void* obr_or_null, const void* dout, void* dq, void* dk, void* dv,
                              void* dgates, void* ws, void* stream) {
  LSRM_TRY(check_desc(desc));
  LSRM_TRY(check_ws(desc, ws));
  if (off == nullptr || q == nullptr || k == nullptr || v == nullptr || gates == nullptr || idx == nullptr ||
      lse == nullptr || dout == nullptr || dq == nullptr || dk == nullptr || dv == nullptr || dgates == nullptr)
    return LSRM_ERR_INVALID_ARG;
  if (desc->pooled_q) {
    // Speed3R: per-head routing lists and the forward's saved branch outputs are required
    if (idx_heads != desc->n_q_heads || obr_or_null == nullptr) return LSRM_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(obr_or_null, 16) || !aligned(dout, 16) ||
        !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16))
      return LSRM_ERR_INVALID_ARG;
    return launch_speed3r_backward(*desc, off, q, k, v, gates, idx, lse, obr_or_null, dout, dq, dk, dv, dgates, ws,
                                   status_of(ws), (cudaStream_t)stream);
  }
  if (idx_heads != 1 && idx_heads != desc->n_kv_heads) return LSRM_ERR_INVALID_ARG;
  if (!aligned(obr_or_null, 16) || !aligned(dout, 16)) return LSRM_ERR_INVALID_ARG;
  const Workspace w = workspace_layout(*desc);
  cudaStream_t s = (cudaStream_t)stream;
  void* kc16 = wsp<void>(ws, w.kc16);
  void* vc16 = wsp<void>(ws, w.vc16);
  LSRM_TRY(launch_compress(*desc, off, nullptr, k, v, nullptr, kc16, nullptr, vc16, nullptr, nullptr, s));
  return launch_backward(*desc, off, q, k, v, kc16, vc16, gates, idx, idx_heads, lse, dout, dq, dk, dv, dgates,
                         wsp<unsigned char>(ws, w.bwd), status_of(ws), s, obr_or_null);
}

lsrm_status lsrm_nsa_last_device_status(void* ws, void* stream) {
  if (ws == nullptr || !aligned(ws, 256)) return LSRM_ERR_WORKSPACE;
  uint32_t word = 0;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess) return LSRM_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return LSRM_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, sizeof(word), s) != cudaSuccess) return LSRM_ERR_CUDA;
  if (word == 0) return LSRM_OK;
  for (int st = 1; st < 32; ++st)
    if (word & (1u << (st - 1))) return (lsrm_status)st;
  return LSRM_ERR_CUDA;
}

const char* lsrm_status_string(lsrm_status s) {
  switch (s) {
    case LSRM_OK: return "ok";
    case LSRM_ERR_INVALID_ARG: return "invalid argument";
    case LSRM_ERR_UNSUPPORTED: return "unsupported configuration";
    case LSRM_ERR_CUDA: return "CUDA error";
    case LSRM_ERR_TIMEOUT: return "device wait timed out";
    case LSRM_ERR_BOUNDS: return "device bounds check failed";
    case LSRM_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
  }
  return "unknown status";
}

}  // extern "C"
