// S3-S7 attention branches with mma.sync (m16n8k16 bf16 -> fp32) tensor cores.
//
// One CTA = one (query block a, KV group g, chunk of 128 query rows).  A query row
// is a (token, head) pair of the block and the group; rows are token-major, so the
// 16 heads of one token that share a KV head form one 16-row MMA tile.  The CTA
// streams 64-key chunks of three key sets through a double-buffered cp.async
// pipeline and keeps one online-softmax state per branch:
//   compressed branch: the B block means (kc, vc) of group g — LSRM page, 方法
//     (compressed features give global coarse context); Speed3R page 2.1;
//   selected branch: every token of the routed blocks idx[a][g] plus the forced
//     blocks — LSRM page, selected active blocks give local detail;
//   window branch: the query's own block, band r(t)-w/2 .. r(t)+w/2-1 — LSRM
//     page, sequence-parallel paragraph (window attention runs inside blocks).
// The gated sum (LSRM page, gate equations) is folded into the epilogue, so the
// branch outputs never reach HBM in the fused mode.
#include "lsrm_common.cuh"

namespace lsrm {

constexpr int kAttnThreads = 256;  // 8 warps x 16 rows
constexpr int kRowsPerCta = 128;
constexpr int kKeysPerChunk = 64;
constexpr int kMaxSel = 1024;       // selected-set entries (routed + forced blocks) per CTA

enum : int { BR_CMP = 1, BR_SLC = 2, BR_WIN = 4 };

struct AttnParams {
  const int32_t* off;
  const uint16_t* q;       // [N][Hq][D]
  const uint16_t* k;       // [N][Hkv][D]
  const uint16_t* v;
  const uint16_t* kc;      // [B][Hkv][D] bf16 block means
  const uint16_t* vc;
  const uint16_t* gates;   // [N][Hq][n_gates]
  const int32_t* idx;      // [B][idx_heads][top_k]
  const int32_t* forced;   // [n_forced]
  uint16_t* out;           // fused mode: [N][Hq][D] bf16
  float* obranch;          // single-branch mode: [N][Hq][D] fp32
  float* lse;              // [N][Hq][lse_stride] (natural log), optional
  uint32_t* status;
  long long N;
  int B, Hq, Hkv, G, top_k, idx_heads, n_forced, window, n_gates, route_all;
  int branches;            // BR_* mask
  int lse_stride;          // entries per (t,h) in lse
  int lse_first;           // lse slot of the first computed branch (branch order cmp, slc, win)
  float scale_log2;        // tau * log2(e)
};

template <int D>
struct Smem {
  static constexpr int kRowBytes = D * 2;
  static constexpr int kChunksPerRow = D / 8;  // 16-byte chunks
  uint16_t q[kRowsPerCta * D];
  uint16_t kbuf[2][kKeysPerChunk * D];
  uint16_t vbuf[2][kKeysPerChunk * D];
  int32_t sel[kMaxSel];       // selected block ids
  int32_t pre[kMaxSel + 1];   // prefix token counts of sel
  int32_t n_sel;
};

// byte offset of 16-byte chunk `ch` of row `row` in a swizzled [rows][D] bf16 tile
template <int D>
__device__ __forceinline__ uint32_t swz(int row, int ch) {
  if (D == 32) return (uint32_t)(row * 64 + ((ch ^ ((row >> 1) & 3)) << 4));
  return (uint32_t)(row * 128 + ((ch ^ (row & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1) nsa_attn_mma_kernel(const AttnParams p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  Smem<D>& S = *reinterpret_cast<Smem<D>*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int chunk_id = blockIdx.x, g = blockIdx.y, a = blockIdx.z;
  const int t0 = p.off[a], n_a = p.off[a + 1] - t0;
  const int rows_total = n_a * p.G;
  const int row0 = chunk_id * kRowsPerCta;
  if (row0 >= rows_total) return;

  // ---- selected set (routed + forced) and its prefix token counts ----
  if (p.branches & BR_SLC) {
    if (tid == 0) {
      int n = 0, tot = 0;
      if (!p.route_all) {
        const int32_t* r = p.idx + ((size_t)a * p.idx_heads + (p.idx_heads == 1 ? 0 : g)) * p.top_k;
        for (int i = 0; i < p.n_forced + p.top_k && n < kMaxSel; ++i) {
          int j = i < p.n_forced ? p.forced[i] : r[i - p.n_forced];
          if (j < 0 || j >= p.B) { raise_status(p.status, LSRM_ERR_BOUNDS); continue; }
          S.sel[n] = j;
          S.pre[n] = tot;
          tot += p.off[j + 1] - p.off[j];
          ++n;
        }
      } else {
        tot = (int)p.N;
      }
      S.pre[n] = tot;
      S.n_sel = n;
    }
  }

  // ---- Q tile: rows row0 .. row0+127 of (a, g) ----
  for (int e = tid; e < kRowsPerCta * Smem<D>::kChunksPerRow; e += kAttnThreads) {
    const int r = e / Smem<D>::kChunksPerRow, ch = e % Smem<D>::kChunksPerRow;
    const int rr = row0 + r;
    const bool ok = rr < rows_total;
    const int t = t0 + (ok ? rr / p.G : 0), h = g * p.G + (ok ? rr % p.G : 0);
    const uint16_t* src = p.q + ((size_t)t * p.Hq + h) * D + ch * 8;
    cp_async16(reinterpret_cast<unsigned char*>(S.q) + swz<D>(r, ch), src, ok);
  }
  cp_async_commit();
  __syncthreads();  // sel/pre visible

  const int n_sel_tok = (p.branches & BR_SLC) ? S.pre[S.n_sel] : 0;
  const int n_cmp_chunks = (p.branches & BR_CMP) ? (p.B + kKeysPerChunk - 1) / kKeysPerChunk : 0;
  const int n_slc_chunks = (n_sel_tok + kKeysPerChunk - 1) / kKeysPerChunk;
  const int n_win_chunks = ((p.branches & BR_WIN) && p.window > 0) ? 1 : 0;
  const int n_chunks = n_cmp_chunks + n_slc_chunks + n_win_chunks;

  // which branch a flat chunk index belongs to, and its first key position
  auto chunk_branch = [&](int c, int& pos0) -> int {
    if (c < n_cmp_chunks) { pos0 = c * kKeysPerChunk; return 0; }
    c -= n_cmp_chunks;
    if (c < n_slc_chunks) { pos0 = c * kKeysPerChunk; return 1; }
    pos0 = 0;
    return 2;
  };
  // number of valid keys in a chunk
  auto chunk_keys = [&](int br, int pos0) -> int {
    const int total = br == 0 ? p.B : (br == 1 ? n_sel_tok : n_a);
    return min(kKeysPerChunk, total - pos0);
  };

  auto load_chunk = [&](int c, int buf) {
    int pos0;
    const int br = chunk_branch(c, pos0);
    const int nk = chunk_keys(br, pos0);
    for (int e = tid; e < kKeysPerChunk * Smem<D>::kChunksPerRow; e += kAttnThreads) {
      const int kk = e / Smem<D>::kChunksPerRow, ch = e % Smem<D>::kChunksPerRow;
      const bool ok = kk < nk;
      const uint16_t *ks, *vs;
      if (br == 0) {
        const size_t base = ((size_t)(ok ? pos0 + kk : 0) * p.Hkv + g) * D + ch * 8;
        ks = p.kc + base;
        vs = p.vc + base;
      } else {
        long long u = 0;
        if (ok) {
          const int pos = pos0 + kk;
          if (br == 2) {
            u = t0 + pos;
          } else if (p.route_all) {
            u = pos;
          } else {
            // binary search pos in the prefix counts of the selected set
            int lo = 0, hi = S.n_sel - 1;
            while (lo < hi) {
              const int mid = (lo + hi + 1) >> 1;
              if (S.pre[mid] <= pos) lo = mid; else hi = mid - 1;
            }
            u = p.off[S.sel[lo]] + (pos - S.pre[lo]);
          }
        }
        const size_t base = ((size_t)u * p.Hkv + g) * D + ch * 8;
        ks = p.k + base;
        vs = p.v + base;
      }
      cp_async16(reinterpret_cast<unsigned char*>(S.kbuf[buf]) + swz<D>(kk, ch), ks, ok);
      cp_async16(reinterpret_cast<unsigned char*>(S.vbuf[buf]) + swz<D>(kk, ch), vs, ok);
    }
    cp_async_commit();
  };

  if (n_chunks > 0) load_chunk(0, 0);

  // ---- per-warp state ----
  constexpr int KT = D / 16;   // k-steps of QK^T
  constexpr int NT = D / 8;    // n-tiles of the output
  const int gq = lane >> 2, cq = lane & 3;
  // rows of this lane: wr0 = warp*16 + gq, wr1 = wr0 + 8
  const int wr[2] = {warp * 16 + gq, warp * 16 + gq + 8};
  int tok_local[2], head[2];
  bool rvalid[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int rr = row0 + wr[i];
    rvalid[i] = rr < rows_total;
    tok_local[i] = rvalid[i] ? rr / p.G : 0;
    head[i] = g * p.G + (rvalid[i] ? rr % p.G : 0);
  }

  uint32_t qa[KT][4];
  float o[NT][4];
  float out_acc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) { o[n][e] = 0.f; out_acc[n][e] = 0.f; }
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  int cur_br = -1;
  bool q_loaded = false;

  // finish a branch: normalise, then either fold into the gated sum or store it
  auto finish_branch = [&](int br) {
    float l_tot[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      float l = l_run[i];
      l += __shfl_xor_sync(0xffffffffu, l, 1);
      l += __shfl_xor_sync(0xffffffffu, l, 2);
      l_tot[i] = l;
    }
    float inv[2], gate[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      inv[i] = l_tot[i] > 0.f ? 1.f / l_tot[i] : 0.f;
      gate[i] = 0.f;
      if (p.out != nullptr && rvalid[i]) {
        const size_t gi = ((size_t)(t0 + tok_local[i]) * p.Hq + head[i]) * p.n_gates + br;
        gate[i] = bf16_to_f32(p.gates[gi]);
      }
      if (p.lse != nullptr && rvalid[i] && cq == 0) {
        int slot = p.lse_first;
        if (p.branches & BR_CMP) slot += (br > 0);
        if ((p.branches & BR_SLC) && br > 1) slot += 1;
        const float L = l_tot[i] > 0.f ? (m_run[i] + __log2f(l_tot[i])) * 0.6931471805599453f : -INFINITY;
        p.lse[((size_t)(t0 + tok_local[i]) * p.Hq + head[i]) * p.lse_stride + slot] = L;
      }
    }
#pragma unroll
    for (int n = 0; n < NT; ++n) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = e >> 1;
        const float val = o[n][e] * inv[i];
        if (p.out != nullptr) out_acc[n][e] += gate[i] * val;
        o[n][e] = val;
      }
      if (p.obranch != nullptr) {
#pragma unroll
        for (int i = 0; i < 2; ++i)
          if (rvalid[i]) {
            float2* dst = reinterpret_cast<float2*>(
                p.obranch + ((size_t)(t0 + tok_local[i]) * p.Hq + head[i]) * D + n * 8 + 2 * cq);
            *dst = make_float2(o[n][2 * i], o[n][2 * i + 1]);
          }
      }
    }
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[n][e] = 0.f;
    m_run[0] = m_run[1] = -INFINITY;
    l_run[0] = l_run[1] = 0.f;
  };

  const uint32_t sq = smem_u32(S.q);
  for (int c = 0; c < n_chunks; ++c) {
    const int buf = c & 1;
    if (c + 1 < n_chunks) {
      load_chunk(c + 1, buf ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (!q_loaded) {
#pragma unroll
      for (int kt = 0; kt < KT; ++kt) {
        const int r = warp * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
        const int ch = kt * 2 + (lane >> 4);
        ldmatrix_x4(qa[kt][0], qa[kt][1], qa[kt][2], qa[kt][3], sq + swz<D>(r, ch));
      }
      q_loaded = true;
    }
    int pos0;
    const int br = chunk_branch(c, pos0);
    if (br != cur_br) {
      if (cur_br >= 0) finish_branch(cur_br);
      cur_br = br;
    }
    const int nk = chunk_keys(br, pos0);
    const uint32_t sk = smem_u32(S.kbuf[buf]), sv = smem_u32(S.vbuf[buf]);

    // S = Q K^T for 16 rows x 64 keys
    float s[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[n][e] = 0.f;
#pragma unroll
    for (int kt = 0; kt < KT; ++kt)
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        const int key = np * 16 + (lane >> 4) * 8 + (lane & 7);
        const int ch = kt * 2 + ((lane >> 3) & 1);
        ldmatrix_x4(b0, b1, b2, b3, sk + swz<D>(key, ch));
        const uint32_t bb0[2] = {b0, b1}, bb1[2] = {b2, b3};
        mma_bf16_16816(s[2 * np], qa[kt], bb0);
        mma_bf16_16816(s[2 * np + 1], qa[kt], bb1);
      }
    // scale, mask, online softmax (log2 domain)
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = e >> 1;
        const int key = n * 8 + 2 * cq + (e & 1);
        bool ok = key < nk;
        if (br == 2) {
          const int r = tok_local[i];
          ok = ok && (key >= r - p.window / 2) && (key <= r + p.window / 2 - 1);
        }
        const float x = ok ? s[n][e] * p.scale_log2 : -INFINITY;
        s[n][e] = x;
        mx[i] = fmaxf(mx[i], x);
      }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 1));
      mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 2));
    }
    float alpha[2], mref[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float mn = fmaxf(m_run[i], mx[i]);
      alpha[i] = (mn == -INFINITY) ? 1.f : fast_exp2(m_run[i] - mn);
      m_run[i] = mn;
      mref[i] = (mn == -INFINITY) ? 0.f : mn;
      l_run[i] *= alpha[i];
    }
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[n][e] *= alpha[e >> 1];
    uint32_t pa[4][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      float pv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        pv[e] = fast_exp2(s[n][e] - mref[e >> 1]);
        l_run[e >> 1] += pv[e];
      }
      const int kk = n >> 1, hi = n & 1;
      pa[kk][hi * 2 + 0] = pack_bf16x2(pv[0], pv[1]);
      pa[kk][hi * 2 + 1] = pack_bf16x2(pv[2], pv[3]);
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
      for (int dn = 0; dn < D / 16; ++dn) {
        uint32_t b0, b1, b2, b3;
        const int key = kk * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
        const int ch = dn * 2 + (lane >> 4);
        ldmatrix_x4_trans(b0, b1, b2, b3, sv + swz<D>(key, ch));
        const uint32_t bb0[2] = {b0, b1}, bb1[2] = {b2, b3};
        mma_bf16_16816(o[2 * dn], pa[kk], bb0);
        mma_bf16_16816(o[2 * dn + 1], pa[kk], bb1);
      }
    __syncthreads();  // buffer `buf` is refilled by the next iteration's prefetch
  }
  if (cur_br >= 0) finish_branch(cur_br);

  if (p.out != nullptr) {
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int i = 0; i < 2; ++i)
        if (rvalid[i]) {
          uint32_t* dst = reinterpret_cast<uint32_t*>(
              p.out + ((size_t)(t0 + tok_local[i]) * p.Hq + head[i]) * D + n * 8 + 2 * cq);
          *dst = pack_bf16x2(out_acc[n][2 * i], out_acc[n][2 * i + 1]);
        }
  }
}

template <int D>
static lsrm_status launch_attn_d(const AttnParams& p, int max_block_len, cudaStream_t stream) {
  const size_t smem = sizeof(Smem<D>);
  if (cudaFuncSetAttribute(nsa_attn_mma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return LSRM_ERR_CUDA;
  const int chunks = (max_block_len * p.G + kRowsPerCta - 1) / kRowsPerCta;
  dim3 grid((unsigned)chunks, (unsigned)p.Hkv, (unsigned)p.B);
  nsa_attn_mma_kernel<D><<<grid, kAttnThreads, smem, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? LSRM_OK : LSRM_ERR_CUDA;
}

lsrm_status launch_attn(const lsrm_nsa_desc& d, const int32_t* off, const void* q, const void* k, const void* v,
                        const void* kc, const void* vc, const void* gates, const int32_t* idx, int idx_heads,
                        int route_all, int branches, void* out, float* obranch, float* lse, int lse_stride,
                        int lse_first, uint32_t* status, cudaStream_t stream) {
  if (d.n_forced + d.top_k > kMaxSel) return LSRM_ERR_UNSUPPORTED;
  if (d.n_blocks > 65535) return LSRM_ERR_UNSUPPORTED;
  AttnParams p{};
  p.off = off;
  p.q = (const uint16_t*)q;
  p.k = (const uint16_t*)k;
  p.v = (const uint16_t*)v;
  p.kc = (const uint16_t*)kc;
  p.vc = (const uint16_t*)vc;
  p.gates = (const uint16_t*)gates;
  p.idx = idx;
  p.forced = d.forced_blocks;
  p.out = (uint16_t*)out;
  p.obranch = obranch;
  p.lse = lse;
  p.status = status;
  p.N = d.n_tokens;
  p.B = d.n_blocks;
  p.Hq = d.n_q_heads;
  p.Hkv = d.n_kv_heads;
  p.G = d.n_q_heads / d.n_kv_heads;
  p.top_k = d.top_k;
  p.idx_heads = idx_heads;
  p.n_forced = d.n_forced;
  p.window = d.window;
  p.n_gates = d.n_gates;
  p.route_all = route_all;
  p.branches = branches;
  p.lse_stride = lse_stride;
  p.lse_first = lse_first;
  const float tau = d.scale > 0 ? d.scale : 1.0f / sqrtf((float)d.head_dim);
  p.scale_log2 = tau * 1.4426950408889634f;
  if (d.head_dim == 32) return launch_attn_d<32>(p, d.max_block_len, stream);
  if (d.head_dim == 64) return launch_attn_d<64>(p, d.max_block_len, stream);
  return LSRM_ERR_UNSUPPORTED;
}

}  // namespace lsrm
