// S3-S7 attention on the 5th-generation tensor cores: TMA -> shared memory, tcgen05.mma
// with accumulators in tensor memory, one softmax thread per query row.
//
// Work unit: one CTA = one (query block a, KV group g, pair of 128-row M tiles).  A query
// row is a (token, head) pair of block a whose head reads KV group g; rows are token-major
// so an M tile is 128/G tokens x G heads and its Q rows arrive with one 3D TMA box.
// All rows of the unit share one key stream, so every K/V tile is loaded once per CTA and
// used by both M tiles:
//   compressed branch: the B block means of group g (LSRM page, 方法: compressed block
//     features give global coarse context; Speed3R page 2.1 compression branch);
//   selected branch: the tokens of the routed (and forced) blocks, one 64-row slot per
//     block (LSRM page: selected active blocks give local fine detail);
//   window branch: the query's own block, band r(t)-w/2 .. r(t)+w/2-1 (LSRM page,
//     sequence-parallel paragraph: window attention runs locally inside blocks).
// The gated sum of the branch outputs (LSRM page, gate equations) happens in the epilogue.
//
// Roles (320 threads): warp 0 issues TMA loads; warp 1 owns tensor memory and issues the
// MMAs (S = Q K^T from shared memory, O += P V with P read from tensor memory); warps
// 2-5 and 6-9 are two softmax warpgroups, one per M tile, so one tile's exponentials
// overlap the other tile's MMAs.  Every wait is bounded (see tc::mbar_wait).
//
// Tensor memory per M tile (256 columns): S [kKeys fp32] | P [kKeys/2, bf16 pairs] | O [D].
#include <cuda.h>
#include <cudaTypedefs.h>

#include <climits>
#include <type_traits>

#include "tc_ptx.cuh"
#include "tma_map.cuh"

namespace lsrm {

using namespace tc;

// One pair in kPolyMod of the exponentials goes through poly_exp2 on the FMA pipe instead of
// MUFU (whose 16 ex2 per clock per SM bound the kernel at d = 32); 0 keeps all on MUFU.
#ifndef LSRM_POLY_MOD
#define LSRM_POLY_MOD 0
#endif
constexpr int kPolyMod = LSRM_POLY_MOD;

constexpr int kTcThreads = 320;
constexpr int kTcMaxSel = 256;

template <int D>
struct TcCfg {
  static constexpr int kRows = 128;
  static constexpr int kKeys = 64;                 // keys per chunk = N of S = Q K^T (one block)
  static constexpr int kStages = D == 32 ? 4 : 3;  // K/V ring
  static constexpr int kCand = D == 64 ? 32 : 1;   // streaming top-k candidate buffer per row
  static constexpr int kCtasPerSm = D == 32 ? 2 : 1;
  static constexpr int kTmemCols = D == 32 ? 256 : 512;   // per CTA (power of two)
  static constexpr int kColsPerTile = kTmemCols / 2;
  static constexpr int kRowBytes = D * 2;
  static constexpr uint32_t kLayout = D == 32 ? kLayoutSW64 : kLayoutSW128;
  static constexpr uint32_t kAtomBytes = 8 * kRowBytes;  // 8 rows of one swizzle atom
  static constexpr int kQBytes = kRows * kRowBytes;
  static constexpr int kKVBytes = kKeys * kRowBytes;
  // tensor memory per tile: S (fp32 scores) | P (bf16 pairs) | O
  static constexpr int kColS = 0, kColP = kKeys, kColO = kKeys + kKeys / 2;
  // second score buffer of the bound pass (odd chunks), in columns no other role uses there
  static constexpr int kColS2 = kColsPerTile - kKeys;
  static constexpr uint32_t kIdescQK = idesc_bf16(128, kKeys, false);
  static constexpr uint32_t kIdescPV = idesc_bf16(128, D, true);
  static_assert(kColO + D <= kColsPerTile, "tensor memory budget");
  static_assert(kColS2 >= kKeys, "second score buffer overlaps the first");
};

template <int D>
struct TcSmem {
  using C = TcCfg<D>;
  uint8_t q[2][C::kQBytes];
  uint8_t k[C::kStages][C::kKVBytes];
  uint8_t v[C::kStages][C::kKVBytes];
  float acc[2][D][128];  // gated sum per tile, column-major so a warp's rows are one bank row
  float cand[2][2 * C::kCand][128];  // top-k candidates per row: values, then block ids
  uint64_t q_full[2], kv_full[C::kStages], kv_empty[C::kStages];
  uint64_t s_full[2], p_full[2], pv_done[2], drain;
  uint64_t s_full2[2], p_full2[2];  // bound pass: the odd chunks' score buffer
  uint32_t tmem_base;
  int abort;
  int n_sel;
  int sel_start[kTcMaxSel];
  int sel_n[kTcMaxSel];
};

struct TcParams {
  const int32_t* off;
  const uint16_t* gates;
  const int32_t* idx;
  const int32_t* forced;
  uint16_t* out;
  float* obranch;
  float* lse;
  uint32_t* status;
  int N, B, Hq, Hkv, G, top_k, idx_heads, n_forced, window, n_gates, route_all, branches, lse_stride, lse_first;
  float scale_log2;
  // compressed-branch key count (block means, or gathered forced tokens); n_ckeys_dev overrides it
  int n_ckeys;
  const int* n_ckeys_dev;
  // query blocks of a fixed size instead of `off` (dense passes over pooled queries or all tokens)
  int uniform_block;
  // streaming top-k of the compressed-branch logits (pooled-query routing, d = 64 only):
  // topk_idx [rows][topk_heads][topk_k]; blocks whose bit is set in forced_bits are skipped
  int32_t* topk_idx;
  int topk_k;
  const uint32_t* forced_bits;
  // per-row lower bound on the topk_k-th largest non-forced logit [rows][topk_heads]: the bound
  // pass (bound_pass = 1: scores only, no softmax, no P V) writes it; the top-k pass reads it
  float* topk_thr;
  int bound_pass;
};

enum : int { TC_CMP = 1, TC_SLC = 2, TC_WIN = 4 };

// chunk sequence shared by the three roles: [cmp chunks][slc chunks][win chunk], 64 keys each
struct Chunks {
  int n_cmp, n_slc, n_win, total;
  __device__ __forceinline__ int branch(int c, int& local) const {
    if (c < n_cmp) { local = c; return 0; }
    if (c < n_cmp + n_slc) { local = c - n_cmp; return 1; }
    local = 0;
    return 2;
  }
  __device__ __forceinline__ bool first_of_branch(int c) const {
    return c == 0 || c == n_cmp || c == n_cmp + n_slc;
  }
};

// first key row (block-mean index or token index) and number of valid keys of chunk (br, local)
template <int D>
__device__ __forceinline__ void chunk_keys(const TcSmem<D>& S, const TcParams& p, int br, int local, int t0,
                                           int n_a, int n_ckeys, int& start, int& nvalid) {
  if (br == 0) {
    start = local * 64;
    nvalid = min(64, n_ckeys - start);
  } else if (br == 1) {
    if (p.route_all) {
      start = p.off[local];
      nvalid = p.off[local + 1] - start;
    } else {
      start = S.sel_start[local];
      nvalid = S.sel_n[local];
    }
  } else {
    start = t0;
    nvalid = n_a;
  }
}

// Streaming top-k merge: the n buffered candidates of one row (values at cand[e * 128], block ids
// at cand[(cap + e) * 128]) enter, in order, the row's 32-entry min-heap (values at heap[i * 128],
// ids at heap[(32 + i) * 128]; the root is the worst entry in the order (logit desc, block asc))
// when strictly above the current root.  Returns the new root value.
__device__ __noinline__ float topk_merge(float* heap, const float* cand, int n, int cap, float thr) {
  auto hv = [&](int i) -> float& { return heap[i * 128]; };
  auto hj = [&](int i) -> int& { return reinterpret_cast<int&>(heap[(32 + i) * 128]); };
  auto worse = [](float va, int ja, float vb, int jb) { return va < vb || (va == vb && ja > jb); };
  for (int e = 0; e < n; ++e) {
    const float sv = cand[e * 128];
    const int jg = reinterpret_cast<const int&>(cand[(cap + e) * 128]);
    if (!(sv > thr)) continue;
    int i = 0;
    while (true) {
      const int lc = 2 * i + 1, rc = lc + 1;
      if (lc >= 32) break;
      int cc = lc;
      if (rc < 32 && worse(hv(rc), hj(rc), hv(lc), hj(lc))) cc = rc;
      if (!worse(hv(cc), hj(cc), sv, jg)) break;
      hv(i) = hv(cc);
      hj(i) = hj(cc);
      i = cc;
    }
    hv(i) = sv;
    hj(i) = jg;
    thr = hv(0);
  }
  return thr;
}

template <int D>
__global__ void __launch_bounds__(kTcThreads, TcCfg<D>::kCtasPerSm)
nsa_attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap kcmap,
                   const __grid_constant__ CUtensorMap vcmap, const TcParams p) {
  using C = TcCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  TcSmem<D>& S = *reinterpret_cast<TcSmem<D>*>(smem_raw + (((raw + 1023u) & ~1023u) - raw));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x, g = blockIdx.y, a = blockIdx.z;
  const int t0 = p.uniform_block ? a * p.uniform_block : p.off[a];
  const int n_a = p.uniform_block ? min(p.uniform_block, p.N - t0) : p.off[a + 1] - t0;
  const int rows_total = n_a * p.G;
  const int tile0 = pair * 2;
  if (tile0 * 128 >= rows_total) return;  // the whole CTA leaves before any setup
  const int tokens_per_tile = 128 / p.G;

  if (threadIdx.x == 0) {
    S.abort = 0;
    int n = 0;
    if ((p.branches & TC_SLC) && !p.route_all) {
      const int32_t* r = p.idx + ((size_t)a * p.idx_heads + (p.idx_heads == 1 ? 0 : g)) * p.top_k;
      for (int i = 0; i < p.n_forced + p.top_k && n < kTcMaxSel; ++i) {
        const int j = i < p.n_forced ? p.forced[i] : r[i - p.n_forced];
        if (j < 0 || j >= p.B) { raise_status(p.status, LSRM_ERR_BOUNDS); continue; }
        S.sel_start[n] = p.off[j];
        S.sel_n[n] = p.off[j + 1] - p.off[j];
        ++n;
      }
    }
    S.n_sel = n;
    for (int t = 0; t < 2; ++t) {
      mbar_init(&S.q_full[t], 1);
      mbar_init(&S.s_full[t], 1);
      mbar_init(&S.p_full[t], 128);
      mbar_init(&S.pv_done[t], 1);
      mbar_init(&S.s_full2[t], 1);
      mbar_init(&S.p_full2[t], 128);
    }
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&S.kv_full[s], 1);
      mbar_init(&S.kv_empty[s], 1);
    }
    mbar_init(&S.drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  Chunks cs;
  const int n_ckeys = p.n_ckeys_dev != nullptr ? *p.n_ckeys_dev : p.n_ckeys;
  cs.n_cmp = (p.branches & TC_CMP) ? (n_ckeys + C::kKeys - 1) / C::kKeys : 0;
  cs.n_slc = (p.branches & TC_SLC) ? (p.route_all ? p.B : S.n_sel) : 0;
  cs.n_win = ((p.branches & TC_WIN) && p.window > 0) ? 1 : 0;
  cs.total = cs.n_cmp + cs.n_slc + cs.n_win;
  volatile int* abort = &S.abort;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0 && cs.total > 0) {
      tma_prefetch_desc(&qmap);
      for (int t = 0; t < 2; ++t) {
        mbar_arrive_expect_tx(&S.q_full[t], C::kQBytes);
        tma_load_3d(S.q[t], &qmap, &S.q_full[t], 0, g * p.G, t0 + (tile0 + t) * tokens_per_tile);
      }
      int issued = 0;
      for (int c = 0; c < cs.total; ++c) {
        const int st = c % C::kStages;
        if (c >= C::kStages && !mbar_wait(&S.kv_empty[st], ((c / C::kStages) + 1) & 1, abort, p.status)) break;
        int local, start, nvalid;
        const int br = cs.branch(c, local);
        chunk_keys<D>(S, p, br, local, t0, n_a, n_ckeys, start, nvalid);
        mbar_arrive_expect_tx(&S.kv_full[st], p.bound_pass ? C::kKVBytes : 2 * C::kKVBytes);
        tma_load_3d(S.k[st], br == 0 ? &kcmap : &kmap, &S.kv_full[st], 0, g, start);
        if (!p.bound_pass) tma_load_3d(S.v[st], br == 0 ? &vcmap : &vmap, &S.kv_full[st], 0, g, start);
        issued = c + 1;
      }
      if (*abort) {
        // let the copies already issued land before the CTA's shared memory goes away
        for (int c = max(0, issued - C::kStages); c < issued; ++c) {
          volatile int no_abort = 0;
          mbar_wait(&S.kv_full[c % C::kStages], (c / C::kStages) & 1, &no_abort, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0 && cs.total > 0) {
      bool ok = mbar_wait(&S.q_full[0], 0, abort, p.status) && mbar_wait(&S.q_full[1], 0, abort, p.status);
      tc_fence_after();
      const uint32_t qaddr[2] = {smem_u32(S.q[0]), smem_u32(S.q[1])};
      // shared-memory descriptors are computed once; a byte offset moves the start-address
      // field (address / 16, bits 0..13; shared addresses stay below 2^18) by offset / 16
      const uint64_t qdesc[2] = {smem_desc(qaddr[0], 16, C::kAtomBytes, C::kLayout),
                                 smem_desc(qaddr[1], 16, C::kAtomBytes, C::kLayout)};
      const uint64_t kdesc = smem_desc(smem_u32(S.k[0]), 16, C::kAtomBytes, C::kLayout);
      const uint64_t vdesc = smem_desc(smem_u32(S.v[0]), C::kKVBytes, C::kAtomBytes, C::kLayout);
      constexpr uint32_t kStageStep = C::kKVBytes >> 4;
      auto issue_qk = [&](int t, int c, int col) {
        const uint32_t d = tmem + t * C::kColsPerTile + col;
        const uint64_t bd = kdesc + (uint64_t)((c % C::kStages) * kStageStep);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) mma_ss(d, qdesc[t] + 2 * k, bd + 2 * k, C::kIdescQK, k > 0 ? 1u : 0u);
      };
      auto issue_pv = [&](int t, int c) {
        const uint32_t d = tmem + t * C::kColsPerTile + C::kColO;
        const uint64_t bd = vdesc + (uint64_t)((c % C::kStages) * kStageStep);
        const bool first = cs.first_of_branch(c);
#pragma unroll
        for (int kk = 0; kk < C::kKeys / 16; ++kk)
          mma_ts(d, tmem + t * C::kColsPerTile + C::kColP + kk * 8, bd + kk * (16 * C::kRowBytes >> 4), C::kIdescPV,
                 (first && kk == 0) ? 0u : 1u);
      };
      // bound pass: scores only, double-buffered (even chunks in S, odd chunks in S2) so that the
      // next chunk's MMAs run while the softmax warps reduce the current one; each buffer has its
      // own full/free barrier pair, completed once per two chunks
      for (int c = 0; ok && p.bound_pass && c < cs.total; ++c) {
        if (!mbar_wait(&S.kv_full[c % C::kStages], (c / C::kStages) & 1, abort, p.status)) { ok = false; break; }
        tc_fence_after();
        const int b = c & 1;
        for (int t = 0; t < 2; ++t) {
          if (c >= 2) {
            if (!mbar_wait(b ? &S.p_full2[t] : &S.p_full[t], ((c >> 1) - 1) & 1, abort, p.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          issue_qk(t, c, b ? C::kColS2 : C::kColS);
          mma_commit(b ? &S.s_full2[t] : &S.s_full[t]);
        }
        if (!ok) break;
        mma_commit(&S.kv_empty[c % C::kStages]);
      }
      for (int c = 0; ok && !p.bound_pass && c < cs.total; ++c) {
        if (!mbar_wait(&S.kv_full[c % C::kStages], (c / C::kStages) & 1, abort, p.status)) { ok = false; break; }
        tc_fence_after();
        for (int t = 0; t < 2; ++t) {
          // S(c) is issued ahead of P(c - 1) V: it overwrites only S, which the softmax released
          // with P(c - 1), and the softmax waits for P(c - 1) V before it stores P(c)
          if (c > 0) {
            if (!mbar_wait(&S.p_full[t], (c - 1) & 1, abort, p.status)) { ok = false; break; }
            tc_fence_after();
          }
          issue_qk(t, c, C::kColS);
          mma_commit(&S.s_full[t]);
          if (c > 0) {
            issue_pv(t, c - 1);
            mma_commit(&S.pv_done[t]);
          }
        }
        if (!ok) break;
        if (c > 0) mma_commit(&S.kv_empty[(c - 1) % C::kStages]);
      }
      for (int t = 0; ok && !p.bound_pass && t < 2; ++t) {
        if (!mbar_wait(&S.p_full[t], (cs.total - 1) & 1, abort, p.status)) { ok = false; break; }
        tc_fence_after();
        issue_pv(t, cs.total - 1);
        mma_commit(&S.pv_done[t]);
      }
      // every MMA issued so far must finish (and every arrive it owes must land) before the
      // CTA can release tensor and shared memory, on the normal path and after an abort alike
      mma_commit(&S.drain);
      volatile int no_abort = 0;
      mbar_wait(&S.drain, 0, &no_abort, nullptr);
    }
  } else {
    // ---------------- softmax warpgroups ----------------
    const int t = (warp - 2) >> 2;               // M tile of this warpgroup
    const int quarter = warp & 3;                // tensor-memory lane quarter this warp may access
    const int row = quarter * 32 + lane;         // row of the M tile = TMEM lane
    const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + t * C::kColsPerTile;
    const int R = (tile0 + t) * 128 + row;
    const bool valid = R < rows_total;
    const int tok_local = R / p.G;
    const int tok = t0 + (valid ? tok_local : 0);
    const int head = g * p.G + R % p.G;
    const size_t orow = (size_t)tok * p.Hq + head;
    float* acc = &S.acc[t][0][row];  // acc[i * 128] = output column i of this row
#pragma unroll
    for (int i = 0; i < D; ++i) acc[i * 128] = 0.f;
    float m = -INFINITY;  // reference of the current branch, log2 units
    float l = 0.f;        // row sum of P for the current branch

    auto finalize = [&](int br, float mb, float lb) {
      const float inv = lb > 0.f ? 1.f / lb : 0.f;
      const float gi = (p.out != nullptr && valid) ? bf16_to_f32(p.gates[orow * p.n_gates + br]) * inv : 0.f;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        uint32_t o[32];
        tmem_ld32(tbase + C::kColO + 32 * i, o);
        tmem_ld_wait();
        if (p.out != nullptr) {
#pragma unroll
          for (int e = 0; e < 32; ++e) acc[(32 * i + e) * 128] = fmaf(gi, __uint_as_float(o[e]), acc[(32 * i + e) * 128]);
        }
        if (p.obranch != nullptr && valid) {
          float4* dst = reinterpret_cast<float4*>(p.obranch + orow * D + 32 * i);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(o[4 * e]) * inv, __uint_as_float(o[4 * e + 1]) * inv,
                                 __uint_as_float(o[4 * e + 2]) * inv, __uint_as_float(o[4 * e + 3]) * inv);
        }
      }
      if (p.lse != nullptr && valid) {
        int slot = p.lse_first;
        if (p.branches & TC_CMP) slot += (br > 0);
        if ((p.branches & TC_SLC) && br > 1) slot += 1;
        p.lse[orow * p.lse_stride + slot] = lb > 0.f ? (mb + __log2f(lb)) * 0.6931471805599453f : -INFINITY;
      }
    };

    // waits are made warp-uniform: the tensor-memory accesses after them are .sync.aligned
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      const bool w = mbar_wait(bar, parity, abort, p.status);
      return __all_sync(0xffffffffu, w);
    };
    const int wlo = tok_local - p.window / 2, whi = tok_local + p.window / 2 - 1;
    const float sc = p.scale_log2;
    int br = 0, nv = 0;
    // raw score of key j of the chunk, or -inf where masked (short block or outside the window band)
    auto masked = [&](uint32_t raw, int j) -> float {
      bool kv = j < nv;
      if (br == 2) kv = kv && j >= wlo && j <= whi;
      return kv ? __uint_as_float(raw) : -INFINITY;
    };
    // ---- streaming top-k of the compressed-branch logits (pooled-query routing) ----
    // A 32-entry min-heap per row, kept in this row's column of the (otherwise unused) output
    // accumulator: values in acc[0..31], block ids in acc[32..63].  The root is the worst entry
    // in the order (logit desc, block asc), so ties evict the larger block id first; keys arrive
    // in increasing block order, so a candidate enters only when strictly above the root.
    // Scores above the (possibly stale) root are first appended to a per-row candidate buffer;
    // the warp merges its rows' buffers together, re-testing every candidate in key order
    // against the live root, which makes the same decisions as inserting key by key while
    // keeping the divergent heap work out of the per-key loop.  Forced blocks never enter the
    // buffer (a 64-bit mask per chunk from the forced-block bitmap).  The merge is one function
    // outside the unrolled per-key code, which would otherwise carry a copy at every call site.
    const bool topk_on = (D == 64) && p.topk_idx != nullptr;
    float thr = -INFINITY;
    int key_base = 0;  // block id of key 0 of the current chunk
    uint64_t fmask = 0;  // forced blocks among the chunk's 64 keys (never candidates)
    int ncand = 0;     // this row's buffered candidates
    float* cbuf = &S.cand[t][0][row];
    auto hv = [&](int i) -> float& { return acc[i * 128]; };
    auto hj = [&](int i) -> int& { return reinterpret_cast<int&>(acc[(32 + i) * 128]); };
    auto worse = [&](float va, int ja, float vb, int jb) { return va < vb || (va == vb && ja > jb); };
    auto topk_append = [&](float sv, int j) {
      if (sv > thr && !((fmask >> j) & 1ull)) {
        cbuf[ncand * 128] = sv;
        reinterpret_cast<int&>(cbuf[(C::kCand + ncand) * 128]) = key_base + j;
        ++ncand;
      }
    };
    auto topk_flush = [&]() {
      thr = topk_merge(acc, cbuf, ncand, C::kCand, thr);
      ncand = 0;
    };
    if (topk_on) {
      // With a lower bound b on the k-th largest non-forced logit, the heap starts full of
      // placeholders just below b: every key at or above b gets in, no key below b can be among
      // the k best (k keys at or above b exist), and the placeholders are all displaced.
      if (p.topk_thr != nullptr && valid) {
        const float b = p.topk_thr[(size_t)(t0 + R) * p.Hkv + g];
        if (b > -INFINITY) thr = nextafterf(b, -INFINITY);
      }
#pragma unroll 1
      for (int i = 0; i < 32; ++i) {
        hv(i) = thr;
        hj(i) = INT_MAX;
      }
    }

    // max of the chunk's raw scores (the scale is positive, so it commutes with the max)
    auto chunk_max_t = [&](auto need_mask_tag) -> float {
      constexpr bool need_mask = decltype(need_mask_tag)::value;
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t r[32];
        tmem_ld32(tbase + C::kColS + 32 * h, r);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float s0 = need_mask ? masked(r[i], 32 * h + i) : __uint_as_float(r[i]);
          const float s1 = need_mask ? masked(r[i + 1], 32 * h + i + 1) : __uint_as_float(r[i + 1]);
          mx[(i >> 1) & 3] = fmax3(mx[(i >> 1) & 3], s0, s1);
        }
      }
      return fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
    };
    // The previous chunk's P V is waited for as late as possible: before the first P store of a
    // chunk, before O is read, and at the latest before P(c) is handed over.
    int pv_wait_for = -1;
    bool pv_ok = true;
    auto wait_pv = [&]() {
      if (pv_wait_for >= 0) {
        pv_ok = wait_all(&S.pv_done[t], pv_wait_for & 1);
        tc_fence_after();
        pv_wait_for = -1;
      }
    };
    // P = exp2(s * scale - mref) as bf16 pairs into tensor memory; returns the chunk's raw max and
    // its sum of P in *lsum.  S is read 16 columns at a time, each load issued before the previous
    // quarter is processed so the tensor-memory latency overlaps the exponentials.
    auto exp_pass_t = [&](float mref, float* lsum, auto need_mask_tag, auto topk_tag) -> float {
      constexpr bool need_mask = decltype(need_mask_tag)::value;
      constexpr bool topk = decltype(topk_tag)::value && D == 64;
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
      const float nm = -mref;
      uint32_t ra[16], rb[16];
      auto quarter = [&](const uint32_t* r, int qd) {
        uint32_t pk[8];
        float qmx = -INFINITY;  // the quarter's max (top-k gate)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int j = 16 * qd + 2 * i;
          const float s0 = need_mask ? masked(r[2 * i], j) : __uint_as_float(r[2 * i]);
          const float s1 = need_mask ? masked(r[2 * i + 1], j + 1) : __uint_as_float(r[2 * i + 1]);
          mx[i & 3] = fmax3(mx[i & 3], s0, s1);
          if constexpr (topk) qmx = fmax3(qmx, s0, s1);
          const float x0 = fmaf(s0, sc, nm), x1 = fmaf(s1, sc, nm);
          float p0, p1;
          if (kPolyMod > 0 && (8 * qd + i) % (kPolyMod > 0 ? kPolyMod : 1) == kPolyMod - 1) {
            p0 = poly_exp2(x0);
            p1 = poly_exp2(x1);
          } else {
            p0 = fast_exp2(x0);
            p1 = fast_exp2(x1);
          }
          ls[i & 3] += p0 + p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
        if (qd == 0) wait_pv();
        if (pv_ok) tmem_st8(tbase + C::kColP + 8 * qd, pk);
        if constexpr (topk) {
          // only quarters where some row of the warp has a score above its root visit the keys
          if (__any_sync(0xffffffffu, qmx > thr)) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int j = 16 * qd + i;
              topk_append(need_mask ? masked(r[i], j) : __uint_as_float(r[i]), j);
            }
            // a quarter appends at most 16 candidates per row
            if (__any_sync(0xffffffffu, ncand > C::kCand - 16)) topk_flush();
          }
        }
      };
      tmem_ld16(tbase + C::kColS, ra);
      tmem_ld_wait();
#pragma unroll
      for (int qd = 0; qd < C::kKeys / 16; ++qd) {
        uint32_t* cur = (qd & 1) ? rb : ra;
        uint32_t* nxt = (qd & 1) ? ra : rb;
        if (qd + 1 < C::kKeys / 16) tmem_ld16(tbase + C::kColS + 16 * (qd + 1), nxt);
        quarter(cur, qd);
        if (qd + 1 < C::kKeys / 16) tmem_ld_wait();
      }
      *lsum = (ls[0] + ls[1]) + (ls[2] + ls[3]);
      return fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
    };
    // masking is decided once per chunk: two straight-line instantiations, no per-key branch
    auto chunk_max = [&](bool need_mask) -> float {
      return need_mask ? chunk_max_t(std::true_type{}) : chunk_max_t(std::false_type{});
    };
    auto exp_pass = [&](bool need_mask, float mref, float* lsum, bool offer = true) -> float {
      if (topk_on && br == 0 && offer)
        return need_mask ? exp_pass_t(mref, lsum, std::true_type{}, std::true_type{})
                         : exp_pass_t(mref, lsum, std::false_type{}, std::true_type{});
      return need_mask ? exp_pass_t(mref, lsum, std::true_type{}, std::false_type{})
                       : exp_pass_t(mref, lsum, std::false_type{}, std::false_type{});
    };

    if (p.bound_pass) {
      // ---- bound pass: per row, the max non-forced logit of each of 64 key groups (chunk c
      // joins group c mod 64), then the topk_k-th largest group max.  Groups are disjoint, so
      // at least topk_k distinct keys score at or above that value: a lower bound on the
      // topk_k-th largest logit that needs no selection in the per-key loop.
      float* gmax = acc;  // gmax[i * 128], i < 64 (the output accumulator is unused here)
#pragma unroll 1
      for (int i = 0; i < 64; ++i) gmax[i * 128] = -INFINITY;
      auto bound_max_t = [&](uint32_t col, auto mask_tag) -> float {
        constexpr bool need_mask = decltype(mask_tag)::value;
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t r[32];
          tmem_ld32(tbase + col + 32 * h, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            float s0 = __uint_as_float(r[i]), s1 = __uint_as_float(r[i + 1]);
            if (need_mask) {
              const int j = 32 * h + i;
              if (j >= nv || ((fmask >> j) & 1ull)) s0 = -INFINITY;
              if (j + 1 >= nv || ((fmask >> (j + 1)) & 1ull)) s1 = -INFINITY;
            }
            mx[(i >> 1) & 3] = fmax3(mx[(i >> 1) & 3], s0, s1);
          }
        }
        return fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
      };
      bool okb = true;
      for (int c = 0; c < cs.total; ++c) {
        const int b = c & 1;
        if (!wait_all(b ? &S.s_full2[t] : &S.s_full[t], (c >> 1) & 1)) { okb = false; break; }
        tc_fence_after();
        nv = min(64, n_ckeys - c * 64);
        const uint32_t w0 = p.forced_bits[c * 2], w1 = p.forced_bits[c * 2 + 1];
        fmask = (uint64_t)w0 | ((uint64_t)w1 << 32);
        const uint32_t col = b ? C::kColS2 : C::kColS;
        const float mx = (nv < 64 || fmask != 0) ? bound_max_t(col, std::true_type{})
                                                 : bound_max_t(col, std::false_type{});
        tc_fence_before();
        mbar_arrive(b ? &S.p_full2[t] : &S.p_full[t]);
        float& gv = gmax[(c & 63) * 128];
        gv = fmaxf(gv, mx);
      }
      if (okb && valid) {
        // the k-th largest of the 64 group maxima: the smallest value with fewer than k above it
        float v[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) v[i] = gmax[i * 128];
        float bound = INFINITY;
#pragma unroll 1
        for (int i = 0; i < 64; ++i) {
          const float vi = gmax[i * 128];
          int above = 0;
#pragma unroll
          for (int j = 0; j < 64; ++j) above += v[j] > vi ? 1 : 0;
          if (above < p.topk_k) bound = fminf(bound, vi);
        }
        p.topk_thr[(size_t)(t0 + R) * p.Hkv + g] = bound;
      }
    }

    int prev_br = -1;
    bool ok = !p.bound_pass;
    for (int c = 0; ok && c < cs.total; ++c) {
      if (!wait_all(&S.s_full[t], c & 1)) { ok = false; break; }
      tc_fence_after();
      pv_wait_for = c - 1;  // P(c - 1) V must be done before P is overwritten and O is read
      int local, start;
      br = cs.branch(c, local);
      const bool first = cs.first_of_branch(c);
      chunk_keys<D>(S, p, br, local, t0, n_a, n_ckeys, start, nv);
      const bool need_mask = br == 2 || nv < 64;
      if (topk_on && br == 0) {
        key_base = local * 64;
        const uint32_t w0 = p.forced_bits[key_base >> 5], w1 = p.forced_bits[(key_base >> 5) + 1];
        fmask = (uint64_t)w0 | ((uint64_t)w1 << 32);
      }
      float lsum;
      if (first) {
        wait_pv();
        if (!pv_ok) { ok = false; break; }
        if (c > 0) finalize(prev_br, m, l);
        const float mraw = chunk_max(need_mask);
        m = mraw == -INFINITY ? -INFINITY : mraw * sc;
        exp_pass(need_mask, m == -INFINITY ? 0.f : m, &lsum);
        l = lsum;
      } else {
        const float mraw = exp_pass(need_mask, m == -INFINITY ? 0.f : m, &lsum);
        if (!pv_ok) { ok = false; break; }
        // move the reference only when the row max would exceed it by more than 2^8
        const float cand = mraw == -INFINITY ? -INFINITY : mraw * sc;
        const bool grow = cand > m + 8.f;
        if (__any_sync(0xffffffffu, grow)) {
          const float mn = grow ? cand : m;
          const float alpha = grow ? (m == -INFINITY ? 0.f : fast_exp2(m - mn)) : 1.f;
#pragma unroll
          for (int i = 0; i < D / 32; ++i) {
            uint32_t o[32];
            tmem_ld32(tbase + C::kColO + 32 * i, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(tbase + C::kColO + 32 * i, o);
          }
          l *= alpha;
          m = mn;
          exp_pass(need_mask, m == -INFINITY ? 0.f : m, &lsum, false);  // candidates were taken
        }
        l += lsum;
      }
      wait_pv();  // chunks whose exponentials stored nothing still keep the phase order
      if (!pv_ok) { ok = false; break; }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&S.p_full[t]);
      prev_br = br;
    }
    if (cs.total == 0 && valid && !p.bound_pass) {  // no keys at all (e.g. an empty forced set): defined outputs
      if (p.obranch != nullptr)
        for (int i = 0; i < D; ++i) p.obranch[orow * D + i] = 0.f;
      if (p.lse != nullptr) p.lse[orow * p.lse_stride + p.lse_first] = -INFINITY;
    }
    if (ok && topk_on) topk_flush();
    if (ok && topk_on && valid) {
      // emit the row's top-k in order (logit desc, block asc); missing entries are -1
      int32_t* dst = p.topk_idx + ((size_t)(t0 + R) * p.Hkv + g) * p.topk_k;
      uint32_t taken = 0;
#pragma unroll 1
      for (int k = 0; k < p.topk_k; ++k) {
        int best = -1;
#pragma unroll 1
        for (int i = 0; i < 32; ++i) {
          if ((taken >> i) & 1u) continue;
          if (best < 0 || worse(hv(best), hj(best), hv(i), hj(i))) best = i;
        }
        taken |= 1u << best;
        dst[k] = hj(best) == INT_MAX ? -1 : hj(best);
      }
    }
    if (ok && cs.total > 0 && wait_all(&S.pv_done[t], (cs.total - 1) & 1)) {
      tc_fence_after();
      finalize(prev_br, m, l);
      if (p.out != nullptr && valid) {
        uint4* dst = reinterpret_cast<uint4*>(p.out + orow * D);
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
          uint4 u;
          u.x = pack_bf16x2(acc[(8 * i + 0) * 128], acc[(8 * i + 1) * 128]);
          u.y = pack_bf16x2(acc[(8 * i + 2) * 128], acc[(8 * i + 3) * 128]);
          u.z = pack_bf16x2(acc[(8 * i + 4) * 128], acc[(8 * i + 5) * 128]);
          u.w = pack_bf16x2(acc[(8 * i + 6) * 128], acc[(8 * i + 7) * 128]);
          dst[i] = u;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ---- host side ------------------------------------------------------------------------------------
namespace {

template <int D>
lsrm_status launch_tc_d(const lsrm_nsa_desc& d, const TcParams& p, const void* q, const void* k, const void* v,
                        const void* kc, const void* vc, long long kc_rows, cudaStream_t stream) {
  CUtensorMap qm, km, vm, kcm, vcm;
  const void* kk = k ? k : kc;
  const void* vv = v ? v : vc;
  const void* kkc = kc ? kc : k;
  const void* vvc = vc ? vc : v;
  if (!make_map(&qm, q, D, d.n_q_heads, d.n_tokens, p.G, 128 / p.G)) return LSRM_ERR_CUDA;
  if (!make_map(&km, kk, D, d.n_kv_heads, k ? d.n_tokens : kc_rows, 1, 64)) return LSRM_ERR_CUDA;
  if (!make_map(&vm, vv, D, d.n_kv_heads, v ? d.n_tokens : kc_rows, 1, 64)) return LSRM_ERR_CUDA;
  if (!make_map(&kcm, kkc, D, d.n_kv_heads, kc ? kc_rows : d.n_tokens, 1, 64)) return LSRM_ERR_CUDA;
  if (!make_map(&vcm, vvc, D, d.n_kv_heads, vc ? kc_rows : d.n_tokens, 1, 64)) return LSRM_ERR_CUDA;
  const size_t smem = sizeof(TcSmem<D>) + 1024;
  if (cudaFuncSetAttribute(nsa_attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return LSRM_ERR_CUDA;
  const int tiles = (d.max_block_len * p.G + 127) / 128;
  dim3 grid((unsigned)((tiles + 1) / 2), (unsigned)d.n_kv_heads, (unsigned)d.n_blocks);
  nsa_attn_tc_kernel<D><<<grid, kTcThreads, smem, stream>>>(qm, km, vm, kcm, vcm, p);
  return cudaGetLastError() == cudaSuccess ? LSRM_OK : LSRM_ERR_CUDA;
}

}  // namespace

lsrm_status launch_attn(const lsrm_nsa_desc& d, const int32_t* off, const void* q, const void* k, const void* v,
                           const void* kc, const void* vc, const void* gates, const int32_t* idx, int idx_heads,
                           int route_all, int branches, void* out, float* obranch, float* lse, int lse_stride,
                           int lse_first, uint32_t* status, cudaStream_t stream) {
  const int G = d.n_q_heads / d.n_kv_heads;
  if (128 % G != 0) return LSRM_ERR_UNSUPPORTED;
  if ((!route_all && d.n_forced + d.top_k > kTcMaxSel) || d.n_blocks > 65535) return LSRM_ERR_UNSUPPORTED;
  TcParams p{};
  p.off = off;
  p.gates = (const uint16_t*)gates;
  p.idx = idx;
  p.forced = d.forced_blocks;
  p.out = (uint16_t*)out;
  p.obranch = obranch;
  p.lse = lse;
  p.status = status;
  p.N = (int)d.n_tokens;
  p.B = d.n_blocks;
  p.Hq = d.n_q_heads;
  p.Hkv = d.n_kv_heads;
  p.G = G;
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
  p.n_ckeys = d.n_blocks;
  if (d.head_dim == 32) return launch_tc_d<32>(d, p, q, k, v, kc, vc, d.n_blocks, stream);
  if (d.head_dim == 64) return launch_tc_d<64>(d, p, q, k, v, kc, vc, d.n_blocks, stream);
  return LSRM_ERR_UNSUPPORTED;
}

// Dense multi-head attention of n_q query rows (q [n_q][H][D]) against n_ckeys rows of
// (kc, vc) ([kc_rows][H][D]), in fixed groups of 256 query rows: the pooled-query compressed
// branch (optionally with the streaming top-k that routes it) and the forced-block part of the
// pooled-query selected branch.  Writes fp32 obranch [n_q][H][D] and the natural-log lse [n_q][H].
// With topk_thr ([n_q][H] fp32 scratch) the top-k pass is preceded by the bound pass, whose
// per-row lower bound on the k-th logit lets the top-k pass skip almost every candidate.
lsrm_status launch_attn_dense(int D, long long n_q, int H, const void* q, const void* kc, const void* vc,
                              long long kc_rows, int n_ckeys, const int* n_ckeys_dev, float tau, float* obranch,
                              float* lse, int32_t* topk_idx, int topk_k, const uint32_t* forced_bits,
                              float* topk_thr, uint32_t* status, cudaStream_t stream) {
  if (topk_idx != nullptr && (D != 64 || topk_k < 1 || topk_k > 32 || forced_bits == nullptr))
    return LSRM_ERR_UNSUPPORTED;
  if ((n_q + 255) / 256 > 65535 || n_q > INT32_MAX) return LSRM_ERR_UNSUPPORTED;
  lsrm_nsa_desc d{};
  d.n_tokens = n_q;
  d.n_blocks = (int32_t)((n_q + 255) / 256);  // query groups (grid z)
  d.max_block_len = 256;
  d.n_q_heads = H;
  d.n_kv_heads = H;
  d.head_dim = D;
  TcParams p{};
  p.status = status;
  p.obranch = obranch;
  p.lse = lse;
  p.N = (int)n_q;
  p.B = n_ckeys;
  p.Hq = H;
  p.Hkv = H;
  p.G = 1;
  p.n_gates = 1;
  p.branches = TC_CMP;
  p.lse_stride = 1;
  p.scale_log2 = tau * 1.4426950408889634f;
  p.n_ckeys = n_ckeys;
  p.n_ckeys_dev = n_ckeys_dev;
  p.uniform_block = 256;
  p.topk_idx = topk_idx;
  p.topk_k = topk_k;
  p.forced_bits = forced_bits;
  if (D == 32) return launch_tc_d<32>(d, p, q, nullptr, nullptr, kc, vc, kc_rows, stream);
  if (D != 64) return LSRM_ERR_UNSUPPORTED;
  if (topk_idx != nullptr && topk_thr != nullptr) {
    TcParams pb = p;
    pb.obranch = nullptr;
    pb.lse = nullptr;
    pb.topk_idx = nullptr;
    pb.topk_thr = topk_thr;
    pb.bound_pass = 1;
    const lsrm_status st = launch_tc_d<64>(d, pb, q, nullptr, nullptr, kc, vc, kc_rows, stream);
    if (st != LSRM_OK) return st;
    p.topk_thr = topk_thr;
  }
  return launch_tc_d<64>(d, p, q, nullptr, nullptr, kc, vc, kc_rows, stream);
}

}  // namespace lsrm
