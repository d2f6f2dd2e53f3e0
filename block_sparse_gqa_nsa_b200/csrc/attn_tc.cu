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
// Tensor memory per M tile (kColsPerTile: 128 columns at d = 32, 256 at d = 64):
// S [kKeys fp32] | P [kKeys/2, bf16 pairs] | O [D].
//
// The same kernel runs the dense passes of the pooled-query (Speed3R) variant at d = 64: the
// compressed branch over all block means with a streaming top-k of its logits (candidates above a
// per-row lower bound on the k-th logit, ranked at the end), the bound pass that computes that
// bound (scores only), and the pass of every token against the gathered forced tokens.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <climits>
#include <type_traits>

#include "tc_ptx.cuh"
#include "tma_map.cuh"

namespace lsrm {

using namespace tc;

// One pair in kPolyMod of the exponentials goes through poly_exp2_pair on the FMA pipe instead of
// MUFU (whose 16 ex2 per clock per SM bound the kernel at d = 32); 0 keeps all on MUFU.  With the
// packed f32x2 softmax arithmetic leaving issue slots free, 1 pair in 6 measured fastest on the
// sparse stage (1 in 5 / 6 / 8 / 10: 3.775 / 3.773 / 3.80 / 3.83 ms; MUFU alone 3.95 ms).
#ifndef LSRM_POLY_MOD
#define LSRM_POLY_MOD 6
#endif
constexpr int kPolyMod = LSRM_POLY_MOD;

constexpr int kTcThreads = 320;
constexpr int kTcMaxSel = 256;

template <int D>
struct TcCfg {
  static constexpr int kRows = 128;
  static constexpr int kKeys = 64;                 // keys per chunk = N of S = Q K^T (one block)
  static constexpr int kStages = D == 32 ? 4 : 3;  // K/V ring
  // streaming top-k candidates per row: logits in the (then unused) output accumulator, block ids
  // in the candidate array
  static constexpr int kCand = D == 64 ? 64 : 1;
  // bound pass: chunks of kBoundKeys keys (one N = 256 MMA per K step), one score buffer per
  // tile (the two tiles alternate), and a ring of 32 KB K slots laid over the K/V stages and the
  // candidate-id array (256 keys measured 6% faster than 128 keys in two buffers per tile)
  static constexpr int kBoundKeys = 256;
  static constexpr int kBoundBufs = 1;
  static constexpr int kBoundStages = 3;
  static constexpr uint32_t kIdescBound = idesc_bf16(128, kBoundKeys, false);
  static constexpr int kCtasPerSm = D == 32 ? 2 : 1;
  static constexpr int kTmemCols = D == 32 ? 256 : 512;   // per CTA (power of two)
  static constexpr int kColsPerTile = kTmemCols / 2;
  static constexpr int kRowBytes = D * 2;
  static constexpr int kBoundSlotBytes = kBoundKeys * kRowBytes;
  static constexpr int kBoundKvSlots = (2 * kStages * kKeys * kRowBytes) / kBoundSlotBytes;
  static constexpr uint32_t kLayout = D == 32 ? kLayoutSW64 : kLayoutSW128;
  static constexpr uint32_t kAtomBytes = 8 * kRowBytes;  // 8 rows of one swizzle atom
  static constexpr int kQBytes = kRows * kRowBytes;
  static constexpr int kKVBytes = kKeys * kRowBytes;
  // tensor memory per tile: S (fp32 scores) | P (bf16 pairs) | O
  static constexpr int kColS = 0, kColP = kKeys, kColO = kKeys + kKeys / 2;

  static constexpr uint32_t kIdescQK = idesc_bf16(128, kKeys, false);
  static constexpr uint32_t kIdescPV = idesc_bf16(128, D, true);
  static_assert(kColO + D <= kColsPerTile, "tensor memory budget");
  static_assert(kCand <= D, "candidate logits live in the output accumulator");
  static_assert(kCand <= 64, "candidate ranks are counted in registers");
  static_assert(D != 64 || kBoundBufs * kBoundKeys <= kColsPerTile, "bound-pass score buffers");
  static_assert(D != 64 || kBoundKvSlots >= 1, "bound-pass K slots over K/V");
};

template <int D>
struct TcSmem {
  using C = TcCfg<D>;
  uint8_t q[2][C::kQBytes];
  uint8_t k[C::kStages][C::kKVBytes];
  uint8_t v[C::kStages][C::kKVBytes];
  float acc[2][D][128];  // gated sum per tile, column-major so a warp's rows are one bank row
  int cand_id[2][C::kCand][128];  // top-k candidate block ids per row (logits in acc)
  uint64_t q_full[2], kv_full[C::kStages], kv_empty[C::kStages];
  uint64_t s_full[2], p_full[2], pv_done[2], drain;
  // bound pass: K ring, and per tile and score buffer a full (MMA) / free (softmax) pair
  uint64_t kb_full[C::kBoundStages], kb_empty[C::kBoundStages];
  uint64_t bs_full[2][C::kBoundBufs], bs_free[2][C::kBoundBufs];
  uint32_t tmem_base;
  int abort;
  int n_sel;
  int win_lo, win_hi;  // window band of the CTA's tokens, relative to the block start
  // key rows of the compressed slot start at c_lo; with the self/cross mixture the compressed slot
  // is the token range [c_lo, c_hi) and the selected slot the token range [s_lo, s_hi)
  int c_lo, c_hi, s_lo, s_hi;
  int sel_start[kTcMaxSel];
  int sel_n[kTcMaxSel];
};
static_assert(sizeof(TcSmem<64>) + 1024 <= 227 * 1024, "shared memory per CTA (d = 64)");
static_assert(sizeof(TcSmem<64>::cand_id) >=
                  (TcCfg<64>::kBoundStages - TcCfg<64>::kBoundKvSlots) * TcCfg<64>::kBoundSlotBytes,
              "bound-pass K slots over the candidate ids");
// bound-pass K slot s: the first kBoundKvSlots over the K/V stages (contiguous), the rest over the
// candidate ids
template <int D>
__device__ __forceinline__ uint8_t* bound_slot(TcSmem<D>& S, int s) {
  using C = TcCfg<D>;
  return s < C::kBoundKvSlots
             ? S.k[0] + s * C::kBoundSlotBytes
             : reinterpret_cast<uint8_t*>(&S.cand_id[0][0][0]) + (s - C::kBoundKvSlots) * C::kBoundSlotBytes;
}
static_assert(2 * (sizeof(TcSmem<32>) + 1024) <= 228 * 1024, "shared memory per SM (d = 32, two CTAs)");

struct TcParams {
  const int32_t* off;
  const uint16_t* gates;
  const int32_t* idx;
  const int32_t* forced;
  uint16_t* out;
  float* obranch;
  uint16_t* obr;  // optional saved branch outputs o_b, bf16 [N][Hq][n_gates][D] (fused forward only)
  float* lse;
  uint32_t* status;
  int N, B, Hq, Hkv, G, top_k, idx_heads, n_forced, window, n_gates, route_all, branches, lse_stride, lse_first;
  float scale_log2;
  // compressed-branch key count (block means, or gathered forced tokens); n_ckeys_dev overrides it
  int n_ckeys;
  const int* n_ckeys_dev;
  // query blocks of a fixed size instead of `off` (dense passes over pooled queries or all tokens)
  int uniform_block;
  // self/cross mixture (kModeMix): blocks [0, mix_bx) are stream x, the rest stream y; the
  // compressed slot (gate 0) attends every token of the query's own stream and the selected slot
  // (gate 1) every token of the other one, both read from the token K / V
  int mix_bx;
  // streaming top-k of the compressed-branch logits (pooled-query routing, d = 64 only):
  // topk_idx [rows][topk_heads][topk_k]; blocks whose bit is set in forced_bits are skipped
  int32_t* topk_idx;
  int topk_k;
  const uint32_t* forced_bits;
  // per-row lower bound on the topk_k-th largest non-forced logit [rows][topk_heads]: the bound
  // pass (bound_pass = 1: scores only, no softmax, no P V) writes it; the top-k pass reads it
  float* topk_thr;
  int bound_pass;
  int n_pairs, n_groups;  // 128-row tile pairs per query block, KV groups (grid x = (a * groups + g) * pairs + pair)
  // optional row -> block id map of the keys (the pooled keys may be stored in another order);
  // the emitted top-k are block ids
  const int32_t* topk_ids;
  // optional exact ranking: fp32 pooled queries [rows][topk_heads][64] and keys [key rows][heads][64]
  // (key rows in the stored order) and the largest L2 norm of a key mean (float bits); with them
  // the candidates are ranked by fp32 logits recomputed from the means, and the gate is widened by
  // a bound on the error of the bf16-operand logits, so the result is the ranking of the exact
  // means rather than of their bf16 roundings
  const float* rescore_q;
  const float* rescore_k;
  const uint32_t* rescore_kmax;
};

enum : int { TC_CMP = 1, TC_SLC = 2, TC_WIN = 4 };

// chunk sequence shared by the three roles: [cmp chunks][slc chunks][win chunk], 64 keys each
struct Chunks {
  int n_cmp, n_slc, n_win, total;
  __device__ __forceinline__ int branch(int c, int& local) const {
    if (c < n_cmp) { local = c; return 0; }
    if (c < n_cmp + n_slc) { local = c - n_cmp; return 1; }
    local = c - n_cmp - n_slc;  // window chunks (several when the band spans more than 64 keys)
    return 2;
  }
  __device__ __forceinline__ bool first_of_branch(int c) const {
    return c == 0 || c == n_cmp || c == n_cmp + n_slc;
  }
};

// Kernel modes.  kModeShort: blocks of at most 64 tokens (a CTA's window band is its whole block,
// one chunk from the block start).  kModeLong: blocks of up to 512 tokens (selected blocks take
// several 64-key chunks, and the window band of a CTA may start inside the block and span several
// chunks).  kModeMix: the self/cross mixture (the compressed slot is the query's own stream and the
// selected slot the other stream, both token ranges in 64-key chunks; no window).
enum : int { kModeShort = 0, kModeLong = 1, kModeMix = 2 };

// first key row (block-mean index or token index) and number of valid keys of chunk (br, local)
template <int D, int kMode>
__device__ __forceinline__ void chunk_keys(const TcSmem<D>& S, const TcParams& p, int br, int local, int t0,
                                           int n_a, int n_ckeys, int& start, int& nvalid) {
  if (br == 0) {
    start = (kMode == kModeMix ? S.c_lo : 0) + local * 64;
    nvalid = min(64, n_ckeys - local * 64);
  } else if (br == 1) {
    if (kMode == kModeMix) {
      start = S.s_lo + 64 * local;
      nvalid = min(64, S.s_hi - start);
    } else if (p.route_all) {
      start = p.off[local];
      nvalid = p.off[local + 1] - start;
    } else {
      start = S.sel_start[local];
      nvalid = S.sel_n[local];
    }
  } else if (kMode == kModeLong) {
    start = t0 + S.win_lo + 64 * local;
    nvalid = min(64, S.win_hi + 1 - (S.win_lo + 64 * local));
  } else {
    start = t0;
    nvalid = n_a;
  }
}

// Top-k over a row's buffered candidates (logits at val[i * 128], key rows at id[i * 128]).  The
// rank of entry i in the order (logit desc, row asc) is the number of entries with a larger logit
// plus those with an equal logit and a lower row; ranks form a permutation of 0..n-1.
constexpr int kMaxCand = 64;

// exact rank from shared memory, ties included (the fallback when two logits are equal)
__device__ __forceinline__ int cand_rank_exact(const float* val, const int* id, int n, int i, float vi) {
  int r = 0;
  const int ji = id[i * 128];
  for (int j = 0; j < n; ++j) {
    const float vj = val[j * 128];
    r += (vj > vi || (vj == vi && id[j * 128] < ji)) ? 1 : 0;
  }
  return r;
}

// Ranks of all n <= kMaxCand candidates, each logit counted against all the others held in
// registers: f(i, r) is called with r = the number of strictly larger logits, which is the rank
// when no two logits are equal.  That holds exactly when the counts sum to n (n - 1) / 2, and
// the return value says so; otherwise the caller takes the exact tie-aware ranks.
template <class F>
__device__ __forceinline__ bool cand_ranks_fast(const float* val, int n, F f) {
  float v[kMaxCand];
#pragma unroll
  for (int j = 0; j < kMaxCand; ++j) v[j] = j < n ? val[j * 128] : -INFINITY;
  int sum = 0;
  for (int i = 0; i < n; ++i) {
    const float vi = val[i * 128];
    int r = 0;
#pragma unroll
    for (int j = 0; j < kMaxCand; ++j) r += v[j] > vi ? 1 : 0;
    f(i, r);
    sum += r;
  }
  return 2 * sum == n * (n - 1);
}

struct KeepBest {
  int n;
  float thr;
};

// fp32 logit (unscaled dot product) of a pooled query row and a pooled key row, 64 dims each
__device__ __noinline__ float rescore_dot64(const float* __restrict__ q, const float* __restrict__ k) {
  const float4* a = reinterpret_cast<const float4*>(q);
  const float4* b = reinterpret_cast<const float4*>(k);
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll 4
  for (int i = 0; i < 16; ++i) {
    const float4 x = __ldg(a + i), y = __ldg(b + i);
    s0 = fmaf(x.x, y.x, s0);
    s1 = fmaf(x.y, y.y, s1);
    s2 = fmaf(x.z, y.z, s2);
    s3 = fmaf(x.w, y.w, s3);
  }
  return (s0 + s1) + (s2 + s3);
}

// Replace the row's n buffered logits by fp32 logits recomputed from the pooled means (the
// key row of candidate i is id[i * 128]).
__device__ __noinline__ void topk_rescore(float* val, const int* id, int n, const float* qrow, const float* kbase,
                                          size_t krow_stride) {
  for (int i = 0; i < n; ++i) val[i * 128] = rescore_dot64(qrow, kbase + (size_t)id[i * 128] * krow_stride);
}

// Keep the k best of a row's n > k buffered candidates, in buffer order; the new gate is the k-th
// best logit (a later key, from a larger block, has to beat it strictly).
__device__ __noinline__ KeepBest topk_keep_best(float* val, int* id, int n, int k) {
  uint64_t keep = 0;
  if (!cand_ranks_fast(val, n, [&](int i, int r) { keep |= (uint64_t)(r < k) << i; })) {
    keep = 0;
    for (int i = 0; i < n; ++i) keep |= (uint64_t)(cand_rank_exact(val, id, n, i, val[i * 128]) < k) << i;
  }
  int m = 0;
  float lo = INFINITY;
  for (int i = 0; i < n; ++i) {
    if (!((keep >> i) & 1ull)) continue;
    const float v = val[i * 128];
    val[m * 128] = v;
    id[m * 128] = id[i * 128];
    lo = fminf(lo, v);
    ++m;
  }
  return KeepBest{m, lo};
}

// A full buffer (k above kCand - 16, where keeping the k best would leave less room than one quarter
// of a chunk can append): the new candidate (logit v, key row j) replaces the worst entry when it
// ranks above it; returns the buffer's new worst logit, the gate for the next candidates.
__device__ __noinline__ float topk_insert_full(float* val, int* id, int n, float v, int j) {
  int w = 0;
  for (int i = 1; i < n; ++i) {
    const float vi = val[i * 128], vw = val[w * 128];
    if (vi < vw || (vi == vw && id[i * 128] > id[w * 128])) w = i;
  }
  const float vw = val[w * 128];
  if (v > vw || (v == vw && j < id[w * 128])) {
    val[w * 128] = v;
    id[w * 128] = j;
  }
  float lo = INFINITY;
  for (int i = 0; i < n; ++i) lo = fminf(lo, val[i * 128]);
  return lo;
}

// The appends of one quarter (16 keys, logits -inf where not eligible) for k above kCand - 16:
// append while the buffer has room, then each new candidate replaces the worst entry (with the
// exact ranking, the buffer is re-scored in fp32 once and each newcomer on arrival); returns the
// buffer count, the gate and whether the buffer holds fp32 logits.
struct Quarter16 {
  float v[16];
};
struct CandState {
  int n;
  float thr;
  bool rescored;
};
__device__ __noinline__ CandState topk_quarter_full(Quarter16 q, int key0, CandState st, float* val, int* id,
                                                    int cap, bool exact, const float* qrow, const float* kbase,
                                                    size_t kstride, float err) {
  for (int i = 0; i < 16; ++i) {
    float sv = q.v[i];
    if (!(sv > st.thr)) continue;
    const int j = key0 + i;
    if (st.n < cap) {
      val[st.n * 128] = sv;
      id[st.n * 128] = j;
      ++st.n;
      continue;
    }
    if (exact) {
      if (!st.rescored) topk_rescore(val, id, st.n, qrow, kbase, kstride);
      st.rescored = true;
      sv = rescore_dot64(qrow, kbase + (size_t)j * kstride);
    }
    const float lo = topk_insert_full(val, id, st.n, sv, j);
    st.thr = exact ? lo - err : lo;
  }
  return st;
}

// Emit the row's k best in order (logit desc, row asc); a row with fewer than k candidates pads
// with -1.
__device__ __noinline__ void topk_emit(const float* val, const int* id, int n, int k, int32_t* dst,
                                       const int32_t* ids) {
  auto put = [&](int r, int i) { dst[r] = ids != nullptr ? ids[id[i * 128]] : id[i * 128]; };
  if (!cand_ranks_fast(val, n, [&](int i, int r) { if (r < k) put(r, i); })) {
    for (int i = 0; i < n; ++i) {
      const int r = cand_rank_exact(val, id, n, i, val[i * 128]);
      if (r < k) put(r, i);
    }
  }
  for (int r = n; r < k; ++r) dst[r] = -1;
}

template <int D, int kMode>
__global__ void __launch_bounds__(kTcThreads, TcCfg<D>::kCtasPerSm)
nsa_attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap kcmap,
                   const __grid_constant__ CUtensorMap vcmap, const TcParams p) {
  using C = TcCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  TcSmem<D>& S = *reinterpret_cast<TcSmem<D>*>(smem_raw + (((raw + 1023u) & ~1023u) - raw));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // grid (pair of 128-row tiles, KV group, query block): the tile pairs and groups of one query
  // block run side by side (they read the same selected blocks, whose K and V rows hold both
  // groups' heads).  Past 65535 query blocks the grid is one-dimensional in the same order,
  // x = (query block * KV groups + group) * pairs + pair.
  int pair, g, a;
  if (gridDim.y * gridDim.z > 1) {
    pair = blockIdx.x;
    g = blockIdx.y;
    a = blockIdx.z;
  } else {
    const unsigned bg = blockIdx.x / (unsigned)p.n_pairs;
    pair = (int)(blockIdx.x - bg * (unsigned)p.n_pairs);
    a = (int)(bg / (unsigned)p.n_groups);
    g = (int)(bg - (unsigned)a * (unsigned)p.n_groups);
  }
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
        if (kMode == kModeLong) {
          // one 64-key chunk per 64 tokens of the block
          for (int s0 = p.off[j]; s0 < p.off[j + 1] && n < kTcMaxSel; s0 += 64) {
            S.sel_start[n] = s0;
            S.sel_n[n] = min(64, p.off[j + 1] - s0);
            ++n;
          }
        } else {
          S.sel_start[n] = p.off[j];
          S.sel_n[n] = p.off[j + 1] - p.off[j];
          ++n;
        }
      }
    }
    S.n_sel = n;
    if (kMode == kModeLong) {
      S.win_lo = max(0, tile0 * tokens_per_tile - p.window / 2);
      S.win_hi = min(n_a - 1, min(n_a, (tile0 + 2) * tokens_per_tile) - 1 + p.window / 2 - 1);
    }
    if (kMode == kModeMix) {
      const int nx = p.off[p.mix_bx], nall = p.off[p.B];
      const bool in_x = a < p.mix_bx;
      S.c_lo = in_x ? 0 : nx;  // own stream
      S.c_hi = in_x ? nx : nall;
      S.s_lo = in_x ? nx : 0;  // the other stream (may be empty)
      S.s_hi = in_x ? nall : nx;
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&S.q_full[t], 1);
      mbar_init(&S.s_full[t], 1);
      mbar_init(&S.p_full[t], 128);
      mbar_init(&S.pv_done[t], 1);
      for (int b = 0; b < C::kBoundBufs; ++b) {
        mbar_init(&S.bs_full[t][b], 1);
        mbar_init(&S.bs_free[t][b], 128);
      }
    }
    for (int s = 0; s < C::kBoundStages; ++s) {
      mbar_init(&S.kb_full[s], 1);
      mbar_init(&S.kb_empty[s], 1);
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
  const int n_ckeys = kMode == kModeMix              ? S.c_hi - S.c_lo
                      : p.n_ckeys_dev != nullptr ? *p.n_ckeys_dev
                                                 : p.n_ckeys;
  cs.n_cmp = (p.branches & TC_CMP) ? (n_ckeys + C::kKeys - 1) / C::kKeys : 0;
  cs.n_slc = (p.branches & TC_SLC) ? (kMode == kModeMix ? (S.s_hi - S.s_lo + 63) / 64 : p.route_all ? p.B : S.n_sel)
                                   : 0;
  // the window band of this CTA's tokens in 64-key chunks (one for blocks of at most 64 tokens)
  cs.n_win = ((p.branches & TC_WIN) && p.window > 0 && kMode != kModeMix)
                 ? (kMode == kModeLong ? (S.win_hi - S.win_lo + 64) / 64 : 1)
                 : 0;
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
      // bound pass (compressed keys only): K alone, kBoundKeys rows per box
      const int nb = (D == 64 && p.bound_pass) ? (n_ckeys + C::kBoundKeys - 1) / C::kBoundKeys : 0;
      for (int c = 0; c < nb; ++c) {
        const int st = c % C::kBoundStages;
        if (c >= C::kBoundStages &&
            !mbar_wait(&S.kb_empty[st], ((c / C::kBoundStages) + 1) & 1, abort, p.status))
          break;
        mbar_arrive_expect_tx(&S.kb_full[st], C::kBoundSlotBytes);
        tma_load_3d(bound_slot(S, st), &kcmap, &S.kb_full[st], 0, g, c * C::kBoundKeys);
        issued = c + 1;
      }
      for (int c = 0; !p.bound_pass && c < cs.total; ++c) {
        const int st = c % C::kStages;
        if (c >= C::kStages && !mbar_wait(&S.kv_empty[st], ((c / C::kStages) + 1) & 1, abort, p.status)) break;
        int local, start, nvalid;
        const int br = cs.branch(c, local);
        chunk_keys<D, kMode>(S, p, br, local, t0, n_a, n_ckeys, start, nvalid);
        mbar_arrive_expect_tx(&S.kv_full[st], 2 * C::kKVBytes);
        tma_load_3d(S.k[st], br == 0 ? &kcmap : &kmap, &S.kv_full[st], 0, g, start);
        tma_load_3d(S.v[st], br == 0 ? &vcmap : &vmap, &S.kv_full[st], 0, g, start);
        issued = c + 1;
      }
      if (*abort) {
        // let the copies already issued land before the CTA's shared memory goes away
        const int ring = p.bound_pass ? C::kBoundStages : C::kStages;
        for (int c = max(0, issued - ring); c < issued; ++c) {
          volatile int no_abort = 0;
          mbar_wait(p.bound_pass ? &S.kb_full[c % ring] : &S.kv_full[c % ring], (c / ring) & 1, &no_abort, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (D == 64 && p.bound_pass && cs.total > 0) {
      // bound pass: the issuing thread is the bottleneck, so the whole warp runs the loop and one
      // elected lane issues each instruction
      bool ok = mbar_wait_w(&S.q_full[0], 0, abort, p.status) && mbar_wait_w(&S.q_full[1], 0, abort, p.status);
      tc_fence_after();
      // shared-memory descriptors are computed once; a byte offset moves the start-address
      // field (address / 16, bits 0..13; shared addresses stay below 2^18) by offset / 16
      const uint64_t qdesc[2] = {smem_desc(smem_u32(S.q[0]), 16, C::kAtomBytes, C::kLayout),
                                 smem_desc(smem_u32(S.q[1]), 16, C::kAtomBytes, C::kLayout)};
      const uint64_t kdesc = smem_desc(smem_u32(S.k[0]), 16, C::kAtomBytes, C::kLayout);
      // bound pass: scores only, N = kBoundKeys per MMA, into kBoundBufs score buffers per tile
      // (one tile's chunk is computed while the other tile's warps reduce theirs); each buffer has
      // its own full/free barrier pair, completed once per kBoundBufs chunks
      const int nb = (n_ckeys + C::kBoundKeys - 1) / C::kBoundKeys;
      for (int c = 0; ok && c < nb; ++c) {
        const int st = c % C::kBoundStages;
        if (!mbar_wait_w(&S.kb_full[st], (c / C::kBoundStages) & 1, abort, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint64_t bd = kdesc + (uint64_t)((smem_u32(bound_slot(S, st)) - smem_u32(S.k[0])) >> 4);
        const int b = c % C::kBoundBufs;
        for (int t = 0; t < 2; ++t) {
          if (c >= C::kBoundBufs) {
            if (!mbar_wait_w(&S.bs_free[t][b], ((c / C::kBoundBufs) + 1) & 1, abort, p.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          const uint32_t d = tmem + t * C::kColsPerTile + b * C::kBoundKeys;
#pragma unroll
          for (int k = 0; k < D / 16; ++k) mma_ss_w(d, qdesc[t] + 2 * k, bd + 2 * k, C::kIdescBound, k > 0 ? 1u : 0u);
          mma_commit_w(&S.bs_full[t][b]);
        }
        if (!ok) break;
        mma_commit_w(&S.kb_empty[st]);
      }
      mma_commit_w(&S.drain);
      volatile int no_abort = 0;
      mbar_wait(&S.drain, 0, &no_abort, nullptr);
    } else if (!p.bound_pass && lane == 0 && cs.total > 0) {
      // attention passes: one thread issues (it mostly waits on the softmax warps)
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
      auto issue_qk = [&](int t, int c) {
        const uint32_t d = tmem + t * C::kColsPerTile + C::kColS;
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
      for (int c = 0; ok && c < cs.total; ++c) {
        if (!mbar_wait(&S.kv_full[c % C::kStages], (c / C::kStages) & 1, abort, p.status)) { ok = false; break; }
        tc_fence_after();
        for (int t = 0; t < 2; ++t) {
          // S(c) is issued ahead of P(c - 1) V: it overwrites only S, which the softmax released
          // with P(c - 1), and the softmax waits for P(c - 1) V before it stores P(c)
          if (c > 0) {
            if (!mbar_wait(&S.p_full[t], (c - 1) & 1, abort, p.status)) { ok = false; break; }
            tc_fence_after();
          }
          issue_qk(t, c);
          mma_commit(&S.s_full[t]);
          if (c > 0) {
            issue_pv(t, c - 1);
            mma_commit(&S.pv_done[t]);
          }
        }
        if (!ok) break;
        if (c > 0) mma_commit(&S.kv_empty[(c - 1) % C::kStages]);
      }
      for (int t = 0; ok && t < 2; ++t) {
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
        if (p.obr != nullptr && valid) {
          uint4* dst = reinterpret_cast<uint4*>(p.obr + (orow * p.n_gates + br) * D + 32 * i);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * e]) * inv, __uint_as_float(o[8 * e + 1]) * inv),
                                pack_bf16x2(__uint_as_float(o[8 * e + 2]) * inv, __uint_as_float(o[8 * e + 3]) * inv),
                                pack_bf16x2(__uint_as_float(o[8 * e + 4]) * inv, __uint_as_float(o[8 * e + 5]) * inv),
                                pack_bf16x2(__uint_as_float(o[8 * e + 6]) * inv, __uint_as_float(o[8 * e + 7]) * inv));
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
    // this row's window band relative to the first key of the current window chunk (with long
    // blocks, moved along as the window chunks come, which are the last of the stream)
    int wlo = tok_local - p.window / 2, whi = tok_local + p.window / 2 - 1;
    const float sc = p.scale_log2;
    int br = 0, nv = 0;
    // raw score of key j of the chunk, or -inf where masked (short block or outside the window band)
    auto masked = [&](uint32_t raw, int j) -> float {
      bool kv = j < nv;
      if (br == 2) kv = kv && j >= wlo && j <= whi;
      return kv ? __uint_as_float(raw) : -INFINITY;
    };
    // ---- streaming top-k of the compressed-branch logits (pooled-query routing) ----
    // Every non-forced key whose logit is above the row's gate is appended, with its block id, to
    // the row's candidate buffer (logits in this row's column of the otherwise unused output
    // accumulator, ids in cand_id).  The gate starts just below a lower bound on the k-th largest
    // non-forced logit (from the bound pass), so every key at or above the bound is a candidate and
    // no key below it can be among the k best (k keys at or above it exist).  With that bound a
    // row collects a few dozen candidates over the whole stream; should the buffer run short, the
    // warp's rows keep their k best and the gate rises to the k-th of them (for k above kCand - 16,
    // where that would leave less room than a quarter chunk appends, a full buffer instead takes
    // each new candidate in place of its worst entry).  The k best of the buffer are ranked at the
    // end.
    const bool topk_on = (D == 64) && p.topk_idx != nullptr;
    float thr = -INFINITY;
    int key_base = 0;    // block id of key 0 of the current chunk
    uint64_t fmask = 0;  // forced blocks among the chunk's 64 keys (never candidates)
    int ncand = 0;       // this row's buffered candidates
    int n_exact = 0;     // leading entries that already hold fp32 logits (exact ranking)
    float* cval = acc;
    int* cid = &S.cand_id[t][0][row];
    // exact ranking (see TcParams::rescore_q): every bf16-operand logit lies within err of the
    // fp32 logit of the means, err = (2^-7 + 2^-14) |q|_2 max_j |k_j|_2: rounding each operand to
    // bf16 moves it by at most 2^-8 of itself, so a product q_i k_i moves by at most
    // (2^-7 + 2^-16) |q_i k_i|; the fp32 sums of 64 products add at most about 2^-18 of
    // sum_i |q_i k_i|; and sum_i |q_i k_i| <= |q|_2 |k|_2.  A key among the exact k best then has a bf16
    // logit at least (bound - 2 err), which is where the gate starts, and after a compaction a key
    // can enter only with a bf16 logit above (k-th exact - err).
    const bool exact = topk_on && p.rescore_q != nullptr;
    const float* qrow = nullptr;
    const float* kbase = nullptr;
    size_t kstride = 0;
    float err = 0.f;
    if (exact && valid) {
      qrow = p.rescore_q + ((size_t)(t0 + R) * p.Hkv + g) * 64;
      kbase = p.rescore_k + (size_t)g * 64;
      kstride = (size_t)p.Hkv * 64;
      float n2 = 0.f;
      for (int i = 0; i < 64; ++i) n2 = fmaf(__ldg(qrow + i), __ldg(qrow + i), n2);
      // (the extra 2^-7 of the bound also covers the rounding of the fp32 norms themselves)
      err = 0.0078125f * 1.0078125f * sqrtf(n2) * __uint_as_float(*p.rescore_kmax) + 1e-30f;
    }
    auto topk_compact = [&]() {
      if (ncand > p.topk_k) {
        // with the exact ranking the entries appended since the last compaction are re-scored in
        // fp32 first (the kept ones, first in the buffer, already hold fp32 logits; keeping the
        // entries within the error slack of the k-th bf16 value instead was measured slower: too
        // many of them stay)
        if (exact && valid)
          topk_rescore(cval + n_exact * 128, cid + n_exact * 128, ncand - n_exact, qrow, kbase, kstride);
        const KeepBest kb = topk_keep_best(cval, cid, ncand, p.topk_k);
        ncand = kb.n;
        n_exact = kb.n;
        thr = exact ? kb.thr - err : kb.thr;
      }
    };
    const bool big_k = topk_on && p.topk_k > C::kCand - 16;
    bool rescored = false;  // a full buffer holds the fp32 logits of the means (exact ranking)
    auto topk_append = [&](float sv, int j) {
      if (sv > thr) {
        cval[ncand * 128] = sv;
        cid[ncand * 128] = key_base + j;
        ++ncand;
      }
    };
    if (topk_on && p.topk_thr != nullptr && valid) {
      const float b = p.topk_thr[(size_t)(t0 + R) * p.Hkv + g];
      if (b > -INFINITY) thr = nextafterf(exact ? b - 2.f * err : b, -INFINITY);
    }
    // forced blocks among compressed-key chunk c (bit j: block 64 c + j); the next chunk's mask
    // is loaded one chunk ahead
    auto load_fmask = [&](int c) -> uint64_t {
      return (uint64_t)p.forced_bits[2 * c] | ((uint64_t)p.forced_bits[2 * c + 1] << 32);
    };
    uint64_t fmask_next = (topk_on && cs.n_cmp > 0) ? load_fmask(0) : 0ull;

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
        // with the top-k on, the running max is kept per quarter (two chains), since the quarter's
        // max is the top-k gate as well
        float qm[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int j = 16 * qd + 2 * i;
          const float s0 = need_mask ? masked(r[2 * i], j) : __uint_as_float(r[2 * i]);
          const float s1 = need_mask ? masked(r[2 * i + 1], j + 1) : __uint_as_float(r[2 * i + 1]);
          // the running max is tracked only where it is the top-k gate; elsewhere the row sum
          // tells when the reference has to move (see the caller)
          if constexpr (topk) qm[i & 1] = fmax3(qm[i & 1], s0, s1);
          float x0, x1;
          ffma2(x0, x1, s0, s1, sc, nm);  // one packed FMA for the pair
          float p0, p1;
          // the polynomial only where every key of the chunk is valid (see poly_exp2_pair)
          if (!need_mask && kPolyMod > 0 && (8 * qd + i) % (kPolyMod > 0 ? kPolyMod : 1) == kPolyMod - 1) {
            poly_exp2_pair(p0, p1, x0, x1);
          } else {
            p0 = fast_exp2(x0);
            p1 = fast_exp2(x1);
          }
          fadd2_acc(ls[2 * (i & 1)], ls[2 * (i & 1) + 1], p0, p1);  // packed row-sum accumulate
          pk[i] = pack_bf16x2(p0, p1);
        }
        if (qd == 0) wait_pv();
        if (pv_ok) tmem_st8(tbase + C::kColP + 8 * qd, pk);
        if constexpr (topk) {
          float qmx = fmaxf(qm[0], qm[1]);
          mx[qd] = fmaxf(mx[qd], qmx);
          // forced blocks take part in the softmax but are never candidates: in the (few) quarters
          // that hold one, they drop out of the gate and of the appends
          const uint32_t qf = (uint32_t)(fmask >> (16 * qd)) & 0xffffu;
          float sv[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) sv[i] = need_mask ? masked(r[i], 16 * qd + i) : __uint_as_float(r[i]);
          if (qf != 0u) {
            qmx = -INFINITY;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              if ((qf >> i) & 1u) sv[i] = -INFINITY;
              qmx = fmaxf(qmx, sv[i]);
            }
          }
          // only quarters where some row of the warp has a key above its gate visit the keys
          if (__any_sync(0xffffffffu, qmx > thr)) {
            if (!big_k) {
#pragma unroll
              for (int i = 0; i < 16; ++i) topk_append(sv[i], 16 * qd + i);
              // a quarter appends at most 16 candidates per row
              if (__any_sync(0xffffffffu, ncand > C::kCand - 16)) topk_compact();
            } else {
              // (one call site: the full-buffer insertion kept out of the unrolled appends)
              Quarter16 qv;
#pragma unroll
              for (int i = 0; i < 16; ++i) qv.v[i] = sv[i];
              const CandState cs2 = topk_quarter_full(qv, key_base + 16 * qd, CandState{ncand, thr, rescored}, cval,
                                                      cid, C::kCand, exact && valid, qrow, kbase, kstride, err);
              ncand = cs2.n;
              thr = cs2.thr;
              rescored = cs2.rescored;
            }
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

    if (D == 64 && p.bound_pass) {
      // ---- bound pass (d = 64 only): per row, the max non-forced logit of each of 64 key groups (the
      // 32-key block b of the stream joins group b mod 64, so 1024 keys already fill 32 groups),
      // then the topk_k-th largest group max.  Groups are disjoint, so
      // at least topk_k distinct keys score at or above that value: a lower bound on the
      // topk_k-th largest logit that needs no selection in the per-key loop.
      float* gmax = acc;  // gmax[i * 128], i < 64 (the output accumulator is unused here)
#pragma unroll 1
      for (int i = 0; i < 64; ++i) gmax[i * 128] = -INFINITY;
      // max over 16 keys; forced keys (bits of qf) and keys past nv drop out
      auto quarter_max = [&](const uint32_t* r, int j0, uint32_t qf, bool tail) -> float {
        float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
          m0 = fmax3(m0, __uint_as_float(r[i]), __uint_as_float(r[i + 1]));
        }
        if (qf != 0u || tail) {
          m0 = -INFINITY;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const bool drop = ((qf >> i) & 1u) || j0 + i >= nv;
            m1 = fmaxf(m1, drop ? -INFINITY : __uint_as_float(r[i]));
          }
        }
        return fmaxf(m0, m1);
      };
      // forced blocks among the chunk's kBoundKeys keys, one word per 32 keys (words past the
      // last key are not read); the next chunk's words are loaded one chunk ahead
      constexpr int kW = C::kBoundKeys / 32;
      const int nb = (n_ckeys + C::kBoundKeys - 1) / C::kBoundKeys;
      auto load_words = [&](int c, uint32_t* w) {
#pragma unroll
        for (int i = 0; i < kW; ++i) w[i] = (c * kW + i) * 32 < n_ckeys ? p.forced_bits[c * kW + i] : 0u;
      };
      uint32_t fw[kW], fw_next[kW];
      if (nb > 0) load_words(0, fw_next);
      bool okb = true;
      for (int c = 0; c < nb; ++c) {
        const int b = c % C::kBoundBufs;
#pragma unroll
        for (int i = 0; i < kW; ++i) fw[i] = fw_next[i];
        if (c + 1 < nb) load_words(c + 1, fw_next);
        nv = min(C::kBoundKeys, n_ckeys - c * C::kBoundKeys);
        const bool tail = nv < C::kBoundKeys;
        if (!wait_all(&S.bs_full[t][b], (c / C::kBoundBufs) & 1)) { okb = false; break; }
        tc_fence_after();
        // 32 columns at a time, each load issued before the previous block is reduced
        const uint32_t col = tbase + b * C::kBoundKeys;
        uint32_t ra[32], rb[32];
        float mxs[kW];  // max of each 32-key block of the chunk
        tmem_ld32(col, ra);
        tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < kW; ++h) {
          uint32_t* cur = (h & 1) ? rb : ra;
          uint32_t* nxt = (h & 1) ? ra : rb;
          if (h + 1 < kW) tmem_ld32(col + 32 * (h + 1), nxt);
          mxs[h] = fmaxf(quarter_max(cur, 32 * h, fw[h] & 0xffffu, tail),
                         quarter_max(cur + 16, 32 * h + 16, fw[h] >> 16, tail));
          if (h + 1 < kW) tmem_ld_wait();
        }
        tc_fence_before();
        mbar_arrive(&S.bs_free[t][b]);
#pragma unroll
        for (int h = 0; h < kW; ++h) {
          float& gv = gmax[((c * kW + h) & 63) * 128];
          gv = fmaxf(gv, mxs[h]);
        }
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
      chunk_keys<D, kMode>(S, p, br, local, t0, n_a, n_ckeys, start, nv);
      if (kMode == kModeLong && br == 2) {
        const int shift = local == 0 ? S.win_lo : 64;  // the chunk starts this many keys further on
        wlo -= shift;
        whi -= shift;
      }
      const bool need_mask = br == 2 || nv < 64;
      if (topk_on && br == 0) {
        key_base = local * 64;
        fmask = fmask_next;
        if (local + 1 < cs.n_cmp) fmask_next = load_fmask(local + 1);
      }
      float lsum;
      if (first) {
        wait_pv();
        if (!pv_ok) { ok = false; break; }
        if (c > 0) finalize(prev_br, m, l);
        if (topk_on && br == 0) {
          // the top-k pass moves its reference by the max (its gate), so it starts from the max
          const float mraw = chunk_max(need_mask);
          m = mraw == -INFINITY ? -INFINITY : mraw * sc;
          exp_pass(need_mask, m == -INFINITY ? 0.f : m, &lsum);
        } else {
          // Start the branch from reference 0 and keep it while the chunk's sum of P lies in
          // [2^-64, 2^16]: every P then stays far inside the normal range (and the largest is at
          // least 2^-70).  Otherwise (or with every key masked) the chunk max is read from S and
          // the chunk redone from it.  Nothing has reached O yet: its first P V overwrites it.
          m = 0.f;
          exp_pass(need_mask, 0.f, &lsum);
          const bool off_range = !(lsum <= 65536.f && lsum >= 5.421010862427522e-20f);
          if (__any_sync(0xffffffffu, off_range)) {
            const float mraw = chunk_max(need_mask);
            if (off_range) m = mraw == -INFINITY ? -INFINITY : mraw * sc;
            exp_pass(need_mask, m == -INFINITY ? 0.f : m, &lsum, false);
          }
        }
        l = lsum;
      } else {
        const float mraw = exp_pass(need_mask, m == -INFINITY ? 0.f : m, &lsum);
        if (!pv_ok) { ok = false; break; }
        // Move the reference only when it has fallen well behind the row max.  With the top-k on,
        // the chunk max is at hand (the gate): move when it exceeds the reference by more than
        // 2^8.  Otherwise the chunk's sum of P decides: every P is at most that sum, so a sum up
        // to 2^16 keeps every P (and O) far inside range, and only a larger sum (or an infinite
        // one) has the chunk max read back from S and the reference moved to it.
        float cand;
        bool grow;
        if (topk_on && br == 0) {
          cand = mraw == -INFINITY ? -INFINITY : mraw * sc;
          grow = cand > m + 8.f;
        } else {
          // (no reference yet, after a first chunk without valid keys: always take the max)
          grow = !(lsum <= 65536.f) || m == -INFINITY;
          cand = -INFINITY;
          if (__any_sync(0xffffffffu, grow)) {
            const float mr = chunk_max(need_mask);
            cand = mr == -INFINITY ? -INFINITY : mr * sc;
          }
        }
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
    // the mixture's cross slot over an empty stream: no keys, a zero output and LSE -inf
    if (kMode == kModeMix && cs.n_slc == 0 && valid && p.lse != nullptr) p.lse[orow * p.lse_stride + p.lse_first + 1] = -INFINITY;
    if (ok && topk_on && valid) {
      if (exact && rescored) n_exact = ncand;  // a full buffer is fp32 throughout
      if (exact) topk_rescore(cval + n_exact * 128, cid + n_exact * 128, ncand - n_exact, qrow, kbase, kstride);
      topk_emit(cval, cid, ncand, p.topk_k, p.topk_idx + ((size_t)(t0 + R) * p.Hkv + g) * p.topk_k, p.topk_ids);
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

template <int D, int kMode>
lsrm_status launch_tc_dl(const lsrm_nsa_desc& d, const TcParams& p, const void* q, const void* k, const void* v,
                        const void* kc, const void* vc, long long kc_rows, cudaStream_t stream) {
  CUtensorMap qm, km, vm, kcm, vcm;
  const void* kk = k ? k : kc;
  const void* vv = v ? v : vc;
  const void* kkc = kc ? kc : k;
  const void* vvc = vc ? vc : v;
  if (!make_map(&qm, q, D, d.n_q_heads, d.n_tokens, p.G, 128 / p.G)) return LSRM_ERR_CUDA;
  if (!make_map(&km, kk, D, d.n_kv_heads, k ? d.n_tokens : kc_rows, 1, 64)) return LSRM_ERR_CUDA;
  if (!make_map(&vm, vv, D, d.n_kv_heads, v ? d.n_tokens : kc_rows, 1, 64)) return LSRM_ERR_CUDA;
  if (!make_map(&kcm, kkc, D, d.n_kv_heads, kc ? kc_rows : d.n_tokens, 1, p.bound_pass ? TcCfg<D>::kBoundKeys : 64))
    return LSRM_ERR_CUDA;
  if (!make_map(&vcm, vvc, D, d.n_kv_heads, vc ? kc_rows : d.n_tokens, 1, 64)) return LSRM_ERR_CUDA;
  const size_t smem = sizeof(TcSmem<D>) + 1024;
  if (cudaFuncSetAttribute(nsa_attn_tc_kernel<D, kMode>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return LSRM_ERR_CUDA;
  const int tiles = (d.max_block_len * p.G + 127) / 128;
  TcParams pp = p;
  pp.n_pairs = (tiles + 1) / 2;
  pp.n_groups = d.n_kv_heads;
  const long long nx = (long long)d.n_blocks * d.n_kv_heads * pp.n_pairs;
  if (nx > INT32_MAX || d.n_kv_heads > 65535) return LSRM_ERR_UNSUPPORTED;
  const dim3 grid = d.n_blocks <= 65535 ? dim3((unsigned)pp.n_pairs, (unsigned)d.n_kv_heads, (unsigned)d.n_blocks)
                                        : dim3((unsigned)nx, 1, 1);
  nsa_attn_tc_kernel<D, kMode><<<grid, kTcThreads, smem, stream>>>(qm, km, vm, kcm, vcm, pp);
  return cudaGetLastError() == cudaSuccess ? LSRM_OK : LSRM_ERR_CUDA;
}

template <int D>
lsrm_status launch_tc_d(const lsrm_nsa_desc& d, const TcParams& p, const void* q, const void* k, const void* v,
                        const void* kc, const void* vc, long long kc_rows, cudaStream_t stream, bool mix = false) {
  if (mix) return launch_tc_dl<D, kModeMix>(d, p, q, k, v, kc, vc, kc_rows, stream);
  // long blocks only exist in the layer passes (the dense passes have fixed 256-row query groups)
  if (d.max_block_len > 64 && p.uniform_block == 0)
    return launch_tc_dl<D, kModeLong>(d, p, q, k, v, kc, vc, kc_rows, stream);
  return launch_tc_dl<D, kModeShort>(d, p, q, k, v, kc, vc, kc_rows, stream);
}

}  // namespace

lsrm_status launch_attn(const lsrm_nsa_desc& d, const int32_t* off, const void* q, const void* k, const void* v,
                           const void* kc, const void* vc, const void* gates, const int32_t* idx, int idx_heads,
                           int route_all, int branches, void* out, float* obranch, float* lse, int lse_stride,
                           int lse_first, uint32_t* status, cudaStream_t stream, void* obr) {
  const int G = d.n_q_heads / d.n_kv_heads;
  if (128 % G != 0) return LSRM_ERR_UNSUPPORTED;
  // selected blocks longer than 64 tokens take several 64-key chunks each
  const int chunks_per_block = (d.max_block_len + 63) / 64;
  if (!route_all && (long long)(d.n_forced + d.top_k) * chunks_per_block > kTcMaxSel) return LSRM_ERR_UNSUPPORTED;
  if (route_all && d.max_block_len > 64) return LSRM_ERR_UNSUPPORTED;
  TcParams p{};
  p.off = off;
  p.gates = (const uint16_t*)gates;
  p.idx = idx;
  p.forced = d.forced_blocks;
  p.out = (uint16_t*)out;
  p.obranch = obranch;
  p.obr = (uint16_t*)obr;
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

// Decoupled self/cross gated mixture over two token streams (blocks [0, bx) and [bx, B)): one
// launch, the compressed slot over the query's own stream and the selected slot over the other,
// gated by gates [N][Hq][2] = (self, cross) and summed in the epilogue.
lsrm_status launch_mixture(const lsrm_nsa_desc& d, const int32_t* off, int32_t bx, const void* q, const void* k,
                           const void* v, const void* gates, void* out, float* lse, uint32_t* status,
                           cudaStream_t stream) {
  const int G = d.n_q_heads / d.n_kv_heads;
  if (128 % G != 0) return LSRM_ERR_UNSUPPORTED;
  TcParams p{};
  p.off = off;
  p.gates = (const uint16_t*)gates;
  p.out = (uint16_t*)out;
  p.lse = lse;
  p.status = status;
  p.N = (int)d.n_tokens;
  p.B = d.n_blocks;
  p.Hq = d.n_q_heads;
  p.Hkv = d.n_kv_heads;
  p.G = G;
  p.n_gates = 2;
  p.branches = TC_CMP | TC_SLC;
  p.lse_stride = 2;
  p.lse_first = 0;
  p.mix_bx = bx;
  const float tau = d.scale > 0 ? d.scale : 1.0f / sqrtf((float)d.head_dim);
  p.scale_log2 = tau * 1.4426950408889634f;
  // both slots read token rows: the compressed slot's tensor maps cover K and V
  if (d.head_dim == 32) return launch_tc_d<32>(d, p, q, k, v, k, v, d.n_tokens, stream, true);
  if (d.head_dim == 64) return launch_tc_d<64>(d, p, q, k, v, k, v, d.n_tokens, stream, true);
  return LSRM_ERR_UNSUPPORTED;
}

// Dense multi-head attention of n_q query rows (q [n_q][H][D]) against n_ckeys rows of
// (kc, vc) ([kc_rows][H][D]), in fixed groups of 256 query rows: the pooled-query compressed
// branch (optionally with the streaming top-k that routes it) and the forced-block part of the
// pooled-query selected branch.  Writes fp32 obranch [n_q][H][D] and the natural-log lse [n_q][H].
// With topk_thr ([n_q][H] fp32 scratch) the top-k pass is preceded by the bound pass, whose
// per-row lower bound on the k-th logit lets the top-k pass skip almost every candidate.  With
// topk_ids the key rows are stored in another order (forced_bits then marks rows) and the
// emitted indices are topk_ids[row].  With rescore_q / rescore_k (fp32 pooled queries [n_q][H][64]
// and keys in the stored row order) and rescore_kmax (the largest key L2 norm as float bits) the top-k
// is the ranking of the fp32 logits of the means (see TcParams).
lsrm_status launch_attn_dense(int D, long long n_q, int H, const void* q, const void* kc, const void* vc,
                              long long kc_rows, int n_ckeys, const int* n_ckeys_dev, float tau, float* obranch,
                              float* lse, int32_t* topk_idx, int topk_k, const uint32_t* forced_bits,
                              float* topk_thr, uint32_t* status, cudaStream_t stream, const int32_t* topk_ids,
                              const float* rescore_q, const float* rescore_k, const uint32_t* rescore_kmax) {
  if (topk_idx != nullptr && (D != 64 || topk_k < 1 || topk_k > TcCfg<64>::kCand || forced_bits == nullptr))
    return LSRM_ERR_UNSUPPORTED;
  if (n_q > INT32_MAX) return LSRM_ERR_UNSUPPORTED;
  lsrm_nsa_desc d{};
  d.n_tokens = n_q;
  d.n_blocks = (int32_t)((n_q + 255) / 256);  // groups of 256 query rows (the query blocks of the grid)
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
  p.topk_ids = topk_ids;
  if (topk_idx != nullptr && rescore_q != nullptr && rescore_k != nullptr && rescore_kmax != nullptr) {
    p.rescore_q = rescore_q;
    p.rescore_k = rescore_k;
    p.rescore_kmax = rescore_kmax;
  }
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
