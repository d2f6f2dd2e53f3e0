// ORACLE — test infrastructure, not product code.
//
// A plain, slow, single-threaded fp64 CPU statement of what the LSRM
// native-sparse-attention (NSA) layer computes.  Only the tests, the smoke
// check and the benchmark's CPU-baseline leg may load it; the CUDA path shares
// no code, header, table or helper with it.
//
// Sources (the pages this follows; "LSRM page" = hyper.ai "LSRM" summary,
// "Speed3R page" = gist.science "Speed3R" technical summary):
//   compression  k_cmp = AvgPool(ResBlock(k_t)), v_cmp likewise  — LSRM page, 方法,
//                equations k^cmp / v^cmp.  ResBlock is a trained module and is
//                taken as the identity, so compression is the block mean.
//   score routing: NSA selects KV blocks by attention scores against the
//                compressed keys — LSRM page, 方法, 3D-aware routing paragraph.
//   geometric routing: nearest volume blocks by 3D Euclidean distance between
//                block centres — LSRM page, same paragraph.
//   branches: compressed context + selected blocks (fine detail) — LSRM page,
//                方法 (after the k^cmp equations); window attention computed
//                locally inside whole blocks — LSRM page, sequence-parallel
//                paragraph; Speed3R page, 2.1 (compression / selection branches).
//   gates: Sigmoid(Linear(x)) gate values weight the branch outputs — LSRM page,
//                方法, gate equations; Speed3R page, 2.1 gated aggregation.
//   camera routing: the query point is projected into every view, the view's
//                nearby image blocks are candidates, ranked by their smallest
//                token-to-query distance — LSRM page, 方法, 3D-aware routing paragraph.
//   self/cross mixture: o^x = w CrossAttn(x,x) + w CrossAttn(x,y) and likewise for
//                y — LSRM page, 方法, the dense blocks' gated cross-attention equations.
//
// Readings where the pages are silent (each also listed in the design notes):
//   * softmax scale tau = 1/sqrt(d); query head h uses KV group floor(h / (Hq/Hkv)).
//   * score routing is per (query block, KV group): Score[a,g,j] is the SUM over
//     the block's tokens and the group's heads of the compressed-branch softmax
//     probabilities p_cmp[t,h,j]; top-k by (score desc, j asc).
//   * geometric routing: centroid c[b] = round-half-up(sum of the block's lattice
//     coordinates / n_b) per axis, i.e. floor((2S + n) / (2n)); distance
//     D = sum over axes of (c[a] - c[j])^2 in int64; top-k by (D asc, j asc);
//     one index list per query block, shared by every KV group.
//   * window: W(t) = { u in block(t) : r(t) - w/2 <= r(u) <= r(t) + w/2 - 1 },
//     r = position inside the block; w = 0 switches the branch off.
//   * the selected key set of (a, g) is the union of the forced blocks and the
//     routed blocks (as a set).
//   * Speed3R variant (pooled_q = 1): the compressed branch uses the block-mean
//     query Qbar[beta(t)] and its output is copied to every token of the block;
//     routing is top-k by the raw pooled logit tau * Qbar . Kbar over the blocks
//     that are not forced; there is no window branch.
//
// Top-k everywhere: a full std::sort on (key, index).  Softmax: max-subtracted
// in fp64.  Inputs arrive as bf16 bit patterns and are widened exactly (or, for
// finite-difference checks, as doubles).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

struct Desc {
  int64_t n_tokens;
  int32_t n_blocks;
  int32_t n_q_heads, n_kv_heads, head_dim;
  int32_t top_k, window;
  double scale;      // 0 -> 1/sqrt(d)
  int32_t pooled_q;  // 0 LSRM, 1 Speed3R
  int32_t n_gates;   // 3 (cmp, slc, win) or 2 (cmp, slc)
};

inline double bf(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}
inline double bf(double x) { return x; }  // fp64 inputs (finite-difference checks)

inline double tau_of(const Desc& D) { return D.scale > 0 ? D.scale : 1.0 / std::sqrt((double)D.head_dim); }

inline int64_t floor_div(int64_t a, int64_t b) {  // b > 0
  int64_t q = a / b;
  if ((a % b != 0) && (a < 0)) --q;
  return q;
}

// softmax-weighted sum over a key list: keys/values are row pointers.
// out[d] = sum_u p_u v_u, p = softmax(tau q.k_u); returns the natural-log LSE.
double attend(const std::vector<double>& q, const std::vector<const double*>& keys,
              const std::vector<const double*>& vals, int d, double tau, double* out) {
  const size_t n = keys.size();
  for (int c = 0; c < d; ++c) out[c] = 0.0;
  if (n == 0) return -INFINITY;
  std::vector<double> s(n);
  double m = -INFINITY;
  for (size_t u = 0; u < n; ++u) {
    double acc = 0.0;
    for (int c = 0; c < d; ++c) acc += q[c] * keys[u][c];
    s[u] = tau * acc;
    m = std::max(m, s[u]);
  }
  double l = 0.0;
  for (size_t u = 0; u < n; ++u) { s[u] = std::exp(s[u] - m); l += s[u]; }
  for (size_t u = 0; u < n; ++u) {
    const double p = s[u] / l;
    for (int c = 0; c < d; ++c) out[c] += p * vals[u][c];
  }
  return m + std::log(l);
}

// widen a [N][H][d] bf16 tensor to double
template <typename T>
std::vector<double> widen(const T* x, size_t count) {
  std::vector<double> r(count);
  for (size_t i = 0; i < count; ++i) r[i] = bf(x[i]);
  return r;
}

template <typename T>
void mean_pool(const Desc& D, const int32_t* off, const T* x, int32_t H, double* out) {
  const int d = D.head_dim;
  for (int32_t b = 0; b < D.n_blocks; ++b) {
    const int64_t n = (int64_t)off[b + 1] - off[b];
    for (int32_t h = 0; h < H; ++h)
      for (int c = 0; c < d; ++c) {
        double s = 0.0;
        for (int64_t t = off[b]; t < off[b + 1]; ++t) s += bf(x[(t * H + h) * d + c]);
        out[((int64_t)b * H + h) * d + c] = n > 0 ? s / (double)n : 0.0;
      }
  }
}

// the key set of the selected branch for (query block a, index row `row`)
std::vector<int32_t> selected_blocks(const Desc& D, const int32_t* row, int32_t n_forced, const int32_t* forced) {
  std::vector<int32_t> s(forced, forced + n_forced);
  for (int i = 0; i < D.top_k; ++i) s.push_back(row[i]);
  std::sort(s.begin(), s.end());
  s.erase(std::unique(s.begin(), s.end()), s.end());
  return s;
}

// ---- templated statements of each step (T = uint16_t bf16 bits, or double)

// ---- S1: block mean-pool.  out[b][h][c] = (1/n_b) sum_{t in b} x[t][h][c]
template <typename T>
int impl_compress(const Desc* D, const int32_t* off, const T* x, int32_t n_heads, double* out) {
  mean_pool(*D, off, x, n_heads, out);
  return 0;
}

// ---- S2b: geometric routing.  idx [B][k]; centroids [B][3] (int64) optional.
template <typename T>
int impl_route_geometric(const Desc* D, const int32_t* off, const int32_t* coords, int32_t* idx,
                           int64_t* centroids) {
  const int32_t B = D->n_blocks, k = D->top_k;
  std::vector<int64_t> c((size_t)B * 3);
  for (int32_t b = 0; b < B; ++b) {
    const int64_t n = (int64_t)off[b + 1] - off[b];
    for (int a = 0; a < 3; ++a) {
      int64_t S = 0;
      for (int64_t t = off[b]; t < off[b + 1]; ++t) S += coords[t * 3 + a];
      c[(size_t)b * 3 + a] = floor_div(2 * S + n, 2 * n);
    }
  }
  if (centroids) std::memcpy(centroids, c.data(), c.size() * sizeof(int64_t));
  std::vector<std::pair<int64_t, int32_t>> key((size_t)B);
  for (int32_t a = 0; a < B; ++a) {
    for (int32_t j = 0; j < B; ++j) {
      int64_t dist = 0;
      for (int ax = 0; ax < 3; ++ax) {
        const int64_t e = c[(size_t)a * 3 + ax] - c[(size_t)j * 3 + ax];
        dist += e * e;
      }
      key[(size_t)j] = {dist, j};
    }
    std::sort(key.begin(), key.end());
    for (int i = 0; i < k; ++i) idx[(int64_t)a * k + i] = key[(size_t)i].second;
  }
  return 0;
}

// ---- S2a: score routing for the listed query blocks.
// kc: [B][Hkv][d] compressed keys (double).  idx out [nq][Hkv][k]; score out [nq][Hkv][B] (optional).
template <typename T>
int impl_route_score(const Desc* D, const int32_t* off, const T* q, const double* kc,
                       int32_t n_qb, const int32_t* qblocks, int32_t* idx, double* score) {
  const int32_t B = D->n_blocks, Hq = D->n_q_heads, Hkv = D->n_kv_heads, d = D->head_dim, k = D->top_k;
  const int32_t G = Hq / Hkv;
  const double tau = tau_of(*D);
  std::vector<double> sc((size_t)Hkv * B), s((size_t)B);
  std::vector<std::pair<double, int32_t>> key;
  for (int32_t qi = 0; qi < n_qb; ++qi) {
    const int32_t a = qblocks[qi];
    std::fill(sc.begin(), sc.end(), 0.0);
    for (int64_t t = off[a]; t < off[a + 1]; ++t)
      for (int32_t h = 0; h < Hq; ++h) {
        const int32_t g = h / G;
        double m = -INFINITY;
        for (int32_t j = 0; j < B; ++j) {
          double acc = 0.0;
          for (int c = 0; c < d; ++c) acc += bf(q[(t * Hq + h) * d + c]) * kc[((size_t)j * Hkv + g) * d + c];
          s[(size_t)j] = tau * acc;
          m = std::max(m, s[(size_t)j]);
        }
        double l = 0.0;
        for (int32_t j = 0; j < B; ++j) { s[(size_t)j] = std::exp(s[(size_t)j] - m); l += s[(size_t)j]; }
        for (int32_t j = 0; j < B; ++j) sc[(size_t)g * B + j] += s[(size_t)j] / l;
      }
    for (int32_t g = 0; g < Hkv; ++g) {
      key.resize((size_t)B);
      for (int32_t j = 0; j < B; ++j) key[(size_t)j] = {-sc[(size_t)g * B + j], j};
      std::sort(key.begin(), key.end());
      for (int i = 0; i < k; ++i) idx[((int64_t)qi * Hkv + g) * k + i] = key[(size_t)i].second;
      if (score) std::memcpy(score + ((int64_t)qi * Hkv + g) * B, sc.data() + (size_t)g * B, sizeof(double) * B);
    }
  }
  return 0;
}

// ---- Speed3R routing: per (a, h) top-k by tau*Qbar[a,h].Kbar[j,h] over non-forced j.
// qc [B][H][d], kc [B][H][d]; idx out [nq][H][k]; logits out [nq][H][B] optional.
template <typename T>
int impl_route_pooled(const Desc* D, const double* qc, const double* kc, int32_t n_forced,
                        const int32_t* forced, int32_t n_qb, const int32_t* qblocks, int32_t* idx,
                        double* logits) {
  const int32_t B = D->n_blocks, H = D->n_q_heads, d = D->head_dim, k = D->top_k;
  const double tau = tau_of(*D);
  std::vector<char> is_forced((size_t)B, 0);
  for (int32_t i = 0; i < n_forced; ++i) is_forced[(size_t)forced[i]] = 1;
  std::vector<std::pair<double, int32_t>> key;
  for (int32_t qi = 0; qi < n_qb; ++qi) {
    const int32_t a = qblocks[qi];
    for (int32_t h = 0; h < H; ++h) {
      key.clear();
      for (int32_t j = 0; j < B; ++j) {
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += qc[((size_t)a * H + h) * d + c] * kc[((size_t)j * H + h) * d + c];
        const double lg = tau * acc;
        if (logits) logits[((int64_t)qi * H + h) * B + j] = lg;
        if (!is_forced[(size_t)j]) key.push_back({-lg, j});
      }
      std::sort(key.begin(), key.end());
      for (int i = 0; i < k; ++i)
        idx[((int64_t)qi * H + h) * k + i] = i < (int)key.size() ? key[(size_t)i].second : -1;
    }
  }
  return 0;
}

// ---- S3: compressed branch for the listed query blocks.  o [tokens of listed blocks][Hq][d]
// (compacted in list order), lse [..][Hq] (natural log).  kc, vc: [B][Hkv][d];
// qc: [B][Hq][d] block-mean queries (used when pooled_q = 1).
template <typename T>
int impl_cmp_attn(const Desc* D, const int32_t* off, const T* q, const double* kc, const double* vc,
                    const double* qc, int32_t n_qb, const int32_t* qblocks, double* o, double* lse) {
  const int32_t B = D->n_blocks, Hq = D->n_q_heads, Hkv = D->n_kv_heads, d = D->head_dim;
  const int32_t G = Hq / Hkv;
  const double tau = tau_of(*D);
  std::vector<const double*> keys((size_t)B), vals((size_t)B);
  std::vector<double> qv((size_t)d);
  int64_t row = 0;
  for (int32_t qi = 0; qi < n_qb; ++qi) {
    const int32_t a = qblocks[qi];
    const int64_t row0 = row;
    for (int64_t t = off[a]; t < off[a + 1]; ++t, ++row)
      for (int32_t h = 0; h < Hq; ++h) {
        if (D->pooled_q && t > off[a]) {
          // pooled query: every token of the block receives the block's output
          for (int c = 0; c < d; ++c) o[(row * Hq + h) * d + c] = o[(row0 * Hq + h) * d + c];
          if (lse) lse[row * Hq + h] = lse[row0 * Hq + h];
          continue;
        }
        const int32_t g = h / G;
        for (int32_t j = 0; j < B; ++j) {
          keys[(size_t)j] = kc + ((size_t)j * Hkv + g) * d;
          vals[(size_t)j] = vc + ((size_t)j * Hkv + g) * d;
        }
        for (int c = 0; c < d; ++c)
          qv[(size_t)c] = D->pooled_q ? qc[((size_t)a * Hq + h) * d + c] : bf(q[(t * Hq + h) * d + c]);
        const double L = attend(qv, keys, vals, d, tau, o + (row * Hq + h) * d);
        if (lse) lse[row * Hq + h] = L;
      }
  }
  return 0;
}

// ---- S4: selected branch.  idx rows: [B][idx_heads][k] with idx_heads in {1, Hkv};
// group g reads row (idx_heads == 1 ? 0 : g).  Forced blocks join every key set.
template <typename T>
int impl_select_attn(const Desc* D, const int32_t* off, const T* q, const T* k,
                       const T* v, const int32_t* idx, int32_t idx_heads, int32_t n_forced,
                       const int32_t* forced, int32_t n_qb, const int32_t* qblocks, double* o, double* lse) {
  const int32_t Hq = D->n_q_heads, Hkv = D->n_kv_heads, d = D->head_dim, K = D->top_k;
  const int32_t G = Hq / Hkv;
  const double tau = tau_of(*D);
  std::vector<double> qv((size_t)d);
  int64_t row = 0;
  for (int32_t qi = 0; qi < n_qb; ++qi) {
    const int32_t a = qblocks[qi];
    // widen the key/value rows of each group's selected set once per query block
    std::vector<std::vector<double>> kw((size_t)Hkv), vw((size_t)Hkv);
    for (int32_t g = 0; g < Hkv; ++g) {
      const int32_t* r = idx + ((int64_t)a * idx_heads + (idx_heads == 1 ? 0 : g)) * K;
      for (int32_t j : selected_blocks(*D, r, n_forced, forced))
        for (int64_t u = off[j]; u < off[j + 1]; ++u)
          for (int c = 0; c < d; ++c) {
            kw[(size_t)g].push_back(bf(k[(u * Hkv + g) * d + c]));
            vw[(size_t)g].push_back(bf(v[(u * Hkv + g) * d + c]));
          }
    }
    for (int64_t t = off[a]; t < off[a + 1]; ++t, ++row)
      for (int32_t h = 0; h < Hq; ++h) {
        const int32_t g = h / G;
        const size_t nk = kw[(size_t)g].size() / (size_t)d;
        std::vector<const double*> keys(nk), vals(nk);
        for (size_t u = 0; u < nk; ++u) { keys[u] = &kw[(size_t)g][u * d]; vals[u] = &vw[(size_t)g][u * d]; }
        for (int c = 0; c < d; ++c) qv[(size_t)c] = bf(q[(t * Hq + h) * d + c]);
        const double L = attend(qv, keys, vals, d, tau, o + (row * Hq + h) * d);
        if (lse) lse[row * Hq + h] = L;
      }
  }
  return 0;
}

// ---- S5: window branch, in-block band.
template <typename T>
int impl_window_attn(const Desc* D, const int32_t* off, const T* q, const T* k,
                       const T* v, int32_t n_qb, const int32_t* qblocks, double* o, double* lse) {
  const int32_t Hq = D->n_q_heads, Hkv = D->n_kv_heads, d = D->head_dim, w = D->window;
  const int32_t G = Hq / Hkv;
  const double tau = tau_of(*D);
  std::vector<double> qv((size_t)d);
  int64_t row = 0;
  for (int32_t qi = 0; qi < n_qb; ++qi) {
    const int32_t a = qblocks[qi];
    const int64_t n = (int64_t)off[a + 1] - off[a];
    std::vector<double> kw((size_t)(n * Hkv * d)), vw((size_t)(n * Hkv * d));
    for (int64_t r = 0; r < n; ++r)
      for (int32_t g = 0; g < Hkv; ++g)
        for (int c = 0; c < d; ++c) {
          kw[(size_t)((r * Hkv + g) * d + c)] = bf(k[((off[a] + r) * Hkv + g) * d + c]);
          vw[(size_t)((r * Hkv + g) * d + c)] = bf(v[((off[a] + r) * Hkv + g) * d + c]);
        }
    for (int64_t r = 0; r < n; ++r, ++row)
      for (int32_t h = 0; h < Hq; ++h) {
        const int32_t g = h / G;
        std::vector<const double*> keys, vals;
        if (w > 0)
          for (int64_t u = 0; u < n; ++u)
            if (u >= r - w / 2 && u <= r + w / 2 - 1) {
              keys.push_back(&kw[(size_t)((u * Hkv + g) * d)]);
              vals.push_back(&vw[(size_t)((u * Hkv + g) * d)]);
            }
        for (int c = 0; c < d; ++c) qv[(size_t)c] = bf(q[((off[a] + r) * Hq + h) * d + c]);
        const double L = attend(qv, keys, vals, d, tau, o + (row * Hq + h) * d);
        if (lse) lse[row * Hq + h] = L;
      }
  }
  return 0;
}

// ---- S6 + S7: the layer output for the listed query blocks:
//   O = g_cmp o_cmp + g_slc o_slc (+ g_win o_win).
// branches (optional): [rows][Hq][n_gates][d]; lse (optional): [rows][Hq][n_gates].
template <typename T>
int impl_forward(const Desc* D, const int32_t* off, const T* q, const T* k, const T* v,
                   const T* gates, const int32_t* idx, int32_t idx_heads, int32_t n_forced,
                   const int32_t* forced, int32_t n_qb, const int32_t* qblocks, double* out, double* branches,
                   double* lse) {
  const int32_t B = D->n_blocks, Hq = D->n_q_heads, Hkv = D->n_kv_heads, d = D->head_dim, NG = D->n_gates;
  int64_t rows = 0;
  for (int32_t qi = 0; qi < n_qb; ++qi) rows += (int64_t)off[qblocks[qi] + 1] - off[qblocks[qi]];
  std::vector<double> kc((size_t)B * Hkv * d), vc((size_t)B * Hkv * d), qc;
  mean_pool(*D, off, k, Hkv, kc.data());
  mean_pool(*D, off, v, Hkv, vc.data());
  if (D->pooled_q) { qc.resize((size_t)B * Hq * d); mean_pool(*D, off, q, Hq, qc.data()); }
  std::vector<double> oc((size_t)(rows * Hq * d)), os((size_t)(rows * Hq * d)), ow((size_t)(rows * Hq * d), 0.0);
  std::vector<double> lc((size_t)(rows * Hq)), ls((size_t)(rows * Hq)), lw((size_t)(rows * Hq), -INFINITY);
  impl_cmp_attn<T>(D, off, q, kc.data(), vc.data(), qc.data(), n_qb, qblocks, oc.data(), lc.data());
  impl_select_attn<T>(D, off, q, k, v, idx, idx_heads, n_forced, forced, n_qb, qblocks, os.data(), ls.data());
  if (NG >= 3) impl_window_attn<T>(D, off, q, k, v, n_qb, qblocks, ow.data(), lw.data());
  int64_t row = 0;
  for (int32_t qi = 0; qi < n_qb; ++qi) {
    const int32_t a = qblocks[qi];
    for (int64_t t = off[a]; t < off[a + 1]; ++t, ++row)
      for (int32_t h = 0; h < Hq; ++h) {
        const T* gt = gates + (t * Hq + h) * NG;
        const double* br[3] = {&oc[(size_t)((row * Hq + h) * d)], &os[(size_t)((row * Hq + h) * d)],
                               &ow[(size_t)((row * Hq + h) * d)]};
        const double* lb[3] = {&lc[(size_t)(row * Hq + h)], &ls[(size_t)(row * Hq + h)], &lw[(size_t)(row * Hq + h)]};
        for (int c = 0; c < d; ++c) {
          double acc = 0.0;
          for (int b = 0; b < NG; ++b) acc += bf(gt[b]) * br[b][c];
          out[(row * Hq + h) * d + c] = acc;
        }
        if (branches)
          for (int b = 0; b < NG; ++b)
            for (int c = 0; c < d; ++c) branches[((row * Hq + h) * NG + b) * d + c] = br[b][c];
        if (lse)
          for (int b = 0; b < NG; ++b) lse[(row * Hq + h) * NG + b] = *lb[b];
      }
  }
  return 0;
}

// ---- S10: backward of the LSRM layer (pooled_q = 0) with the routing indices fixed.
// Chain rule through the gated sum, the three softmax attentions and the mean-pool:
//   dgates[t,h,b] = <dO[t,h], o_b[t,h]>,  dO_b = g_b dO,
//   per branch: dV_u += sum_t P[t,u] dO_b[t];  dS[t,u] = P[t,u] (dO_b[t].V_u - dO_b[t].o_b[t]);
//               dQ[t] += tau sum_u dS[t,u] K_u;   dK_u += tau sum_t dS[t,u] Q_t;
//   compressed keys: dK[u] += dKbar[beta(u)] / n_beta(u) (and V likewise).
// Outputs cover all tokens: dq [N][Hq][d], dk, dv [N][Hkv][d], dgates [N][Hq][n_gates].
// nthreads > 1 splits the query blocks across threads; each thread keeps its own
// key-side accumulators, which are summed in thread order.
// With a query-block list (n_qb, qblocks), only those query blocks contribute: dq and dgates of
// their rows are the full gradients, dk and dv hold the listed blocks' contributions alone, and
// the other rows of dq and dgates are left untouched.
template <typename T>
int impl_backward(const Desc* D, const int32_t* off, const T* q, const T* k, const T* v,
                    const T* gates, const int32_t* idx, int32_t idx_heads, const T* dout,
                    double* dq, double* dk, double* dv, double* dgates, int32_t n_qb,
                    const int32_t* qblocks, int32_t nthreads) {
  if (D->pooled_q) return 1;
  const int32_t B = D->n_blocks, Hq = D->n_q_heads, Hkv = D->n_kv_heads, d = D->head_dim, NG = D->n_gates;
  const int32_t G = Hq / Hkv, K = D->top_k, w = D->window;
  const int64_t N = D->n_tokens;
  const double tau = tau_of(*D);
  std::vector<double> kc((size_t)B * Hkv * d), vc((size_t)B * Hkv * d);
  mean_pool(*D, off, k, Hkv, kc.data());
  mean_pool(*D, off, v, Hkv, vc.data());
  const std::vector<double> Kw = widen(k, (size_t)(N * Hkv * d)), Vw = widen(v, (size_t)(N * Hkv * d));
  if (nthreads < 1) nthreads = 1;
  const size_t kv_sz = (size_t)(N * Hkv * d), kvc_sz = (size_t)B * Hkv * d;
  std::vector<std::vector<double>> dK(nthreads, std::vector<double>(kv_sz, 0.0)),
      dV(nthreads, std::vector<double>(kv_sz, 0.0)), dKc(nthreads, std::vector<double>(kvc_sz, 0.0)),
      dVc(nthreads, std::vector<double>(kvc_sz, 0.0));

  auto work = [&](int tid) {
    std::vector<double> qv((size_t)d), go((size_t)d), ob((size_t)d), dqv((size_t)d);
    std::vector<double> s, p;
    const int32_t nq = qblocks ? n_qb : B;
    for (int32_t qi = tid; qi < nq; qi += nthreads) {
      const int32_t a = qblocks ? qblocks[qi] : qi;
      // per group: token ids of the selected set
      std::vector<std::vector<int64_t>> sel((size_t)Hkv);
      for (int32_t g = 0; g < Hkv; ++g) {
        const int32_t* r = idx + ((int64_t)a * idx_heads + (idx_heads == 1 ? 0 : g)) * K;
        for (int32_t j : selected_blocks(*D, r, 0, nullptr))
          for (int64_t u = off[j]; u < off[j + 1]; ++u) sel[(size_t)g].push_back(u);
      }
      const int64_t n_a = (int64_t)off[a + 1] - off[a];
      for (int64_t t = off[a]; t < off[a + 1]; ++t)
        for (int32_t h = 0; h < Hq; ++h) {
          const int32_t g = h / G;
          for (int c = 0; c < d; ++c) { qv[(size_t)c] = bf(q[(t * Hq + h) * d + c]); dqv[(size_t)c] = 0.0; }
          const T* gt = gates + (t * Hq + h) * NG;
          for (int br = 0; br < NG; ++br) {
            // key list of this branch: pointers into widened K/V (or compressed K/V)
            std::vector<const double*> kp, vp;
            std::vector<int64_t> tok;  // token id (or block id for the compressed branch)
            if (br == 0) {
              for (int32_t j = 0; j < B; ++j) {
                kp.push_back(&kc[((size_t)j * Hkv + g) * d]);
                vp.push_back(&vc[((size_t)j * Hkv + g) * d]);
                tok.push_back(j);
              }
            } else if (br == 1) {
              for (int64_t u : sel[(size_t)g]) {
                kp.push_back(&Kw[(size_t)((u * Hkv + g) * d)]);
                vp.push_back(&Vw[(size_t)((u * Hkv + g) * d)]);
                tok.push_back(u);
              }
            } else if (w > 0) {
              const int64_t r = t - off[a];
              for (int64_t ru = 0; ru < n_a; ++ru)
                if (ru >= r - w / 2 && ru <= r + w / 2 - 1) {
                  const int64_t u = off[a] + ru;
                  kp.push_back(&Kw[(size_t)((u * Hkv + g) * d)]);
                  vp.push_back(&Vw[(size_t)((u * Hkv + g) * d)]);
                  tok.push_back(u);
                }
            }
            const size_t n = kp.size();
            if (n == 0) { dgates[(t * Hq + h) * NG + br] = 0.0; continue; }
            s.assign(n, 0.0);
            double m = -INFINITY;
            for (size_t u = 0; u < n; ++u) {
              double acc = 0.0;
              for (int c = 0; c < d; ++c) acc += qv[(size_t)c] * kp[u][c];
              s[u] = tau * acc;
              m = std::max(m, s[u]);
            }
            double l = 0.0;
            for (size_t u = 0; u < n; ++u) { s[u] = std::exp(s[u] - m); l += s[u]; }
            p.assign(n, 0.0);
            for (int c = 0; c < d; ++c) ob[(size_t)c] = 0.0;
            for (size_t u = 0; u < n; ++u) {
              p[u] = s[u] / l;
              for (int c = 0; c < d; ++c) ob[(size_t)c] += p[u] * vp[u][c];
            }
            const double gb = bf(gt[br]);
            double dg = 0.0, Dt = 0.0;
            for (int c = 0; c < d; ++c) {
              const double g_out = bf(dout[(t * Hq + h) * d + c]);
              dg += g_out * ob[(size_t)c];
              go[(size_t)c] = gb * g_out;
              Dt += go[(size_t)c] * ob[(size_t)c];
            }
            dgates[(t * Hq + h) * NG + br] = dg;
            for (size_t u = 0; u < n; ++u) {
              double dp = 0.0;
              for (int c = 0; c < d; ++c) dp += go[(size_t)c] * vp[u][c];
              const double ds = p[u] * (dp - Dt);
              double* dkr;
              double* dvr;
              if (br == 0) {
                dkr = &dKc[tid][((size_t)tok[u] * Hkv + g) * d];
                dvr = &dVc[tid][((size_t)tok[u] * Hkv + g) * d];
              } else {
                dkr = &dK[tid][(size_t)((tok[u] * Hkv + g) * d)];
                dvr = &dV[tid][(size_t)((tok[u] * Hkv + g) * d)];
              }
              for (int c = 0; c < d; ++c) {
                dqv[(size_t)c] += tau * ds * kp[u][c];
                dkr[c] += tau * ds * qv[(size_t)c];
                dvr[c] += p[u] * go[(size_t)c];
              }
            }
          }
          for (int c = 0; c < d; ++c) dq[(t * Hq + h) * d + c] = dqv[(size_t)c];
        }
    }
  };
  if (nthreads == 1) work(0);
  else {
    std::vector<std::thread> th;
    for (int i = 0; i < nthreads; ++i) th.emplace_back(work, i);
    for (auto& x : th) x.join();
  }
  for (size_t i = 0; i < kv_sz; ++i) { dk[i] = 0.0; dv[i] = 0.0; }
  for (int tid = 0; tid < nthreads; ++tid) {
    for (size_t i = 0; i < kv_sz; ++i) { dk[i] += dK[(size_t)tid][i]; dv[i] += dV[(size_t)tid][i]; }
  }
  // mean-pool backward: every token of block b receives dKbar[b] / n_b
  for (int32_t b = 0; b < B; ++b) {
    const int64_t n = (int64_t)off[b + 1] - off[b];
    for (int32_t g = 0; g < Hkv; ++g)
      for (int c = 0; c < d; ++c) {
        double gk = 0.0, gv = 0.0;
        for (int tid = 0; tid < nthreads; ++tid) {
          gk += dKc[(size_t)tid][((size_t)b * Hkv + g) * d + c];
          gv += dVc[(size_t)tid][((size_t)b * Hkv + g) * d + c];
        }
        for (int64_t u = off[b]; u < off[b + 1]; ++u) {
          dk[(u * Hkv + g) * d + c] += gk / (double)n;
          dv[(u * Hkv + g) * d + c] += gv / (double)n;
        }
      }
  }
  return 0;
}

// ---- S9 backward: the Speed3R pooled-query layer (pooled_q = 1, MHA, gates (cmp, slc)) with the
// routing indices fixed (Speed3R page, 2.1: compression, selection and gated aggregation; the
// model trains end to end, so the gradient flows through all of them).  Chain rule:
//   compressed: every token t of block a receives o_blk(a), the softmax attention of the
//     block-mean query Qbar_a = (1/n_a) sum_{t in a} q_t over all block means, so its upstream
//     gradient is Gbar_a = sum_{t in a} g_cmp[t] dO[t];
//     dS_j = P_j (Gbar_a . Vbar_j - Gbar_a . o_blk(a)),
//     dQbar_a = tau sum_j dS_j Kbar_j,  dKbar_j += tau dS_j Qbar_a,  dVbar_j += P_j Gbar_a,
//     and each token t of a receives dQbar_a / n_a;
//   selected: per token as in the LSRM layer, over the tokens of (forced U routed) blocks;
//   dgates[t,h,0] = <dO[t], o_blk(a)>, dgates[t,h,1] = <dO[t], o_slc(t)>;
//   mean-pool of K and V: every token u of block j receives dKbar_j / n_j and dVbar_j / n_j.
// idx [B][H][k].  nthreads > 1 splits the query blocks across threads (own accumulators, summed
// in thread order).
template <typename T>
int impl_backward_pooled(const Desc* D, const int32_t* off, const T* q, const T* k, const T* v, const T* gates,
                         const int32_t* idx, int32_t n_forced, const int32_t* forced, const T* dout, double* dq,
                         double* dk, double* dv, double* dgates, int32_t nthreads) {
  const int32_t B = D->n_blocks, H = D->n_q_heads, d = D->head_dim, NG = D->n_gates, K = D->top_k;
  if (H != D->n_kv_heads || NG != 2) return 1;
  const int64_t N = D->n_tokens;
  const double tau = tau_of(*D);
  std::vector<double> qc((size_t)B * H * d), kc((size_t)B * H * d), vc((size_t)B * H * d);
  mean_pool(*D, off, q, H, qc.data());
  mean_pool(*D, off, k, H, kc.data());
  mean_pool(*D, off, v, H, vc.data());
  const std::vector<double> Kw = widen(k, (size_t)(N * H * d)), Vw = widen(v, (size_t)(N * H * d));
  if (nthreads < 1) nthreads = 1;
  const size_t kv_sz = (size_t)(N * H * d), kvc_sz = (size_t)B * H * d;
  std::vector<std::vector<double>> dK(nthreads, std::vector<double>(kv_sz, 0.0)),
      dV(nthreads, std::vector<double>(kv_sz, 0.0)), dKc(nthreads, std::vector<double>(kvc_sz, 0.0)),
      dVc(nthreads, std::vector<double>(kvc_sz, 0.0));
  auto work = [&](int tid) {
    std::vector<double> qv((size_t)d), go((size_t)d), ob((size_t)d), dqv((size_t)d), gbar((size_t)d);
    std::vector<double> s, p;
    for (int32_t a = tid; a < B; a += nthreads) {
      const int64_t n_a = (int64_t)off[a + 1] - off[a];
      for (int32_t h = 0; h < H; ++h) {
        // ---- compressed branch of block a, head h (pooled query)
        const double* qbar = &qc[((size_t)a * H + h) * d];
        s.assign((size_t)B, 0.0);
        double m = -INFINITY;
        for (int32_t j = 0; j < B; ++j) {
          double acc = 0.0;
          for (int c = 0; c < d; ++c) acc += qbar[c] * kc[((size_t)j * H + h) * d + c];
          s[(size_t)j] = tau * acc;
          m = std::max(m, s[(size_t)j]);
        }
        double l = 0.0;
        for (int32_t j = 0; j < B; ++j) { s[(size_t)j] = std::exp(s[(size_t)j] - m); l += s[(size_t)j]; }
        for (int c = 0; c < d; ++c) { ob[(size_t)c] = 0.0; gbar[(size_t)c] = 0.0; }
        for (int32_t j = 0; j < B; ++j)
          for (int c = 0; c < d; ++c) ob[(size_t)c] += s[(size_t)j] / l * vc[((size_t)j * H + h) * d + c];
        for (int64_t t = off[a]; t < off[a + 1]; ++t) {
          const double gc = bf(gates[(t * H + h) * NG + 0]);
          double dg = 0.0;
          for (int c = 0; c < d; ++c) {
            const double g_out = bf(dout[(t * H + h) * d + c]);
            dg += g_out * ob[(size_t)c];
            gbar[(size_t)c] += gc * g_out;
          }
          dgates[(t * H + h) * NG + 0] = dg;
        }
        double Dt = 0.0;
        for (int c = 0; c < d; ++c) Dt += gbar[(size_t)c] * ob[(size_t)c];
        std::vector<double> dqbar((size_t)d, 0.0);
        for (int32_t j = 0; j < B; ++j) {
          const double pj = s[(size_t)j] / l;
          double dp = 0.0;
          for (int c = 0; c < d; ++c) dp += gbar[(size_t)c] * vc[((size_t)j * H + h) * d + c];
          const double ds = pj * (dp - Dt);
          double* dkr = &dKc[(size_t)tid][((size_t)j * H + h) * d];
          double* dvr = &dVc[(size_t)tid][((size_t)j * H + h) * d];
          for (int c = 0; c < d; ++c) {
            dqbar[(size_t)c] += tau * ds * kc[((size_t)j * H + h) * d + c];
            dkr[c] += tau * ds * qbar[c];
            dvr[c] += pj * gbar[(size_t)c];
          }
        }
        // ---- selected branch of every token of a, head h: forced U routed blocks
        std::vector<int64_t> sel;
        for (int32_t j : selected_blocks(*D, idx + ((int64_t)a * H + h) * K, n_forced, forced))
          for (int64_t u = off[j]; u < off[j + 1]; ++u) sel.push_back(u);
        const size_t n = sel.size();
        for (int64_t t = off[a]; t < off[a + 1]; ++t) {
          for (int c = 0; c < d; ++c) {
            qv[(size_t)c] = bf(q[(t * H + h) * d + c]);
            dqv[(size_t)c] = dqbar[(size_t)c] / (double)n_a;
          }
          if (n == 0) {
            dgates[(t * H + h) * NG + 1] = 0.0;
          } else {
            s.assign(n, 0.0);
            double ms = -INFINITY;
            for (size_t u = 0; u < n; ++u) {
              double acc = 0.0;
              for (int c = 0; c < d; ++c) acc += qv[(size_t)c] * Kw[(size_t)((sel[u] * H + h) * d + c)];
              s[u] = tau * acc;
              ms = std::max(ms, s[u]);
            }
            double ls = 0.0;
            for (size_t u = 0; u < n; ++u) { s[u] = std::exp(s[u] - ms); ls += s[u]; }
            p.assign(n, 0.0);
            for (int c = 0; c < d; ++c) ob[(size_t)c] = 0.0;
            for (size_t u = 0; u < n; ++u) {
              p[u] = s[u] / ls;
              for (int c = 0; c < d; ++c) ob[(size_t)c] += p[u] * Vw[(size_t)((sel[u] * H + h) * d + c)];
            }
            const double gb = bf(gates[(t * H + h) * NG + 1]);
            double dg = 0.0, Ds = 0.0;
            for (int c = 0; c < d; ++c) {
              const double g_out = bf(dout[(t * H + h) * d + c]);
              dg += g_out * ob[(size_t)c];
              go[(size_t)c] = gb * g_out;
              Ds += go[(size_t)c] * ob[(size_t)c];
            }
            dgates[(t * H + h) * NG + 1] = dg;
            for (size_t u = 0; u < n; ++u) {
              const double* ku = &Kw[(size_t)((sel[u] * H + h) * d)];
              const double* vu = &Vw[(size_t)((sel[u] * H + h) * d)];
              double dp = 0.0;
              for (int c = 0; c < d; ++c) dp += go[(size_t)c] * vu[c];
              const double ds = p[u] * (dp - Ds);
              double* dkr = &dK[(size_t)tid][(size_t)((sel[u] * H + h) * d)];
              double* dvr = &dV[(size_t)tid][(size_t)((sel[u] * H + h) * d)];
              for (int c = 0; c < d; ++c) {
                dqv[(size_t)c] += tau * ds * ku[c];
                dkr[c] += tau * ds * qv[(size_t)c];
                dvr[c] += p[u] * go[(size_t)c];
              }
            }
          }
          for (int c = 0; c < d; ++c) dq[(t * H + h) * d + c] = dqv[(size_t)c];
        }
      }
    }
  };
  if (nthreads == 1) work(0);
  else {
    std::vector<std::thread> th;
    for (int i = 0; i < nthreads; ++i) th.emplace_back(work, i);
    for (auto& x : th) x.join();
  }
  for (size_t i = 0; i < kv_sz; ++i) { dk[i] = 0.0; dv[i] = 0.0; }
  for (int tid = 0; tid < nthreads; ++tid)
    for (size_t i = 0; i < kv_sz; ++i) { dk[i] += dK[(size_t)tid][i]; dv[i] += dV[(size_t)tid][i]; }
  for (int32_t b = 0; b < B; ++b) {
    const int64_t n = (int64_t)off[b + 1] - off[b];
    for (int32_t h = 0; h < H; ++h)
      for (int c = 0; c < d; ++c) {
        double gk = 0.0, gv = 0.0;
        for (int tid = 0; tid < nthreads; ++tid) {
          gk += dKc[(size_t)tid][((size_t)b * H + h) * d + c];
          gv += dVc[(size_t)tid][((size_t)b * H + h) * d + c];
        }
        for (int64_t u = off[b]; u < off[b + 1]; ++u) {
          dk[(u * H + h) * d + c] += gk / (double)n;
          dv[(u * H + h) * d + c] += gv / (double)n;
        }
      }
  }
  return 0;
}

// ---- a scalar loss L = sum O * dO for the listed blocks (finite-difference checks of the backward)
template <typename T>
double impl_loss(const Desc* D, const int32_t* off, const T* q, const T* k, const T* v,
                   const T* gates, const int32_t* idx, int32_t idx_heads, const T* dout, int32_t n_forced = 0,
                   const int32_t* forced = nullptr) {
  const int32_t B = D->n_blocks, Hq = D->n_q_heads, d = D->head_dim;
  std::vector<int32_t> all((size_t)B);
  for (int32_t b = 0; b < B; ++b) all[(size_t)b] = b;
  std::vector<double> out((size_t)(D->n_tokens * Hq * d));
  impl_forward<T>(D, off, q, k, v, gates, idx, idx_heads, n_forced, forced, B, all.data(), out.data(), nullptr,
                  nullptr);
  double L = 0.0;
  for (size_t i = 0; i < out.size(); ++i) L += out[i] * bf(dout[i]);
  return L;
}

// ---- f4: decoupled self/cross gated mixture over two token streams (LSRM page, 方法, the
// gated cross-attention equations of the dense transformer blocks):
//   o^x = w^{x-self} CrossAttn(x, x) + w^{x-cross} CrossAttn(x, y),
//   o^y = w^{y-self} CrossAttn(y, y) + w^{y-cross} CrossAttn(y, x).
// Stream x is blocks [0, bx) (tokens [0, off[bx])), stream y blocks [bx, B).  CrossAttn(a, b) is
// softmax attention of a's queries over every token of b (grouped-query heads as elsewhere).
// gates [N][Hq][2] = (w_self, w_cross), inputs like the NSA gates (the Sigmoid(Linear) that makes
// them is trained and out of scope).  An empty stream contributes a zero output (LSE -inf).
// branches (optional): [rows][Hq][2][d] = (self, cross); lse (optional): [rows][Hq][2].
template <typename T>
int impl_mixture(const Desc* D, const int32_t* off, const T* q, const T* k, const T* v, const T* gates, int32_t bx,
                 int32_t n_qb, const int32_t* qblocks, double* out, double* branches, double* lse) {
  const int32_t B = D->n_blocks, Hq = D->n_q_heads, Hkv = D->n_kv_heads, d = D->head_dim;
  if (bx < 0 || bx > B) return 1;
  const int32_t G = Hq / Hkv;
  const double tau = tau_of(*D);
  const int64_t nx = off[bx], N = off[B];
  // the key/value rows of both streams, widened once
  const std::vector<double> kw = widen(k, (size_t)(N * Hkv * d)), vw = widen(v, (size_t)(N * Hkv * d));
  std::vector<double> qv((size_t)d), o2((size_t)(2 * d));
  int64_t row = 0;
  for (int32_t qi = 0; qi < n_qb; ++qi) {
    const int32_t a = qblocks[qi];
    const bool in_x = a < bx;
    // token ranges of the query's own stream and of the other one
    const int64_t self_lo = in_x ? 0 : nx, self_hi = in_x ? nx : N;
    const int64_t cross_lo = in_x ? nx : 0, cross_hi = in_x ? N : nx;
    for (int64_t t = off[a]; t < off[a + 1]; ++t, ++row)
      for (int32_t h = 0; h < Hq; ++h) {
        const int32_t g = h / G;
        for (int c = 0; c < d; ++c) qv[(size_t)c] = bf(q[(t * Hq + h) * d + c]);
        double L[2];
        for (int s = 0; s < 2; ++s) {
          const int64_t lo = s == 0 ? self_lo : cross_lo, hi = s == 0 ? self_hi : cross_hi;
          std::vector<const double*> keys, vals;
          for (int64_t u = lo; u < hi; ++u) {
            keys.push_back(&kw[(size_t)((u * Hkv + g) * d)]);
            vals.push_back(&vw[(size_t)((u * Hkv + g) * d)]);
          }
          L[s] = attend(qv, keys, vals, d, tau, &o2[(size_t)(s * d)]);
        }
        const T* w = gates + (t * Hq + h) * 2;
        for (int c = 0; c < d; ++c)
          out[(row * Hq + h) * d + c] = bf(w[0]) * o2[(size_t)c] + bf(w[1]) * o2[(size_t)(d + c)];
        if (branches)
          for (int s = 0; s < 2; ++s)
            for (int c = 0; c < d; ++c) branches[((row * Hq + h) * 2 + s) * d + c] = o2[(size_t)(s * d + c)];
        if (lse)
          for (int s = 0; s < 2; ++s) lse[(row * Hq + h) * 2 + s] = L[s];
      }
  }
  return 0;
}

// ---- f2: camera-projection routing (LSRM page, 方法, 3D-aware routing paragraph).  Each token
// has a 3D point; the query point of block a is its centroid (as in S2b).
//   volume part: the k_vol volume blocks (ids [0, n_vol)) nearest by centroid distance, as S2b;
//   image part: the query point is projected into every view by that view's camera,
//     h = P_v [c; 1] (int64), pixel = (floor(h0 / h2), floor(h1 / h2)) when h2 > 0 (in front of
//     the camera; views behind it give nothing), tile = floor(pixel / tile_px); the image blocks
//     of the tiles within Chebyshev distance `radius` of that tile in the view's tile grid
//     (tile_block[v][ty][tx], -1 = no block) are the candidates, ranked by the smallest squared
//     distance from any of their tokens to the query point, ties to the lower block id; the
//     k_img best are kept.  Should fewer than k_img candidates exist, the other image blocks
//     fill the list by centroid distance (ties to the lower id).
// idx [B][k_vol + k_img]: the volume part in rank order, then the image part.
int impl_route_camera(const Desc* D, const int32_t* off, const int32_t* coords, int32_t n_vol, int32_t n_views,
                      const int32_t* proj, int32_t tiles_x, int32_t tiles_y, int32_t tile_px,
                      const int32_t* tile_block, int32_t radius, int32_t k_vol, int32_t k_img, int32_t* idx) {
  const int32_t B = D->n_blocks;
  if (n_vol < k_vol || B - n_vol < k_img || tile_px < 1 || radius < 0) return 1;
  std::vector<int64_t> c((size_t)B * 3);
  for (int32_t b = 0; b < B; ++b) {
    const int64_t n = (int64_t)off[b + 1] - off[b];
    for (int a = 0; a < 3; ++a) {
      int64_t S = 0;
      for (int64_t t = off[b]; t < off[b + 1]; ++t) S += coords[t * 3 + a];
      c[(size_t)b * 3 + a] = floor_div(2 * S + n, 2 * n);
    }
  }
  auto dist2 = [](const int64_t* p, const int64_t* q) {
    int64_t s = 0;
    for (int a = 0; a < 3; ++a) s += (p[a] - q[a]) * (p[a] - q[a]);
    return s;
  };
  const int32_t K = k_vol + k_img;
  for (int32_t a = 0; a < B; ++a) {
    const int64_t* qa = &c[(size_t)a * 3];
    std::vector<std::pair<int64_t, int32_t>> vol;
    for (int32_t j = 0; j < n_vol; ++j) vol.push_back({dist2(qa, &c[(size_t)j * 3]), j});
    std::sort(vol.begin(), vol.end());
    for (int32_t i = 0; i < k_vol; ++i) idx[(int64_t)a * K + i] = vol[(size_t)i].second;
    // candidates from every view's tile neighbourhood
    std::vector<int32_t> cand;
    for (int32_t v = 0; v < n_views; ++v) {
      int64_t h[3];
      for (int r = 0; r < 3; ++r) {
        const int32_t* P = proj + ((int64_t)v * 3 + r) * 4;
        h[r] = (int64_t)P[0] * qa[0] + (int64_t)P[1] * qa[1] + (int64_t)P[2] * qa[2] + (int64_t)P[3];
      }
      if (h[2] <= 0) continue;
      const int64_t tx = floor_div(floor_div(h[0], h[2]), tile_px), ty = floor_div(floor_div(h[1], h[2]), tile_px);
      for (int64_t y = ty - radius; y <= ty + radius; ++y)
        for (int64_t x = tx - radius; x <= tx + radius; ++x) {
          if (x < 0 || y < 0 || x >= tiles_x || y >= tiles_y) continue;
          const int32_t b = tile_block[((int64_t)v * tiles_y + y) * tiles_x + x];
          if (b >= 0) cand.push_back(b);
        }
    }
    std::sort(cand.begin(), cand.end());
    cand.erase(std::unique(cand.begin(), cand.end()), cand.end());
    std::vector<std::pair<int64_t, int32_t>> img;
    for (int32_t b : cand) {
      int64_t best = INT64_MAX;
      for (int64_t t = off[b]; t < off[b + 1]; ++t) {
        const int64_t p[3] = {coords[t * 3], coords[t * 3 + 1], coords[t * 3 + 2]};
        best = std::min(best, dist2(qa, p));
      }
      img.push_back({best, b});
    }
    std::sort(img.begin(), img.end());
    int32_t n = 0;
    for (; n < k_img && n < (int32_t)img.size(); ++n) idx[(int64_t)a * K + k_vol + n] = img[(size_t)n].second;
    if (n < k_img) {
      std::vector<std::pair<int64_t, int32_t>> fill;
      for (int32_t j = n_vol; j < B; ++j)
        if (!std::binary_search(cand.begin(), cand.end(), j)) fill.push_back({dist2(qa, &c[(size_t)j * 3]), j});
      std::sort(fill.begin(), fill.end());
      for (size_t i = 0; n < k_img; ++n, ++i) idx[(int64_t)a * K + k_vol + n] = fill[i].second;
    }
  }
  return 0;
}

}  // namespace

// ------------------------------------------------------------------------------------------
// C entry points.  "_bf16" functions take bf16 bit patterns (uint16); "_f64" functions take
// doubles (used to perturb inputs by tiny steps for finite differences).
// ------------------------------------------------------------------------------------------
extern "C" {

int oracle_compress(const Desc* D, const int32_t* off, const uint16_t* x, int32_t n_heads, double* out) {
  return impl_compress<uint16_t>(D, off, x, n_heads, out);
}
int oracle_compress_f64(const Desc* D, const int32_t* off, const double* x, int32_t n_heads, double* out) {
  return impl_compress<double>(D, off, x, n_heads, out);
}
int oracle_route_geometric(const Desc* D, const int32_t* off, const int32_t* coords, int32_t* idx,
                           int64_t* centroids) {
  return impl_route_geometric<uint16_t>(D, off, coords, idx, centroids);
}
int oracle_route_score(const Desc* D, const int32_t* off, const uint16_t* q, const double* kc, int32_t n_qb,
                       const int32_t* qblocks, int32_t* idx, double* score) {
  return impl_route_score<uint16_t>(D, off, q, kc, n_qb, qblocks, idx, score);
}
int oracle_route_pooled(const Desc* D, const double* qc, const double* kc, int32_t n_forced, const int32_t* forced,
                        int32_t n_qb, const int32_t* qblocks, int32_t* idx, double* logits) {
  return impl_route_pooled<uint16_t>(D, qc, kc, n_forced, forced, n_qb, qblocks, idx, logits);
}
int oracle_cmp_attn(const Desc* D, const int32_t* off, const uint16_t* q, const double* kc, const double* vc,
                    const double* qc, int32_t n_qb, const int32_t* qblocks, double* o, double* lse) {
  return impl_cmp_attn<uint16_t>(D, off, q, kc, vc, qc, n_qb, qblocks, o, lse);
}
int oracle_select_attn(const Desc* D, const int32_t* off, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                       const int32_t* idx, int32_t idx_heads, int32_t n_forced, const int32_t* forced, int32_t n_qb,
                       const int32_t* qblocks, double* o, double* lse) {
  return impl_select_attn<uint16_t>(D, off, q, k, v, idx, idx_heads, n_forced, forced, n_qb, qblocks, o, lse);
}
int oracle_window_attn(const Desc* D, const int32_t* off, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                       int32_t n_qb, const int32_t* qblocks, double* o, double* lse) {
  return impl_window_attn<uint16_t>(D, off, q, k, v, n_qb, qblocks, o, lse);
}
int oracle_forward(const Desc* D, const int32_t* off, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                   const uint16_t* gates, const int32_t* idx, int32_t idx_heads, int32_t n_forced,
                   const int32_t* forced, int32_t n_qb, const int32_t* qblocks, double* out, double* branches,
                   double* lse) {
  return impl_forward<uint16_t>(D, off, q, k, v, gates, idx, idx_heads, n_forced, forced, n_qb, qblocks, out,
                                branches, lse);
}
int oracle_forward_f64(const Desc* D, const int32_t* off, const double* q, const double* k, const double* v,
                       const double* gates, const int32_t* idx, int32_t idx_heads, int32_t n_forced,
                       const int32_t* forced, int32_t n_qb, const int32_t* qblocks, double* out, double* branches,
                       double* lse) {
  return impl_forward<double>(D, off, q, k, v, gates, idx, idx_heads, n_forced, forced, n_qb, qblocks, out,
                              branches, lse);
}
int oracle_backward(const Desc* D, const int32_t* off, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                    const uint16_t* gates, const int32_t* idx, int32_t idx_heads, const uint16_t* dout, double* dq,
                    double* dk, double* dv, double* dgates, int32_t n_qb, const int32_t* qblocks,
                    int32_t nthreads) {
  return impl_backward<uint16_t>(D, off, q, k, v, gates, idx, idx_heads, dout, dq, dk, dv, dgates, n_qb, qblocks,
                                 nthreads);
}
int oracle_backward_f64(const Desc* D, const int32_t* off, const double* q, const double* k, const double* v,
                        const double* gates, const int32_t* idx, int32_t idx_heads, const double* dout, double* dq,
                        double* dk, double* dv, double* dgates, int32_t n_qb, const int32_t* qblocks,
                        int32_t nthreads) {
  return impl_backward<double>(D, off, q, k, v, gates, idx, idx_heads, dout, dq, dk, dv, dgates, n_qb, qblocks,
                               nthreads);
}
double oracle_loss_f64(const Desc* D, const int32_t* off, const double* q, const double* k, const double* v,
                       const double* gates, const int32_t* idx, int32_t idx_heads, const double* dout) {
  return impl_loss<double>(D, off, q, k, v, gates, idx, idx_heads, dout);
}
double oracle_loss_forced_f64(const Desc* D, const int32_t* off, const double* q, const double* k, const double* v,
                              const double* gates, const int32_t* idx, int32_t idx_heads, const double* dout,
                              int32_t n_forced, const int32_t* forced) {
  return impl_loss<double>(D, off, q, k, v, gates, idx, idx_heads, dout, n_forced, forced);
}
int oracle_backward_pooled(const Desc* D, const int32_t* off, const uint16_t* q, const uint16_t* k,
                           const uint16_t* v, const uint16_t* gates, const int32_t* idx, int32_t n_forced,
                           const int32_t* forced, const uint16_t* dout, double* dq, double* dk, double* dv,
                           double* dgates, int32_t nthreads) {
  return impl_backward_pooled<uint16_t>(D, off, q, k, v, gates, idx, n_forced, forced, dout, dq, dk, dv, dgates,
                                        nthreads);
}
int oracle_backward_pooled_f64(const Desc* D, const int32_t* off, const double* q, const double* k,
                               const double* v, const double* gates, const int32_t* idx, int32_t n_forced,
                               const int32_t* forced, const double* dout, double* dq, double* dk, double* dv,
                               double* dgates, int32_t nthreads) {
  return impl_backward_pooled<double>(D, off, q, k, v, gates, idx, n_forced, forced, dout, dq, dk, dv, dgates,
                                      nthreads);
}
int oracle_route_camera(const Desc* D, const int32_t* off, const int32_t* coords, int32_t n_vol, int32_t n_views,
                        const int32_t* proj, int32_t tiles_x, int32_t tiles_y, int32_t tile_px,
                        const int32_t* tile_block, int32_t radius, int32_t k_vol, int32_t k_img, int32_t* idx) {
  return impl_route_camera(D, off, coords, n_vol, n_views, proj, tiles_x, tiles_y, tile_px, tile_block, radius, k_vol,
                           k_img, idx);
}
int oracle_mixture(const Desc* D, const int32_t* off, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                   const uint16_t* gates, int32_t bx, int32_t n_qb, const int32_t* qblocks, double* out,
                   double* branches, double* lse) {
  return impl_mixture<uint16_t>(D, off, q, k, v, gates, bx, n_qb, qblocks, out, branches, lse);
}

}  // extern "C"
