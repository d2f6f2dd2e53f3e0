// S10 backward of the LSRM layer with the routing indices fixed.
//
// L = sum(out * dout) with out = sum_b g_b o_b (LSRM page, gate equations), o_b the softmax
// attention of branch b (compressed block means, selected blocks, in-block window).  With the
// forward's per-branch LSE, P_b = exp(tau q.k - lse_b) and, per branch:
//   dgates_b = <dO, o_b>,  G_b = g_b dO,  Delta_b = <G_b, o_b> = g_b dgates_b,
//   dS = P (G_b V^T - Delta_b),  dQ += tau dS K,  dK += tau dS^T Q,  dV += P^T G_b,
// and the compressed keys/values are block means, so every token of block j receives
// dKbar_j / n_j (and dVbar_j / n_j).
//
// Kernels (tcgen05 MMAs, bf16 operands, fp32 accumulators in tensor memory; every sum in a fixed
// order, no float atomics):
//   bwd_query_tc:  one CTA per (128 query rows, KV group, query block): per branch, pass A sums
//                  dgates_b = sum_u P_u dP_u, pass B accumulates dQ_b = dS K.
//   bwd_kv_tc:     the keys as the M dimension: local (one key block, group: the selected branch
//                  from the query blocks that routed to it, ascending, from inverse routing
//                  lists, then the window branch of its own block) and compressed (128 block
//                  means, group, query split: partial dKbar, dVbar).
//   bwd_finish:    dK = local part + (sum of the splits' dKbar of the token's block) / n_block.
// The key passes compute S^T and dP^T (keys x query rows) directly, so P^T g and dS^T are
// already in the A-operand layout of the dV and dK products.
#include <type_traits>

#include "lsrm_common.cuh"
#include "tc_ptx.cuh"
#include "tma_map.cuh"

namespace lsrm {


struct BwdParams {
  const int32_t* off;
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const uint16_t* kc;     // bf16 block means [B][Hkv][D]
  const uint16_t* vc;
  const uint16_t* gates;  // [N][Hq][NG]
  const int32_t* idx;     // [B][idx_heads][top_k]
  const float* lse;       // [N][Hq][NG] natural log
  const uint16_t* dout;   // [N][Hq][D]
  const uint16_t* obr;    // optional saved branch outputs o_b, bf16 [N][Hq][NG][D]: no pass A
  uint16_t* dq;
  uint16_t* dgates;
  float4* rowc;           // [NG][N][Hq]: lse (log2 units), gate, Delta, token position (int bits)
  float* dk_tok;          // [N][Hkv][D] selected + window part
  float* dv_tok;
  float* dkc_part;        // [splits][B][Hkv][D]
  float* dvc_part;
  const int* inv_start;   // [n_lists + 1]
  const int* inv_list;    // query blocks routed to each key block, ascending per list
  uint16_t* dk;
  uint16_t* dv;
  uint32_t* status;
  long long N;
  int B, Hq, Hkv, G, NG, top_k, idx_heads, window, n_lists;
  int q_tiles;  // 128-row tiles per query block in the query pass (grid x = (a * Hkv + g) * tiles + tile)
  float tau, scale_log2;
};

// ------------------------------------------------------------------------------------------------
// query pass on the tensor cores: per 128-row tile and branch, pass A forms S = Q K^T and
// dP = dO V^T and sums dgates_b = <dO, o_b> = sum_u P_u dP_u in fp32 (P = exp(tau q.k - lse_b),
// normalised by the saved LSE; no P V product is needed); pass B forms dS = P (g_b dP - Delta_b)
// with Delta_b = g_b dgates_b and accumulates dQ_b = dS K.
//   TMEM (256 columns): S [0, 64) | dP [64, 128) | dS as bf16 pairs [128, 160) | dQ_b
//   warp 0 TMA (Q and dO tiles once, then K/V chunks: every branch is streamed twice),
//   warp 1 MMA issuer, warps 2-9 element-wise: two warps per TMEM lane quarter, each taking
//   32 of a chunk's 64 keys (no online softmax here: the LSE is known, so the halves are
//   independent).
// ------------------------------------------------------------------------------------------------
constexpr int kBqtThreads = 320;
constexpr int kBqtMaxSel = 256;

template <int D>
struct BqtCfg {
  static constexpr int kKeys = 64;
  static constexpr int kStages = D == 32 ? 4 : 3;
  static constexpr int kCtasPerSm = D == 32 ? 2 : 1;
  static constexpr int kTmemCols = 256;
  static constexpr int kColS = 0, kColDP = 64, kColP = 128, kColO = 160;
  static constexpr int kRowBytes = D * 2;
  static constexpr uint32_t kLayout = D == 32 ? tc::kLayoutSW64 : tc::kLayoutSW128;
  static constexpr uint32_t kAtomBytes = 8 * kRowBytes;
  static constexpr int kQBytes = 128 * kRowBytes;
  static constexpr int kKVBytes = kKeys * kRowBytes;
  static constexpr uint32_t kIdescNK = tc::idesc_bf16(128, kKeys, false);  // [rows x keys] from K-major B
  static constexpr uint32_t kIdescND = tc::idesc_bf16(128, D, true);       // [rows x D] from MN-major B
  static_assert(kColO + D <= kTmemCols, "tensor memory budget");
};

template <int D>
struct BqtSmem {
  using C = BqtCfg<D>;
  uint8_t q[C::kQBytes];
  uint8_t go[C::kQBytes];  // dO rows of the tile
  uint8_t k[C::kStages][C::kKVBytes];
  uint8_t v[C::kStages][C::kKVBytes];
  float acc[D][128];       // dQ of the tile, column-major
  float xdg[128];          // half 1's partial dgates sum, handed to half 0
  float dgs[128];          // the full sum, handed back
  float dlt[3][2][128];    // with saved branch outputs: Delta_b of each thread's row (its own slot)
  uint64_t q_full, kv_full[C::kStages], kv_empty[C::kStages], s_full, p_full, pv_done, drain;
  uint64_t xfer[4], back[4];  // pass-A end hand-over between the two warps that own 32 rows
  uint32_t tmem_base;
  int abort;
  int n_sel;
  int sel_start[kBqtMaxSel];
  int sel_n[kBqtMaxSel];
};

// chunk sequence of the query pass: per branch, pass A then pass B over the branch's chunks, or
// pass B alone when the forward's branch outputs were saved (two_pass = 0)
struct BqtSeq {
  int n[3];
  int total;
  int two_pass;
  __device__ __forceinline__ void decode(int c, int& br, int& pass, int& local, bool& first, bool& last) const {
    const int m = two_pass ? 2 : 1;
    br = 0;
    while (c >= m * n[br]) { c -= m * n[br]; ++br; }
    pass = two_pass ? (c >= n[br] ? 1 : 0) : 1;
    local = c - (two_pass && pass ? n[br] : 0);
    first = local == 0;
    last = local == n[br] - 1;
  }
};

template <int D>
__global__ void __launch_bounds__(kBqtThreads, BqtCfg<D>::kCtasPerSm)
bwd_query_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap omap,
                    const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                    const __grid_constant__ CUtensorMap kcmap, const __grid_constant__ CUtensorMap vcmap,
                    const BwdParams p) {
  using namespace tc;
  using C = BqtCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  BqtSmem<D>& S = *reinterpret_cast<BqtSmem<D>*>(smem_raw + (((raw + 1023u) & ~1023u) - raw));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // grid (tile, KV group, query block), a block's groups and tiles side by side; past 65535
  // query blocks one-dimensional in the same order, x = (query block * KV groups + group) * tiles + tile
  int tile, g, a;
  if (gridDim.y * gridDim.z > 1) {
    tile = blockIdx.x;
    g = blockIdx.y;
    a = blockIdx.z;
  } else {
    const unsigned bg = blockIdx.x / (unsigned)p.q_tiles;
    tile = (int)(blockIdx.x - bg * (unsigned)p.q_tiles);
    a = (int)(bg / (unsigned)p.Hkv);
    g = (int)(bg - (unsigned)a * (unsigned)p.Hkv);
  }
  const int t0 = p.off[a], n_a = p.off[a + 1] - t0;
  const int rows_total = n_a * p.G;
  if (tile * 128 >= rows_total) return;
  const int tokens_per_tile = 128 / p.G;

  if (threadIdx.x == 0) {
    S.abort = 0;
    int n = 0;
    const int32_t* r = p.idx + ((size_t)a * p.idx_heads + (p.idx_heads == 1 ? 0 : g)) * p.top_k;
    for (int i = 0; i < p.top_k && n < kBqtMaxSel; ++i) {
      const int j = r[i];
      if (j < 0 || j >= p.B) { raise_status(p.status, LSRM_ERR_BOUNDS); continue; }
      int len = p.off[j + 1] - p.off[j];
      if (len > C::kKeys) { raise_status(p.status, LSRM_ERR_BOUNDS); len = C::kKeys; }
      S.sel_start[n] = p.off[j];
      S.sel_n[n] = len;
      ++n;
    }
    S.n_sel = n;
    mbar_init(&S.q_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&S.kv_full[s], 1);
      mbar_init(&S.kv_empty[s], 1);
    }
    mbar_init(&S.s_full, 1);
    mbar_init(&S.p_full, 256);
    mbar_init(&S.pv_done, 1);
    mbar_init(&S.drain, 1);
    for (int q = 0; q < 4; ++q) {
      mbar_init(&S.xfer[q], 32);
      mbar_init(&S.back[q], 32);
    }
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
  BqtSeq seq;
  seq.n[0] = (p.B + C::kKeys - 1) / C::kKeys;
  seq.n[1] = S.n_sel;
  seq.n[2] = (p.NG == 3 && p.window > 0) ? 1 : 0;
  seq.two_pass = p.obr == nullptr ? 1 : 0;
  seq.total = (seq.two_pass ? 2 : 1) * (seq.n[0] + seq.n[1] + seq.n[2]);
  volatile int* abort = &S.abort;
  auto chunk_start = [&](int br, int local, int& start, int& nv) {
    if (br == 0) {
      start = local * C::kKeys;
      nv = min(C::kKeys, p.B - start);
    } else if (br == 1) {
      start = S.sel_start[local];
      nv = S.sel_n[local];
    } else {
      start = t0;
      nv = min(C::kKeys, n_a);
    }
  };

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0 && seq.total > 0) {
      mbar_arrive_expect_tx(&S.q_full, 2 * C::kQBytes);
      tma_load_3d(S.q, &qmap, &S.q_full, 0, g * p.G, t0 + tile * tokens_per_tile);
      tma_load_3d(S.go, &omap, &S.q_full, 0, g * p.G, t0 + tile * tokens_per_tile);
      int issued = 0;
      for (int c = 0; c < seq.total; ++c) {
        const int st = c % C::kStages;
        if (c >= C::kStages && !mbar_wait(&S.kv_empty[st], ((c / C::kStages) + 1) & 1, abort, p.status)) break;
        int br, pass, local, start, nv;
        bool first, last;
        seq.decode(c, br, pass, local, first, last);
        chunk_start(br, local, start, nv);
        mbar_arrive_expect_tx(&S.kv_full[st], 2 * C::kKVBytes);
        tma_load_3d(S.k[st], br == 0 ? &kcmap : &kmap, &S.kv_full[st], 0, g, start);
        tma_load_3d(S.v[st], br == 0 ? &vcmap : &vmap, &S.kv_full[st], 0, g, start);
        issued = c + 1;
      }
      if (*abort) {
        volatile int no_abort = 0;
        mbar_wait(&S.q_full, 0, &no_abort, nullptr);
        for (int c = max(0, issued - C::kStages); c < issued; ++c)
          mbar_wait(&S.kv_full[c % C::kStages], (c / C::kStages) & 1, &no_abort, nullptr);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (seq.total > 0) {  // whole warp; one elected lane issues
      bool ok = mbar_wait_w(&S.q_full, 0, abort, p.status);
      // descriptors computed once; a byte offset moves the start-address field by offset / 16
      const uint64_t qd = smem_desc(smem_u32(S.q), 16, C::kAtomBytes, C::kLayout);
      const uint64_t od = smem_desc(smem_u32(S.go), 16, C::kAtomBytes, C::kLayout);
      const uint64_t kd_k = smem_desc(smem_u32(S.k[0]), 16, C::kAtomBytes, C::kLayout);
      const uint64_t vd_k = smem_desc(smem_u32(S.v[0]), 16, C::kAtomBytes, C::kLayout);
      const uint64_t kd_mn = smem_desc(smem_u32(S.k[0]), C::kKVBytes, C::kAtomBytes, C::kLayout);
      const uint64_t vd_mn = smem_desc(smem_u32(S.v[0]), C::kKVBytes, C::kAtomBytes, C::kLayout);
      constexpr uint32_t kStep = C::kKVBytes >> 4, kRow16 = (16 * C::kRowBytes) >> 4;
      // both passes: S = Q K^T and dP = dO V^T  (both [128 x 64], K-major B); a pass-A chunk's
      // K/V stage is free as soon as these complete
      auto first_stage = [&](int c, int pass) {
        const uint64_t so = (uint64_t)((c % C::kStages) * kStep);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss_w(tmem + C::kColS, qd + 2 * kk, kd_k + so + 2 * kk, C::kIdescNK, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss_w(tmem + C::kColDP, od + 2 * kk, vd_k + so + 2 * kk, C::kIdescNK, kk > 0 ? 1u : 0u);
        mma_commit_w(&S.s_full);
        if (!pass) mma_commit_w(&S.kv_empty[c % C::kStages]);
      };
      // pass B only: dQ_b += dS K  (A from tensor memory, MN-major B)
      auto second_stage = [&](int c, bool first) {
        const uint64_t bd = kd_mn + (uint64_t)((c % C::kStages) * kStep);
#pragma unroll
        for (int kk = 0; kk < C::kKeys / 16; ++kk)
          mma_ts_w(tmem + C::kColO, tmem + C::kColP + kk * 8, bd + kk * kRow16, C::kIdescND,
                 (first && kk == 0) ? 0u : 1u);
        mma_commit_w(&S.pv_done);
        mma_commit_w(&S.kv_empty[c % C::kStages]);
      };
      int prev_pass = 0;
      bool prev_first = false;
      for (int c = 0; ok && c < seq.total; ++c) {
        if (!mbar_wait_w(&S.kv_full[c % C::kStages], (c / C::kStages) & 1, abort, p.status)) { ok = false; break; }
        int br, pass, local;
        bool first, last;
        seq.decode(c, br, pass, local, first, last);
        if (c > 0) {
          // the element-wise warps are done with S, dP and P(c - 1)
          if (!mbar_wait_w(&S.p_full, (c - 1) & 1, abort, p.status)) { ok = false; break; }
        }
        tc_fence_after();
        // S(c) (and dP(c)) go ahead of the P(c - 1) product: they touch other columns, and the
        // element-wise warps wait for that product before they store P(c)
        first_stage(c, pass);
        if (c > 0 && prev_pass) second_stage(c - 1, prev_first);
        prev_pass = pass;
        prev_first = first;
      }
      if (ok && mbar_wait_w(&S.p_full, (seq.total - 1) & 1, abort, p.status)) {
        tc_fence_after();
        if (prev_pass) second_stage(seq.total - 1, prev_first);
      }
      mma_commit_w(&S.drain);
      volatile int no_abort = 0;
      mbar_wait(&S.drain, 0, &no_abort, nullptr);
    }
  } else {
    // ---------------- element-wise warps ----------------
    const int h = (warp - 2) >> 2;        // key half: keys [32 h, 32 h + 32) of every chunk
    const int quarter = warp & 3;         // tensor-memory lane quarter
    const int row = quarter * 32 + lane;
    const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16);
    const int R = tile * 128 + row;
    const bool valid = R < rows_total;
    const int tok_local = R / p.G;
    const size_t orow = (size_t)(t0 + (valid ? tok_local : 0)) * p.Hq + g * p.G + R % p.G;
    const int wlo = tok_local - p.window / 2, whi = tok_local + p.window / 2 - 1;
    const float sc = p.scale_log2;
    float lse2[3] = {0.f, 0.f, 0.f}, gate[3] = {0.f, 0.f, 0.f};
#pragma unroll
    for (int b = 0; b < 3; ++b) {
      if (valid && b < p.NG) {
        lse2[b] = p.lse[orow * p.NG + b] * 1.4426950408889634f;
        gate[b] = bf16_to_f32(p.gates[orow * p.NG + b]);
      }
    }
    float* acc = &S.acc[0][row];
    if (h == 0) {
#pragma unroll
      for (int i = 0; i < D; ++i) acc[i * 128] = 0.f;
      for (int b = 0; b < p.NG; ++b)
        if (seq.n[b] == 0 && valid) {  // a branch without keys has no gradient
          p.dgates[orow * p.NG + b] = 0;
          p.rowc[((size_t)b * p.N + t0 + tok_local) * p.Hq + g * p.G + R % p.G] =
              make_float4(INFINITY, 0.f, 0.f, __int_as_float(tok_local));
        }
    }
    // With the forward's branch outputs saved, dgates_b = <dO, o_b> and Delta_b = g_b dgates_b come
    // straight from them (fp32 dot products over d) and pass A is skipped.
    if (p.obr != nullptr && valid) {
      const uint4* go = reinterpret_cast<const uint4*>(p.dout + orow * D);
#pragma unroll 1
      for (int b = 0; b < p.NG; ++b) {
        if (seq.n[b] == 0) continue;
        const uint4* ob = reinterpret_cast<const uint4*>(p.obr + (orow * p.NG + b) * D);
        float dg = 0.f;
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
          const uint4 x = go[i], y = ob[i];
          const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            dg = fmaf(bf16_to_f32((uint16_t)(xs[e] & 0xffffu)), bf16_to_f32((uint16_t)(ys[e] & 0xffffu)), dg);
            dg = fmaf(bf16_to_f32((uint16_t)(xs[e] >> 16)), bf16_to_f32((uint16_t)(ys[e] >> 16)), dg);
          }
        }
        // constant indices only (selects), so the per-branch arrays stay in registers
        const float gb = b == 0 ? gate[0] : (b == 1 ? gate[1] : gate[2]);
        const float lb = b == 0 ? lse2[0] : (b == 1 ? lse2[1] : lse2[2]);
        const float db = gb * dg;
        S.dlt[b][h][row] = db;  // read back when the branch's chunks start (kept out of registers)
        if (h == 0) {
          p.dgates[orow * p.NG + b] = __bfloat16_as_ushort(__float2bfloat16_rn(dg));
          p.rowc[((size_t)b * p.N + t0 + tok_local) * p.Hq + g * p.G + R % p.G] =
              make_float4(lb, gb, db, __int_as_float(tok_local));
        }
      }
    }
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      const bool w = mbar_wait(bar, parity, abort, p.status);
      return __all_sync(0xffffffffu, w);
    };
    // pv_done completes once per pass-B chunk (its dS K product).  While the k-th pass-B chunk is
    // worked on it has completed k - 1 or k phases: that chunk's S was issued after the product of
    // pass-B chunk k - 2 (or much later than it), and product k needs this chunk's dS
    int pv_seen = 0;
    auto pv_wait_through = [&](int j) -> bool {
      while (pv_seen <= j) {
        if (!wait_all(&S.pv_done, pv_seen & 1)) return false;
        ++pv_seen;
      }
      tc_fence_after();
      return true;
    };
    // Pass A: this half's share of dgates_b = sum_u P_u dP_u over its 32 keys, in fp32.
    // Pass B: dS of its 32 keys as bf16 pairs.  S and dP are read 16 columns at a time, the next
    // quarter's loads issued before the current one is processed.
    int pv_before_store = -1;
    bool pv_ok = true;
    float dg_part = 0.f;
    auto chunk_pass = [&](auto mask_tag, auto pass_tag, int nv, int br, float l2, float gb, float dlt) {
      constexpr bool kMask = decltype(mask_tag)::value;
      constexpr bool kPassB = decltype(pass_tag)::value;
      const float nl2 = -l2, ndlt = -dlt;
      uint32_t sa[16], sb[16], da[16], db[16];
      auto quarter_pass = [&](const uint32_t* sr, const uint32_t* dr, int qd) {
        uint32_t pk[8];
        float dgq[2] = {0.f, 0.f};
        // key pairs: the scale, the dS factor and the products are packed f32x2 operations
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float s0 = __uint_as_float(sr[2 * i]), s1 = __uint_as_float(sr[2 * i + 1]);
          const float d0 = __uint_as_float(dr[2 * i]), d1 = __uint_as_float(dr[2 * i + 1]);
          float x0, x1;
          ffma2(x0, x1, s0, s1, sc, nl2);
          float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
          if constexpr (kMask) {
            const int j = 32 * h + 16 * qd + 2 * i;
            bool kv0 = j < nv, kv1 = j + 1 < nv;
            if (br == 2) {
              kv0 = kv0 && j >= wlo && j <= whi;
              kv1 = kv1 && j + 1 >= wlo && j + 1 <= whi;
            }
            p0 = kv0 ? p0 : 0.f;
            p1 = kv1 ? p1 : 0.f;
          }
          if constexpr (kPassB) {
            float t0, t1, v0, v1;
            ffma2(t0, t1, d0, d1, gb, ndlt);  // g_b dP - Delta
            fmul2(v0, v1, p0, p1, t0, t1);
            pk[i] = pack_bf16x2(v0, v1);
          } else {
            ffma2_acc(dgq[0], dgq[1], p0, p1, d0, d1);
          }
        }
        if constexpr (kPassB) {
          if (qd == 0) pv_ok = pv_wait_through(pv_before_store);
          if (pv_ok) tmem_st8(tbase + C::kColP + 16 * h + 8 * qd, pk);
        } else {
          dg_part += dgq[0] + dgq[1];
        }
      };
      tmem_ld16(tbase + C::kColS + 32 * h, sa);
      tmem_ld16(tbase + C::kColDP + 32 * h, da);
      tmem_ld_wait();
      tmem_ld16(tbase + C::kColS + 32 * h + 16, sb);
      tmem_ld16(tbase + C::kColDP + 32 * h + 16, db);
      quarter_pass(sa, da, 0);
      tmem_ld_wait();
      quarter_pass(sb, db, 1);
    };
    float delta = 0.f;
    int nb = 0;      // pass-B chunks done
    int merges = 0;  // pass-A ends done
    for (int c = 0; c < seq.total; ++c) {
      int br, pass, local, start, nv;
      bool first, last;
      seq.decode(c, br, pass, local, first, last);
      chunk_start(br, local, start, nv);
      if (!wait_all(&S.s_full, c & 1)) break;
      tc_fence_after();
      pv_before_store = nb - 1;  // the dS columns are free once the previous dS K product is done
      if (!pass && first) dg_part = 0.f;
      if (!seq.two_pass && first) delta = valid ? S.dlt[br][h][row] : 0.f;
      const float l2 = br == 0 ? lse2[0] : (br == 1 ? lse2[1] : lse2[2]);
      const float gb = br == 0 ? gate[0] : (br == 1 ? gate[1] : gate[2]);
      const bool need_mask = br == 2 || nv < 32 * (h + 1);
      if (need_mask) {
        if (pass) chunk_pass(std::true_type{}, std::true_type{}, nv, br, l2, gb, delta);
        else chunk_pass(std::true_type{}, std::false_type{}, nv, br, l2, gb, delta);
      } else {
        if (pass) chunk_pass(std::false_type{}, std::true_type{}, nv, br, l2, gb, delta);
        else chunk_pass(std::false_type{}, std::false_type{}, nv, br, l2, gb, delta);
      }
      if (!pv_ok) break;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&S.p_full);
      if (pass) ++nb;
      if (!last) continue;
      if (pass == 0) {
        // dgates_b: the two halves' sums meet (half 1 hands over, half 0 adds and hands back)
        const uint32_t par = merges & 1;
        ++merges;
        float dg;
        if (h == 1) {
          S.xdg[row] = dg_part;
          mbar_arrive(&S.xfer[quarter]);
          if (!wait_all(&S.back[quarter], par)) break;
          dg = S.dgs[row];
        } else {
          if (!wait_all(&S.xfer[quarter], par)) break;
          dg = dg_part + S.xdg[row];
          S.dgs[row] = dg;
          mbar_arrive(&S.back[quarter]);
        }
        delta = gb * dg;
        if (h == 0 && valid) {
          p.dgates[orow * p.NG + br] = __bfloat16_as_ushort(__float2bfloat16_rn(dg));
          p.rowc[((size_t)br * p.N + t0 + tok_local) * p.Hq + g * p.G + R % p.G] =
              make_float4(l2, gb, delta, __int_as_float(tok_local));
        }
      } else {
        if (!pv_wait_through(nb - 1)) break;  // dQ_b is final
        if (h == 0) {
#pragma unroll
          for (int i = 0; i < D / 32; ++i) {
            uint32_t o[32];
            tmem_ld32(tbase + C::kColO + 32 * i, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) acc[(32 * i + e) * 128] = fmaf(p.tau, __uint_as_float(o[e]), acc[(32 * i + e) * 128]);
          }
        }
      }
    }
    if (h == 0 && valid) {
      uint4* dst = reinterpret_cast<uint4*>(p.dq + orow * D);
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

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ------------------------------------------------------------------------------------------------
// key passes on the tensor cores.  The keys are the M dimension: a CTA holds a 128-row key tile
// (128 block means for the compressed branch; one block's <= 64 tokens, padded, for the selected
// and window branches) and streams the query rows that attend to it in chunks of 64:
//   S^T = K Q^T and dP^T = V dO^T  ([128 x 64], K-major operands from shared memory)
//   P^T = exp(tau S^T - lse) per query row, Pg = P^T g, dS^T = P^T (g dP^T - Delta)
//   dV += Pg dO and dK += dS^T Q   ([128 x D], A from tensor memory, MN-major B)
// The per-row constants of each chunk (LSE in log2 units, gate, Delta, token position, written
// by the query pass as one float4 per branch, token and head) arrive by TMA with its Q and dO.
//   compressed: CTA = (128 block means, group, query split), rows = the split's tokens x G heads
//   local:      CTA = (key block j, group), rows = the query blocks that routed to j (ascending,
//               selected branch), then block j itself (window branch)
// TMEM: S^T [0, 64) | dP^T [64, 128) | Pg [128, 160) | dS^T [160, 192) | dV | dK
// ------------------------------------------------------------------------------------------------
constexpr int kKvThreads = 320;

template <int D>
struct KvCfg {
  static constexpr int kRowsPerChunk = 64;
  static constexpr int kStages = 4;
  static constexpr int kTmemCols = D == 32 ? 256 : 512;
  static constexpr int kCtasPerSm = D == 32 ? 2 : 1;
  static constexpr int kColS = 0, kColDP = 64, kColPg = 128, kColDS = 160, kColDV = 192, kColDK = 192 + D;
  static constexpr int kRowBytes = D * 2;
  static constexpr uint32_t kLayout = D == 32 ? tc::kLayoutSW64 : tc::kLayoutSW128;
  static constexpr uint32_t kAtomBytes = 8 * kRowBytes;
  static constexpr int kKeyBytes = 128 * kRowBytes;
  static constexpr int kChunkBytes = kRowsPerChunk * kRowBytes;
  static constexpr uint32_t kIdescNR = tc::idesc_bf16(128, kRowsPerChunk, false);  // [keys x rows]
  static constexpr uint32_t kIdescND = tc::idesc_bf16(128, D, true);               // [keys x D]
  static_assert(kColDK + D <= kTmemCols, "tensor memory budget");
};

template <int D>
struct KvSmem {
  using C = KvCfg<D>;
  uint8_t kt[C::kKeyBytes];  // key tile (K), 128 rows
  uint8_t vt[C::kKeyBytes];  // key tile (V)
  uint8_t q[C::kStages][C::kChunkBytes];
  uint8_t go[C::kStages][C::kChunkBytes];  // dO rows
  float4 rv[C::kStages][64];               // per query row: lse (log2), gate, Delta, token position
  int br[C::kStages];                      // branch of the chunk in each stage
  int nrows[C::kStages];                   // valid rows of the chunk in each stage
  uint64_t key_full, full[C::kStages], empty[C::kStages], s_full, p_full, pv_done, drain;
  uint32_t tmem_base;
  int abort;
  int total;
};

// walks the query-row chunks of a key tile in order
struct KvCursor {
  int e = 0, r0 = 0;  // entry (query block or split), first row of the chunk within it
};

template <int D, bool kLocal>
__global__ void __launch_bounds__(kKvThreads, KvCfg<D>::kCtasPerSm)
bwd_kv_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                 const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap omap,
                 const __grid_constant__ CUtensorMap rmap, const BwdParams p) {
  using namespace tc;
  using C = KvCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  KvSmem<D>& S = *reinterpret_cast<KvSmem<D>*>(smem_raw + (((raw + 1023u) & ~1023u) - raw));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.y;
  // the key tile
  const int j = blockIdx.x;
  const int key0 = kLocal ? p.off[j] : j * 128;
  const int n_keys = kLocal ? min(64, p.off[j + 1] - key0) : min(128, p.B - key0);
  // the query-row entries: one token range (compressed), or the routed query blocks then j itself
  const int split = blockIdx.z;
  const long long t_lo = p.N * split / kBwdSplits, t_hi = p.N * (split + 1) / kBwdSplits;
  int l0 = 0, n_sel_e = 0;
  if (kLocal) {
    const int list = p.idx_heads == 1 ? j : j * p.Hkv + g;
    l0 = p.inv_start[list];
    n_sel_e = p.inv_start[list + 1] - l0;
  }
  const int n_entries = kLocal ? n_sel_e + (p.window > 0 ? 1 : 0) : 1;
  // entry e: branch, first token, rows (tokens x G)
  auto entry = [&](int e, int& br, int& t0a, int& rows) {
    if (!kLocal) {
      br = 0;
      t0a = (int)t_lo;
      rows = (int)(t_hi - t_lo) * p.G;
    } else {
      const int a = e < n_sel_e ? p.inv_list[l0 + e] : j;
      br = e < n_sel_e ? 1 : 2;
      t0a = p.off[a];
      rows = (p.off[a + 1] - t0a) * p.G;
    }
  };
  auto skip_empty = [&](KvCursor& cu) {
    int br, t0a, rows;
    while (cu.e < n_entries) {
      entry(cu.e, br, t0a, rows);
      if (cu.r0 < rows) break;
      ++cu.e;
      cu.r0 = 0;
    }
  };

  if (threadIdx.x == 0) {
    S.abort = 0;
    int total = 0;
    for (int e = 0; e < n_entries; ++e) {
      int br, t0a, rows;
      entry(e, br, t0a, rows);
      total += (rows + C::kRowsPerChunk - 1) / C::kRowsPerChunk;
    }
    S.total = n_keys > 0 ? total : 0;
    mbar_init(&S.key_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    mbar_init(&S.s_full, 1);
    mbar_init(&S.p_full, kLocal ? 128 : 256);  // local tiles have 64 keys: lane quarters 0 and 1
    mbar_init(&S.pv_done, 1);
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
  const int total = S.total;
  volatile int* abort = &S.abort;
  auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
    const bool w = mbar_wait(bar, parity, abort, p.status);
    return __all_sync(0xffffffffu, w);
  };

  if (warp == 0) {
    // ---------------- producer: key tile once, then Q / dO chunks with their row constants ----------------
    if (lane == 0 && total > 0) {
      const int key_rows = kLocal ? 64 : 128;
      mbar_arrive_expect_tx(&S.key_full, 2 * key_rows * C::kRowBytes);
      tma_load_3d(S.kt, &kmap, &S.key_full, 0, g, key0);
      tma_load_3d(S.vt, &vmap, &S.key_full, 0, g, key0);
      KvCursor cu;
      skip_empty(cu);
      int issued = 0;
      for (int c = 0; c < total; ++c) {
        const int st = c % C::kStages;
        if (c >= C::kStages && !mbar_wait(&S.empty[st], ((c / C::kStages) + 1) & 1, abort, p.status)) break;
        int br, t0a, rows;
        entry(cu.e, br, t0a, rows);
        const int t_first = t0a + cu.r0 / p.G;
        S.br[st] = br;
        S.nrows[st] = min(C::kRowsPerChunk, rows - cu.r0);
        mbar_arrive_expect_tx(&S.full[st], 2 * C::kChunkBytes + C::kRowsPerChunk * 16);
        tma_load_3d(S.q[st], &qmap, &S.full[st], 0, g * p.G, t_first);
        tma_load_3d(S.go[st], &omap, &S.full[st], 0, g * p.G, t_first);
        tma_load_3d(S.rv[st], &rmap, &S.full[st], 0, g * p.G, br * p.N + t_first);
        issued = c + 1;
        cu.r0 += C::kRowsPerChunk;
        skip_empty(cu);
      }
      if (*abort) {
        volatile int no_abort = 0;
        mbar_wait(&S.key_full, 0, &no_abort, nullptr);
        for (int c = max(0, issued - C::kStages); c < issued; ++c)
          mbar_wait(&S.full[c % C::kStages], (c / C::kStages) & 1, &no_abort, nullptr);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (total > 0) {  // whole warp; one elected lane issues
      bool ok = mbar_wait_w(&S.key_full, 0, abort, p.status);
      // descriptors computed once; a byte offset moves the start-address field by offset / 16
      const uint64_t ktd = smem_desc(smem_u32(S.kt), 16, C::kAtomBytes, C::kLayout);
      const uint64_t vtd = smem_desc(smem_u32(S.vt), 16, C::kAtomBytes, C::kLayout);
      const uint64_t qd_k = smem_desc(smem_u32(S.q[0]), 16, C::kAtomBytes, C::kLayout);
      const uint64_t od_k = smem_desc(smem_u32(S.go[0]), 16, C::kAtomBytes, C::kLayout);
      const uint64_t qd_mn = smem_desc(smem_u32(S.q[0]), C::kChunkBytes, C::kAtomBytes, C::kLayout);
      const uint64_t od_mn = smem_desc(smem_u32(S.go[0]), C::kChunkBytes, C::kAtomBytes, C::kLayout);
      constexpr uint32_t kStep = C::kChunkBytes >> 4, kRow16 = (16 * C::kRowBytes) >> 4;
      auto first_stage = [&](int c) {
        const uint64_t so = (uint64_t)((c % C::kStages) * kStep);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss_w(tmem + C::kColS, ktd + 2 * kk, qd_k + so + 2 * kk, C::kIdescNR, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss_w(tmem + C::kColDP, vtd + 2 * kk, od_k + so + 2 * kk, C::kIdescNR, kk > 0 ? 1u : 0u);
        mma_commit_w(&S.s_full);
      };
      auto second_stage = [&](int c) {
        const int st = c % C::kStages;
        const uint64_t so = (uint64_t)(st * kStep);
#pragma unroll
        for (int kk = 0; kk < C::kRowsPerChunk / 16; ++kk) {
          const uint32_t acc = (c == 0 && kk == 0) ? 0u : 1u;
          mma_ts_w(tmem + C::kColDV, tmem + C::kColPg + 8 * kk, od_mn + so + kk * kRow16, C::kIdescND, acc);
          mma_ts_w(tmem + C::kColDK, tmem + C::kColDS + 8 * kk, qd_mn + so + kk * kRow16, C::kIdescND, acc);
        }
        mma_commit_w(&S.pv_done);
        mma_commit_w(&S.empty[st]);
      };
      for (int c = 0; ok && c < total; ++c) {
        if (!mbar_wait_w(&S.full[c % C::kStages], (c / C::kStages) & 1, abort, p.status)) { ok = false; break; }
        if (c > 0) {
          if (!mbar_wait_w(&S.p_full, (c - 1) & 1, abort, p.status)) { ok = false; break; }
        }
        tc_fence_after();
        first_stage(c);  // ahead of the products of chunk c - 1 (other columns; see the query pass)
        if (c > 0) second_stage(c - 1);
      }
      if (ok && mbar_wait_w(&S.p_full, (total - 1) & 1, abort, p.status)) {
        tc_fence_after();
        second_stage(total - 1);
      }
      mma_commit_w(&S.drain);
      volatile int no_abort = 0;
      mbar_wait(&S.drain, 0, &no_abort, nullptr);
    }
  } else {
    // ---------------- element-wise warps: one thread per key, 32 of the chunk's 64 rows ----------------
    const int h = (warp - 2) >> 2;  // row half: rows [32 h, 32 h + 32) of every chunk
    const int quarter = warp & 3;
    const int key = quarter * 32 + lane;  // key of the tile = TMEM lane
    const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16);
    const bool active = !kLocal || quarter < 2;
    const float sc = p.scale_log2;
    const int wh = p.window / 2;
    int pv_seen = 0;
    auto pv_wait_through = [&](int jj) -> bool {
      while (pv_seen <= jj) {
        if (!wait_all(&S.pv_done, pv_seen & 1)) return false;
        ++pv_seen;
      }
      tc_fence_after();
      return true;
    };
    int kv_before_store = -1;
    bool kv_ok = true;
    auto chunk_pass = [&](int st, auto window_tag, auto mask_tag) {
      constexpr bool kWindow = decltype(window_tag)::value;
      constexpr bool kMask = decltype(mask_tag)::value;  // rows past the chunk's valid rows
      const int nrows = S.nrows[st];
      uint32_t sa[16], da[16];
      auto quarter_pass = [&](const uint32_t* sr, const uint32_t* dr, int qd) {
        uint32_t pg[8], ds[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float a2[2], b2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int r = 32 * h + 16 * qd + 2 * i + e;
            const float4 rv = S.rv[st][r];
            float pr = fast_exp2(fmaf(__uint_as_float(sr[2 * i + e]), sc, -rv.x));
            if constexpr (kWindow) {
              const int tp = __float_as_int(rv.w);
              pr = (key >= tp - wh && key <= tp + wh - 1) ? pr : 0.f;
            }
            if constexpr (kMask) pr = r < nrows ? pr : 0.f;
            a2[e] = pr * rv.y;
            b2[e] = pr * fmaf(rv.y, __uint_as_float(dr[2 * i + e]), -rv.z);
          }
          pg[i] = pack_bf16x2(a2[0], a2[1]);
          ds[i] = pack_bf16x2(b2[0], b2[1]);
        }
        if (qd == 0) kv_ok = pv_wait_through(kv_before_store);
        if (kv_ok) {
          tmem_st8(tbase + C::kColPg + 16 * h + 8 * qd, pg);
          tmem_st8(tbase + C::kColDS + 16 * h + 8 * qd, ds);
        }
      };
      // one quarter of S and dP in flight at a time: with two, the 64 registers of loads pushed the
      // kernel past its 96-register budget into spills (sequential loads measured 5% faster)
      tmem_ld16(tbase + C::kColS + 32 * h, sa);
      tmem_ld16(tbase + C::kColDP + 32 * h, da);
      tmem_ld_wait();
      quarter_pass(sa, da, 0);
      tmem_ld16(tbase + C::kColS + 32 * h + 16, sa);
      tmem_ld16(tbase + C::kColDP + 32 * h + 16, da);
      tmem_ld_wait();
      quarter_pass(sa, da, 1);
    };
    bool ok = active;
    for (int c = 0; ok && c < total; ++c) {
      if (!wait_all(&S.s_full, c & 1)) { ok = false; break; }
      tc_fence_after();
      kv_before_store = c - 1;  // Pg and dS are free once chunk c - 1's products are done
      const int st = c % C::kStages;
      const bool partial = S.nrows[st] < C::kRowsPerChunk;
      if (kLocal && S.br[st] == 2) {
        if (partial) chunk_pass(st, std::true_type{}, std::true_type{});
        else chunk_pass(st, std::true_type{}, std::false_type{});
      } else {
        if (partial) chunk_pass(st, std::false_type{}, std::true_type{});
        else chunk_pass(st, std::false_type{}, std::false_type{});
      }
      if (!kv_ok) { ok = false; break; }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&S.p_full);
    }
    if (active && h == 0) {
      float* dkp;
      float* dvp;
      size_t rowi;
      if (kLocal) {
        dkp = p.dk_tok;
        dvp = p.dv_tok;
        rowi = ((size_t)(key0 + key) * p.Hkv + g) * D;
      } else {
        dkp = p.dkc_part;
        dvp = p.dvc_part;
        rowi = (((size_t)split * p.B + key0 + key) * p.Hkv + g) * D;
      }
      const bool store = key < n_keys;
      if (total == 0) {
        if (store)
          for (int i = 0; i < D; ++i) {
            dkp[rowi + i] = 0.f;
            dvp[rowi + i] = 0.f;
          }
      } else if (ok && pv_wait_through(total - 1)) {  // warp-uniform: the loads are .sync.aligned
#pragma unroll
        for (int i = 0; i < D / 32; ++i) {
          uint32_t o[32];
          tmem_ld32(tbase + C::kColDK + 32 * i, o);
          tmem_ld_wait();
          if (store) {
            float4* dst = reinterpret_cast<float4*>(dkp + rowi + 32 * i);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_float4(p.tau * __uint_as_float(o[4 * e]), p.tau * __uint_as_float(o[4 * e + 1]),
                                   p.tau * __uint_as_float(o[4 * e + 2]), p.tau * __uint_as_float(o[4 * e + 3]));
          }
          tmem_ld32(tbase + C::kColDV + 32 * i, o);
          tmem_ld_wait();
          if (store) {
            float4* dsv = reinterpret_cast<float4*>(dvp + rowi + 32 * i);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dsv[e] = make_float4(__uint_as_float(o[4 * e]), __uint_as_float(o[4 * e + 1]),
                                   __uint_as_float(o[4 * e + 2]), __uint_as_float(o[4 * e + 3]));
          }
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

// dK = local part + (sum over splits of dKbar of the token's block) / n_block, as bf16
__global__ void bwd_finish_kernel(const BwdParams p, int D) {
  const int b = blockIdx.x;
  const int u0 = p.off[b], n = p.off[b + 1] - u0;
  const int HD = p.Hkv * D;
  const float inv = n > 0 ? 1.f / (float)n : 0.f;
  for (int e = threadIdx.x; e < HD; e += blockDim.x) {
    float sk = 0.f, sv = 0.f;
    for (int s = 0; s < kBwdSplits; ++s) {
      sk += p.dkc_part[((size_t)s * p.B + b) * HD + e];
      sv += p.dvc_part[((size_t)s * p.B + b) * HD + e];
    }
    for (int r = 0; r < n; ++r) {
      const size_t i = (size_t)(u0 + r) * HD + e;
      p.dk[i] = __bfloat16_as_ushort(__float2bfloat16_rn(p.dk_tok[i] + sk * inv));
      p.dv[i] = __bfloat16_as_ushort(__float2bfloat16_rn(p.dv_tok[i] + sv * inv));
    }
  }
}

// ---- inverse routing lists: for each key block (and group), the query blocks that selected it ----
__global__ void inv_count_kernel(const int32_t* __restrict__ idx, int B, int ih, int k, int* count,
                                 uint32_t* status) {
  const long long n = (long long)B * ih * k;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
    const int gg = (int)((e / k) % ih);
    const int j = idx[e];
    if (j < 0 || j >= B) { raise_status(status, LSRM_ERR_BOUNDS); continue; }
    atomicAdd(count + (size_t)j * ih + gg, 1);
  }
}
// exclusive scan of the list counts by one CTA of kScanThreads: each thread scans a contiguous
// slice, the slice totals are scanned in shared memory, then every slice is written
constexpr int kScanThreads = 1024;
__global__ void __launch_bounds__(kScanThreads) inv_scan_kernel(const int* count, int n, int* start) {
  __shared__ int part[kScanThreads];
  const int per = (n + kScanThreads - 1) / kScanThreads;
  const int lo = min(n, threadIdx.x * per), hi = min(n, lo + per);
  int s = 0;
  for (int i = lo; i < hi; ++i) s += count[i];
  part[threadIdx.x] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int i = 0; i < kScanThreads; ++i) { const int c = part[i]; part[i] = acc; acc += c; }
    start[n] = acc;
  }
  __syncthreads();
  int acc = part[threadIdx.x];
  for (int i = lo; i < hi; ++i) { start[i] = acc; acc += count[i]; }
}
__global__ void inv_fill_kernel(const int32_t* __restrict__ idx, int B, int ih, int k, const int* start,
                                int* cursor, int* list) {
  const long long n = (long long)B * ih * k;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
    const int a = (int)(e / ((long long)ih * k)), gg = (int)((e / k) % ih);
    const int j = idx[e];
    if (j < 0 || j >= B) continue;
    const int li = j * ih + gg;
    list[start[li] + atomicAdd(cursor + li, 1)] = a;
  }
}
// sort every list ascending (fixed summation order); lists are short, insertion sort per thread
__global__ void inv_sort_kernel(const int* start, int n_lists, int* list) {
  for (int li = blockIdx.x * blockDim.x + threadIdx.x; li < n_lists; li += gridDim.x * blockDim.x) {
    const int s = start[li], e = start[li + 1];
    for (int i = s + 1; i < e; ++i) {
      const int x = list[i];
      int j = i - 1;
      while (j >= s && list[j] > x) { list[j + 1] = list[j]; --j; }
      list[j + 1] = x;
    }
  }
}

template <int D>
static lsrm_status launch_backward_d(const lsrm_nsa_desc& d, const BwdParams& p, int idx_heads, cudaStream_t s) {
  const int G = p.G;
  const int tiles = (d.max_block_len * G + 127) / 128;
  CUtensorMap qm, om, km, vm, kcm, vcm;
  if (!make_map(&qm, p.q, D, d.n_q_heads, d.n_tokens, G, 128 / G) ||
      !make_map(&om, p.dout, D, d.n_q_heads, d.n_tokens, G, 128 / G) ||
      !make_map(&km, p.k, D, d.n_kv_heads, d.n_tokens, 1, 64) || !make_map(&vm, p.v, D, d.n_kv_heads, d.n_tokens, 1, 64) ||
      !make_map(&kcm, p.kc, D, d.n_kv_heads, d.n_blocks, 1, 64) ||
      !make_map(&vcm, p.vc, D, d.n_kv_heads, d.n_blocks, 1, 64))
    return LSRM_ERR_CUDA;
  size_t sm = sizeof(BqtSmem<D>) + 1024;
  if (cudaFuncSetAttribute(bwd_query_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) !=
      cudaSuccess)
    return LSRM_ERR_CUDA;
  const long long nx = (long long)tiles * d.n_kv_heads * d.n_blocks;
  if (nx > INT32_MAX || d.n_kv_heads > 65535) return LSRM_ERR_UNSUPPORTED;
  BwdParams pq = p;
  pq.q_tiles = tiles;
  const dim3 grid = d.n_blocks <= 65535 ? dim3((unsigned)tiles, (unsigned)d.n_kv_heads, (unsigned)d.n_blocks)
                                        : dim3((unsigned)nx, 1, 1);
  bwd_query_tc_kernel<D><<<grid, kBqtThreads, sm, s>>>(qm, om, km, vm, kcm, vcm, pq);
  CUtensorMap k64, v64, kc128, vc128, q64, o64;
  if (!make_map(&k64, p.k, D, d.n_kv_heads, d.n_tokens, 1, 64) || !make_map(&v64, p.v, D, d.n_kv_heads, d.n_tokens, 1, 64) ||
      !make_map(&kc128, p.kc, D, d.n_kv_heads, d.n_blocks, 1, 128) ||
      !make_map(&vc128, p.vc, D, d.n_kv_heads, d.n_blocks, 1, 128) ||
      !make_map(&q64, p.q, D, d.n_q_heads, d.n_tokens, G, 64 / G) ||
      !make_map(&o64, p.dout, D, d.n_q_heads, d.n_tokens, G, 64 / G))
    return LSRM_ERR_CUDA;
  sm = sizeof(KvSmem<D>) + 1024;
  if (cudaFuncSetAttribute(bwd_kv_tc_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) !=
          cudaSuccess ||
      cudaFuncSetAttribute(bwd_kv_tc_kernel<D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) !=
          cudaSuccess)
    return LSRM_ERR_CUDA;
  CUtensorMap rmap;
  if (!make_map_rows(&rmap, p.rowc, d.n_q_heads, (long long)p.NG * d.n_tokens, G, 64 / G)) return LSRM_ERR_CUDA;
  bwd_kv_tc_kernel<D, true><<<dim3(d.n_blocks, d.n_kv_heads, 1), kKvThreads, sm, s>>>(k64, v64, q64, o64, rmap, p);
  bwd_kv_tc_kernel<D, false><<<dim3((d.n_blocks + 127) / 128, d.n_kv_heads, kBwdSplits), kKvThreads, sm, s>>>(
      kc128, vc128, q64, o64, rmap, p);
  bwd_finish_kernel<<<d.n_blocks, 256, 0, s>>>(p, D);
  (void)idx_heads;
  return cudaGetLastError() == cudaSuccess ? LSRM_OK : LSRM_ERR_CUDA;
}

lsrm_status launch_backward(const lsrm_nsa_desc& d, const int32_t* off, const void* q, const void* k, const void* v,
                            const void* kc, const void* vc, const void* gates, const int32_t* idx, int idx_heads,
                            const float* lse, const void* dout, void* dq, void* dk, void* dv, void* dgates,
                            unsigned char* ws_bwd, uint32_t* status, cudaStream_t s, const void* obr) {
  if (d.top_k > 256 || d.n_gates < 2 || d.n_gates > 3 || d.max_block_len > 64 || 64 % (d.n_q_heads / d.n_kv_heads) != 0)
    return LSRM_ERR_UNSUPPORTED;
  const BwdWs w = bwd_layout(d, idx_heads);
  BwdParams p{};
  p.off = off;
  p.q = (const uint16_t*)q;
  p.k = (const uint16_t*)k;
  p.v = (const uint16_t*)v;
  p.kc = (const uint16_t*)kc;
  p.vc = (const uint16_t*)vc;
  p.gates = (const uint16_t*)gates;
  p.idx = idx;
  p.lse = lse;
  p.dout = (const uint16_t*)dout;
  p.obr = (const uint16_t*)obr;
  p.dq = (uint16_t*)dq;
  p.dgates = (uint16_t*)dgates;
  p.rowc = reinterpret_cast<float4*>(ws_bwd + w.rowc);
  p.dk_tok = reinterpret_cast<float*>(ws_bwd + w.dk_tok);
  p.dv_tok = reinterpret_cast<float*>(ws_bwd + w.dv_tok);
  p.dkc_part = reinterpret_cast<float*>(ws_bwd + w.dkc);
  p.dvc_part = reinterpret_cast<float*>(ws_bwd + w.dvc);
  p.inv_start = reinterpret_cast<const int*>(ws_bwd + w.inv_start);
  p.inv_list = reinterpret_cast<const int*>(ws_bwd + w.inv_list);
  p.dk = (uint16_t*)dk;
  p.dv = (uint16_t*)dv;
  p.status = status;
  p.N = d.n_tokens;
  p.B = d.n_blocks;
  p.Hq = d.n_q_heads;
  p.Hkv = d.n_kv_heads;
  p.G = d.n_q_heads / d.n_kv_heads;
  p.NG = d.n_gates;
  p.top_k = d.top_k;
  p.idx_heads = idx_heads;
  p.window = d.n_gates == 3 ? d.window : 0;
  p.n_lists = d.n_blocks * idx_heads;
  p.tau = d.scale > 0 ? d.scale : 1.0f / sqrtf((float)d.head_dim);
  p.scale_log2 = p.tau * 1.4426950408889634f;
  // inverse routing lists
  int* count = reinterpret_cast<int*>(ws_bwd + w.inv_count);
  int* cursor = reinterpret_cast<int*>(ws_bwd + w.inv_cursor);
  int* start = reinterpret_cast<int*>(ws_bwd + w.inv_start);
  int* list = reinterpret_cast<int*>(ws_bwd + w.inv_list);
  if (cudaMemsetAsync(count, 0, (size_t)p.n_lists * 4, s) != cudaSuccess) return LSRM_ERR_CUDA;
  if (cudaMemsetAsync(cursor, 0, (size_t)p.n_lists * 4, s) != cudaSuccess) return LSRM_ERR_CUDA;
  const int grid = 148 * 4;
  inv_count_kernel<<<grid, 256, 0, s>>>(idx, d.n_blocks, idx_heads, d.top_k, count, status);
  inv_scan_kernel<<<1, kScanThreads, 0, s>>>(count, p.n_lists, start);
  inv_fill_kernel<<<grid, 256, 0, s>>>(idx, d.n_blocks, idx_heads, d.top_k, start, cursor, list);
  inv_sort_kernel<<<(p.n_lists + 127) / 128, 128, 0, s>>>(start, p.n_lists, list);
  if (d.head_dim == 32) return launch_backward_d<32>(d, p, idx_heads, s);
  if (d.head_dim == 64) return launch_backward_d<64>(d, p, idx_heads, s);
  return LSRM_ERR_UNSUPPORTED;
}

}  // namespace lsrm
