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
// Kernels (mma.sync m16n8k16 bf16 -> fp32; every sum in a fixed order, no float atomics):
//   bwd_query:   one CTA per (query block, KV group, 128 rows): o_b recomputed -> dgates, Delta;
//                then dQ from a second pass over each branch's keys.
//   bwd_kv_local: one CTA per (key block, KV group): dK, dV of the block's tokens from the
//                selected branch (query blocks that routed to it, in ascending order, from an
//                inverse routing list) and from the window branch (its own block).
//   bwd_kv_cmp:  one CTA per (64 block means, KV group, query split): partial dKbar, dVbar.
//   bwd_finish:  dK = local part + (sum of the splits' dKbar of the token's block) / n_block.
// The key-side passes compute S^T and dP^T (keys x query rows) directly, so P^T and dS^T are
// already in the A-operand layout of the dV and dK products.
#include <type_traits>

#include "lsrm_common.cuh"
#include "tc_ptx.cuh"
#include "tma_map.cuh"

namespace lsrm {

constexpr int kBkThreads = 128;   // 4 warps x 16 keys

template <int D>
__device__ __forceinline__ uint32_t bswz(int row, int ch) {
  if (D == 32) return (uint32_t)(row * 64 + ((ch ^ ((row >> 1) & 3)) << 4));
  return (uint32_t)(row * 128 + ((ch ^ (row & 7)) << 4));
}

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
  uint16_t* dq;
  uint16_t* dgates;
  float* delta;           // [N][Hq][NG]
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
  float tau, scale_log2;
};

// ------------------------------------------------------------------------------------------------
// query pass on the tensor cores: per 128-row tile and branch, pass A recomputes o_b = P V
// (P = exp(tau q.k - lse_b), normalised by the saved LSE) to get dgates_b and Delta_b; pass B
// forms dS = P (g_b dO V^T - Delta_b) and accumulates dQ_b = dS K.
//   TMEM (256 columns): S [0, 64) | dP [64, 128) | P or dS as bf16 pairs [128, 160) | O or dQ_b
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
  uint64_t q_full, kv_full[C::kStages], kv_empty[C::kStages], s_full, p_full, pv_done, drain;
  uint32_t tmem_base;
  int abort;
  int n_sel;
  int sel_start[kBqtMaxSel];
  int sel_n[kBqtMaxSel];
};

// chunk order: for each branch with keys, its chunks twice (pass A, then pass B)
struct BqtSeq {
  int n[3];
  int total;
  __device__ __forceinline__ void decode(int c, int& br, int& pass, int& local, bool& first, bool& last) const {
    br = 0;
    while (c >= 2 * n[br]) { c -= 2 * n[br]; ++br; }
    pass = c >= n[br];
    local = c - pass * n[br];
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
  const int tile = blockIdx.x, g = blockIdx.y, a = blockIdx.z;
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
  seq.total = 2 * (seq.n[0] + seq.n[1] + seq.n[2]);
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
    if (lane == 0 && seq.total > 0) {
      bool ok = mbar_wait(&S.q_full, 0, abort, p.status);
      const uint32_t qaddr = smem_u32(S.q), oaddr = smem_u32(S.go);
      // pass A: S = Q K^T;  pass B: S = Q K^T and dP = dO V^T  (both [128 x 64], K-major B)
      auto first_stage = [&](int c, int pass) {
        const uint32_t kaddr = smem_u32(S.k[c % C::kStages]), vaddr = smem_u32(S.v[c % C::kStages]);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          mma_ss(tmem + C::kColS, smem_desc(qaddr + kk * 32, 16, C::kAtomBytes, C::kLayout),
                 smem_desc(kaddr + kk * 32, 16, C::kAtomBytes, C::kLayout), C::kIdescNK, kk > 0 ? 1u : 0u);
        }
        if (pass) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            mma_ss(tmem + C::kColDP, smem_desc(oaddr + kk * 32, 16, C::kAtomBytes, C::kLayout),
                   smem_desc(vaddr + kk * 32, 16, C::kAtomBytes, C::kLayout), C::kIdescNK, kk > 0 ? 1u : 0u);
          }
        }
        mma_commit(&S.s_full);
      };
      // pass A: O += P V;  pass B: dQ_b += dS K  (A from tensor memory, MN-major B)
      auto second_stage = [&](int c, int pass, bool first) {
        const uint32_t baddr = smem_u32(pass ? S.k[c % C::kStages] : S.v[c % C::kStages]);
#pragma unroll
        for (int kk = 0; kk < C::kKeys / 16; ++kk) {
          const uint64_t bd = smem_desc(baddr + kk * 16 * C::kRowBytes, C::kKVBytes, C::kAtomBytes, C::kLayout);
          mma_ts(tmem + C::kColO, tmem + C::kColP + kk * 8, bd, C::kIdescND, (first && kk == 0) ? 0u : 1u);
        }
        mma_commit(&S.pv_done);
        mma_commit(&S.kv_empty[c % C::kStages]);
      };
      int prev_pass = 0;
      bool prev_first = false;
      for (int c = 0; ok && c < seq.total; ++c) {
        if (!mbar_wait(&S.kv_full[c % C::kStages], (c / C::kStages) & 1, abort, p.status)) { ok = false; break; }
        int br, pass, local;
        bool first, last;
        seq.decode(c, br, pass, local, first, last);
        if (c > 0) {
          // the element-wise warps are done with S, dP and P(c - 1)
          if (!mbar_wait(&S.p_full, (c - 1) & 1, abort, p.status)) { ok = false; break; }
          tc_fence_after();
          second_stage(c - 1, prev_pass, prev_first);
        }
        tc_fence_after();
        first_stage(c, pass);
        prev_pass = pass;
        prev_first = first;
      }
      if (ok && mbar_wait(&S.p_full, (seq.total - 1) & 1, abort, p.status)) {
        tc_fence_after();
        second_stage(seq.total - 1, prev_pass, prev_first);
      }
      mma_commit(&S.drain);
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
          p.delta[orow * p.NG + b] = 0.f;
        }
    }
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      const bool w = mbar_wait(bar, parity, abort, p.status);
      return __all_sync(0xffffffffu, w);
    };
    // one pv_done phase per chunk; while chunk c is worked on it has completed c - 1 or c phases
    int pv_seen = 0;
    auto pv_wait_through = [&](int j) -> bool {
      while (pv_seen <= j) {
        if (!wait_all(&S.pv_done, pv_seen & 1)) return false;
        ++pv_seen;
      }
      tc_fence_after();
      return true;
    };
    auto swz = [](int r, int ch) -> uint32_t {
      if (D == 32) return (uint32_t)(r * 64 + ((ch ^ ((r >> 1) & 3)) << 4));
      return (uint32_t)(r * 128 + ((ch ^ (r & 7)) << 4));
    };
    // P (pass A) or dS (pass B) of this half's 32 keys as bf16 pairs; S and dP are read 16
    // columns at a time, the next quarter's loads issued before the current one is processed
    auto chunk_pass = [&](auto mask_tag, auto pass_tag, int nv, int br, float l2, float gb, float dlt) {
      constexpr bool kMask = decltype(mask_tag)::value;
      constexpr bool kPassB = decltype(pass_tag)::value;
      uint32_t sa[16], sb[16], da[16], db[16];
      auto quarter_pass = [&](const uint32_t* sr, const uint32_t* dr, int qd) {
        uint32_t pk[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float v2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int j = 32 * h + 16 * qd + 2 * i + e;
            bool kv = true;
            if constexpr (kMask) {
              kv = j < nv;
              if (br == 2) kv = kv && j >= wlo && j <= whi;
            }
            float pr = fast_exp2(fmaf(__uint_as_float(sr[2 * i + e]), sc, -l2));
            if constexpr (kMask) pr = kv ? pr : 0.f;
            if constexpr (kPassB) pr *= fmaf(gb, __uint_as_float(dr[2 * i + e]), -dlt);
            v2[e] = pr;
          }
          pk[i] = pack_bf16x2(v2[0], v2[1]);
        }
        tmem_st8(tbase + C::kColP + 16 * h + 8 * qd, pk);
      };
      tmem_ld16(tbase + C::kColS + 32 * h, sa);
      if constexpr (kPassB) tmem_ld16(tbase + C::kColDP + 32 * h, da);
      tmem_ld_wait();
      tmem_ld16(tbase + C::kColS + 32 * h + 16, sb);
      if constexpr (kPassB) tmem_ld16(tbase + C::kColDP + 32 * h + 16, db);
      quarter_pass(sa, da, 0);
      tmem_ld_wait();
      quarter_pass(sb, db, 1);
    };
    float delta = 0.f;
    for (int c = 0; c < seq.total; ++c) {
      int br, pass, local, start, nv;
      bool first, last;
      seq.decode(c, br, pass, local, first, last);
      chunk_start(br, local, start, nv);
      if (!wait_all(&S.s_full, c & 1)) break;
      tc_fence_after();
      if (!pv_wait_through(c - 1)) break;  // the P / dS columns are free again
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
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&S.p_full);
      if (last) {
        if (!pv_wait_through(c)) break;
        if (pass == 0) {
          // o_b is final: dgates_b = <dO, o_b>, Delta_b = g_b dgates_b
          float dg = 0.f;
#pragma unroll
          for (int i = 0; i < D / 32; ++i) {
            uint32_t o[32];
            tmem_ld32(tbase + C::kColO + 32 * i, o);
            tmem_ld_wait();
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
              const uint4 u = *reinterpret_cast<const uint4*>(S.go + swz(row, 4 * i + ch));
              const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                dg = fmaf(__uint_as_float(w4[e] << 16), __uint_as_float(o[8 * ch + 2 * e]), dg);
                dg = fmaf(__uint_as_float(w4[e] & 0xFFFF0000u), __uint_as_float(o[8 * ch + 2 * e + 1]), dg);
              }
            }
          }
          delta = gb * dg;
          if (h == 0 && valid) {
            p.dgates[orow * p.NG + br] = __bfloat16_as_ushort(__float2bfloat16_rn(dg));
            p.delta[orow * p.NG + br] = delta;
          }
        } else if (h == 0) {
          // dQ_b is final: add tau dQ_b to the tile's dQ
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
// key passes: S^T = K Q^T, dP^T = V G^T for 64 keys (4 warps x 16) against query rows staged
// 64 at a time and consumed in 16-row sub-tiles
// ------------------------------------------------------------------------------------------------
constexpr int kBkRows = 64;

template <int D>
struct BkSmem {
  uint16_t kt[64 * D];
  uint16_t vt[64 * D];
  uint16_t q[kBkRows * D];
  uint16_t g[kBkRows * D];  // G_b = g_b dO rows
  float lse2[kBkRows];      // log2-unit LSE of the rows
  float dlt[kBkRows];
  int tok[kBkRows];         // query token position inside its block (window mask), -1 = invalid row
};

// A fragments of the warp's 16 keys (K and V)
template <int D>
__device__ __forceinline__ void bk_key_frags(const BkSmem<D>& S, int warp, int lane, uint32_t (&ka)[D / 16][4],
                                             uint32_t (&va)[D / 16][4]) {
#pragma unroll
  for (int kt = 0; kt < D / 16; ++kt) {
    const int r = warp * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
    const int ch = kt * 2 + (lane >> 4);
    ldmatrix_x4(ka[kt][0], ka[kt][1], ka[kt][2], ka[kt][3], smem_u32(S.kt) + bswz<D>(r, ch));
    ldmatrix_x4(va[kt][0], va[kt][1], va[kt][2], va[kt][3], smem_u32(S.vt) + bswz<D>(r, ch));
  }
}

// accumulate the staged rows [sub*16, sub*16+16) into the warp's dK / dV (16 keys x D)
template <int D, bool kWindow>
__device__ __forceinline__ void bk_tile(const BkSmem<D>& S, int sub, int lane, int key_valid, const int (&key_pos)[2],
                                        int window, float scale_log2, const uint32_t (&ka)[D / 16][4],
                                        const uint32_t (&va)[D / 16][4], float (&dk)[D / 8][4],
                                        float (&dv)[D / 8][4]) {
  constexpr int KT = D / 16;
  const int gq = lane >> 2, cq = lane & 3;
  const int rb = sub * 16;
  float st[2][4], dpt[2][4];  // [row n-tile][frag]: rows = keys gq, gq+8; cols = query rows 8 n + 2 cq (+1)
#pragma unroll
  for (int n = 0; n < 2; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) { st[n][e] = 0.f; dpt[n][e] = 0.f; }
#pragma unroll
  for (int kt = 0; kt < KT; ++kt) {
    uint32_t b0, b1, b2, b3;
    const int r = rb + (lane >> 4) * 8 + (lane & 7);
    const int ch = kt * 2 + ((lane >> 3) & 1);
    ldmatrix_x4(b0, b1, b2, b3, smem_u32(S.q) + bswz<D>(r, ch));
    const uint32_t q0[2] = {b0, b1}, q1[2] = {b2, b3};
    mma_bf16_16816(st[0], ka[kt], q0);
    mma_bf16_16816(st[1], ka[kt], q1);
    ldmatrix_x4(b0, b1, b2, b3, smem_u32(S.g) + bswz<D>(r, ch));
    const uint32_t g0[2] = {b0, b1}, g1[2] = {b2, b3};
    mma_bf16_16816(dpt[0], va[kt], g0);
    mma_bf16_16816(dpt[1], va[kt], g1);
  }
  // P^T and dS^T (keys x rows), masked
  uint32_t pa[4], da[4];
#pragma unroll
  for (int n = 0; n < 2; ++n) {
    float pv[4], dv4[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int krow = gq + 8 * (e >> 1);             // key of the warp tile
      const int qrow = rb + n * 8 + 2 * cq + (e & 1);  // staged query row
      const int r = S.tok[qrow];
      bool ok = krow < key_valid && r >= 0;
      if (kWindow) {
        const int u = key_pos[e >> 1];
        ok = ok && u >= r - window / 2 && u <= r + window / 2 - 1;
      }
      const float pp = ok ? fast_exp2(st[n][e] * scale_log2 - S.lse2[qrow]) : 0.f;
      pv[e] = pp;
      dv4[e] = pp * (dpt[n][e] - S.dlt[qrow]);
    }
    pa[n * 2 + 0] = pack_bf16x2(pv[0], pv[1]);
    pa[n * 2 + 1] = pack_bf16x2(pv[2], pv[3]);
    da[n * 2 + 0] = pack_bf16x2(dv4[0], dv4[1]);
    da[n * 2 + 1] = pack_bf16x2(dv4[2], dv4[3]);
  }
  // dV += P^T G, dK += dS^T Q (B operands: staged rows of G / Q, transposed loads)
#pragma unroll
  for (int dn = 0; dn < D / 16; ++dn) {
    uint32_t b0, b1, b2, b3;
    const int r = rb + ((lane >> 3) & 1) * 8 + (lane & 7);
    const int ch = dn * 2 + (lane >> 4);
    ldmatrix_x4_trans(b0, b1, b2, b3, smem_u32(S.g) + bswz<D>(r, ch));
    const uint32_t g0[2] = {b0, b1}, g1[2] = {b2, b3};
    mma_bf16_16816(dv[2 * dn], pa, g0);
    mma_bf16_16816(dv[2 * dn + 1], pa, g1);
    ldmatrix_x4_trans(b0, b1, b2, b3, smem_u32(S.q) + bswz<D>(r, ch));
    const uint32_t q0[2] = {b0, b1}, q1[2] = {b2, b3};
    mma_bf16_16816(dk[2 * dn], da, q0);
    mma_bf16_16816(dk[2 * dn + 1], da, q1);
  }
}

// stage kBkRows query rows (row0.. of the token range starting at t_base) of group g for branch br;
// G_b = g_b dO is formed here, rounded to bf16
template <int D>
__device__ __forceinline__ void bk_stage_rows(BkSmem<D>& S, const BwdParams& p, int g, int br, int row0,
                                              int rows_total, long long t_base, int tid) {
  constexpr int CPR = D / 8;
  for (int e = tid; e < kBkRows * CPR; e += kBkThreads) {
    const int r = e / CPR, ch = e % CPR;
    const int rr = row0 + r;
    const bool ok = rr < rows_total;
    const long long t = t_base + (ok ? rr / p.G : 0);
    const int h = g * p.G + (ok ? rr % p.G : 0);
    const size_t src = ((size_t)t * p.Hq + h) * D + ch * 8;
    cp_async16(reinterpret_cast<unsigned char*>(S.q) + bswz<D>(r, ch), p.q + src, ok);
    uint4 u = make_uint4(0, 0, 0, 0);
    if (ok) {
      const float gt = bf16_to_f32(p.gates[((size_t)t * p.Hq + h) * p.NG + br]);
      const uint4 dd = *reinterpret_cast<const uint4*>(p.dout + src);
      const uint32_t w[4] = {dd.x, dd.y, dd.z, dd.w};
      uint32_t o4[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        o4[i] = pack_bf16x2(__uint_as_float(w[i] << 16) * gt, __uint_as_float(w[i] & 0xFFFF0000u) * gt);
      u = make_uint4(o4[0], o4[1], o4[2], o4[3]);
    }
    *reinterpret_cast<uint4*>(reinterpret_cast<unsigned char*>(S.g) + bswz<D>(r, ch)) = u;
  }
  for (int r = tid; r < kBkRows; r += kBkThreads) {
    const int rr = row0 + r;
    if (rr < rows_total) {
      const long long t = t_base + rr / p.G;
      const int h = g * p.G + rr % p.G;
      const size_t row = (size_t)t * p.Hq + h;
      S.lse2[r] = p.lse[row * p.NG + br] * 1.4426950408889634f;
      S.dlt[r] = p.delta[row * p.NG + br];
      S.tok[r] = rr / p.G;
    } else {
      S.lse2[r] = 0.f;
      S.dlt[r] = 0.f;
      S.tok[r] = -1;
    }
  }
  cp_async_commit();
  cp_async_wait<0>();
}

template <int D>
__device__ __forceinline__ void bk_load_keys(BkSmem<D>& S, const uint16_t* k, const uint16_t* v, long long first,
                                             int n_keys, int Hkv, int g, int tid) {
  constexpr int CPR = D / 8;
  for (int e = tid; e < 64 * CPR; e += kBkThreads) {
    const int r = e / CPR, ch = e % CPR;
    const bool ok = r < n_keys;
    const size_t src = ((size_t)(first + (ok ? r : 0)) * Hkv + g) * D + ch * 8;
    cp_async16(reinterpret_cast<unsigned char*>(S.kt) + bswz<D>(r, ch), k + src, ok);
    cp_async16(reinterpret_cast<unsigned char*>(S.vt) + bswz<D>(r, ch), v + src, ok);
  }
  cp_async_commit();
  cp_async_wait<0>();
}

// store the warp's 16 rows of dK (scaled by tau) and dV as fp32 into [row][Hkv][D] at dst_row0
template <int D>
__device__ __forceinline__ void bk_store(float* dkp, float* dvp, size_t dst_row0, int n_keys, int warp, int lane,
                                         int Hkv, int g, float tau, const float (&dk)[D / 8][4],
                                         const float (&dv)[D / 8][4]) {
  const int gq = lane >> 2, cq = lane & 3;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int kr = warp * 16 + gq + 8 * i;
    if (kr >= n_keys) continue;
    const size_t row = ((dst_row0 + kr) * Hkv + g) * D;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      *reinterpret_cast<float2*>(dkp + row + n * 8 + 2 * cq) = make_float2(tau * dk[n][2 * i], tau * dk[n][2 * i + 1]);
      *reinterpret_cast<float2*>(dvp + row + n * 8 + 2 * cq) = make_float2(dv[n][2 * i], dv[n][2 * i + 1]);
    }
  }
}

// selected + window parts of dK, dV for the tokens of key block j, group g
template <int D>
__global__ void __launch_bounds__(kBkThreads) bwd_kv_local_kernel(const BwdParams p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  BkSmem<D>& S = *reinterpret_cast<BkSmem<D>*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int j = blockIdx.x, g = blockIdx.y;
  const int u0 = p.off[j], n_j = min(64, p.off[j + 1] - u0);
  bk_load_keys<D>(S, p.k, p.v, u0, n_j, p.Hkv, g, tid);
  __syncthreads();
  uint32_t ka[D / 16][4], va[D / 16][4];
  bk_key_frags<D>(S, warp, lane, ka, va);
  const int key_valid = n_j - warp * 16;  // valid keys among this warp's 16
  const int gq = lane >> 2;
  const int key_pos[2] = {warp * 16 + gq, warp * 16 + gq + 8};
  float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) { dk[n][e] = 0.f; dv[n][e] = 0.f; }
  // selected branch: every query block whose routed set contains j, in ascending order; the
  // last pass is the window branch of block j itself
  const int list = p.idx_heads == 1 ? j : j * p.Hkv + g;
  const int l0 = p.inv_start[list], l1 = p.inv_start[list + 1];
  const int l_end = p.window > 0 ? l1 + 1 : l1;
  for (int li = l0; li < l_end; ++li) {
    const bool window = li == l1;
    const int a = window ? j : p.inv_list[li];
    const int br = window ? 2 : 1;
    const int t_base = p.off[a], rows_total = (p.off[a + 1] - t_base) * p.G;
    for (int row0 = 0; row0 < rows_total; row0 += kBkRows) {
      __syncthreads();
      bk_stage_rows<D>(S, p, g, br, row0, rows_total, t_base, tid);
      __syncthreads();
      const int subs = min(4, (rows_total - row0 + 15) / 16);
      for (int sub = 0; sub < subs; ++sub) {
        if (window)
          bk_tile<D, true>(S, sub, lane, key_valid, key_pos, p.window, p.scale_log2, ka, va, dk, dv);
        else
          bk_tile<D, false>(S, sub, lane, key_valid, key_pos, p.window, p.scale_log2, ka, va, dk, dv);
      }
    }
  }
  bk_store<D>(p.dk_tok, p.dv_tok, (size_t)u0, n_j, warp, lane, p.Hkv, g, p.tau, dk, dv);
}

// compressed part: partial dKbar / dVbar of 64 block means of group g over one split of the query tokens
template <int D>
__global__ void __launch_bounds__(kBkThreads) bwd_kv_cmp_kernel(const BwdParams p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  BkSmem<D>& S = *reinterpret_cast<BkSmem<D>*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int jc = blockIdx.x, g = blockIdx.y, split = blockIdx.z;
  const int j0 = jc * 64, n_j = min(64, p.B - j0);
  bk_load_keys<D>(S, p.kc, p.vc, j0, n_j, p.Hkv, g, tid);
  __syncthreads();
  uint32_t ka[D / 16][4], va[D / 16][4];
  bk_key_frags<D>(S, warp, lane, ka, va);
  const int key_valid = n_j - warp * 16;
  const int key_pos[2] = {0, 0};
  float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) { dk[n][e] = 0.f; dv[n][e] = 0.f; }
  // this split's query tokens (all heads of group g), rows token-major with G rows per token
  const long long t_lo = p.N * split / kBwdSplits, t_hi = p.N * (split + 1) / kBwdSplits;
  const int rows_total = (int)((t_hi - t_lo) * p.G);
  for (int row0 = 0; row0 < rows_total; row0 += kBkRows) {
    __syncthreads();
    bk_stage_rows<D>(S, p, g, 0, row0, rows_total, t_lo, tid);
    __syncthreads();
    const int subs = min(4, (rows_total - row0 + 15) / 16);
    for (int sub = 0; sub < subs; ++sub)
      bk_tile<D, false>(S, sub, lane, key_valid, key_pos, 0, p.scale_log2, ka, va, dk, dv);
  }
  bk_store<D>(p.dkc_part, p.dvc_part, (size_t)split * p.B + j0, n_j, warp, lane, p.Hkv, g, p.tau, dk, dv);
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
  bwd_query_tc_kernel<D><<<dim3(tiles, d.n_kv_heads, d.n_blocks), kBqtThreads, sm, s>>>(qm, om, km, vm, kcm, vcm, p);
  sm = sizeof(BkSmem<D>);
  bwd_kv_local_kernel<D><<<dim3(d.n_blocks, d.n_kv_heads), kBkThreads, sm, s>>>(p);
  bwd_kv_cmp_kernel<D><<<dim3((d.n_blocks + 63) / 64, d.n_kv_heads, kBwdSplits), kBkThreads, sm, s>>>(p);
  bwd_finish_kernel<<<d.n_blocks, 256, 0, s>>>(p, D);
  (void)idx_heads;
  return cudaGetLastError() == cudaSuccess ? LSRM_OK : LSRM_ERR_CUDA;
}

lsrm_status launch_backward(const lsrm_nsa_desc& d, const int32_t* off, const void* q, const void* k, const void* v,
                            const void* kc, const void* vc, const void* gates, const int32_t* idx, int idx_heads,
                            const float* lse, const void* dout, void* dq, void* dk, void* dv, void* dgates,
                            unsigned char* ws_bwd, uint32_t* status, cudaStream_t s) {
  if (d.top_k > 256 || d.n_gates < 2 || d.n_gates > 3 || d.n_blocks > 65535 || 128 % (d.n_q_heads / d.n_kv_heads) != 0)
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
  p.dq = (uint16_t*)dq;
  p.dgates = (uint16_t*)dgates;
  p.delta = reinterpret_cast<float*>(ws_bwd + w.delta);
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
