// Backward of the pooled-query (Speed3R) layer (Speed3R page, section 2: the model trains end to
// end through the global sparse attention), with the routing fixed.  The forward is
//   out = g_cmp o_cmp + g_slc o_slc,
//   o_cmp[t] = softmax(tau Qbar[a] Kbar^T) Vbar for every token t of block a (pooled query),
//   o_slc[t] = softmax over the tokens of F u R(a, h) of tau q[t] k^T, times v,
// with Qbar, Kbar, Vbar the block means.  Chain rule, per head:
//   dgates = (<dO, o_cmp>, <dO, o_slc>);
//   pooled branch: Gbar[a] = sum_{t in a} g_cmp[t] dO[t] is the gradient of o_cmp[a]; with
//     Delta_bar = <Gbar, o_cmp>, dS = P (Gbar Vbar^T - Delta_bar) gives dQbar = tau dS Kbar,
//     dKbar = tau dS^T Qbar, dVbar = P^T Gbar; the block mean hands dXbar / n_b to every token;
//   selected branch: with dO_s = g_slc dO and Delta = <dO_s, o_slc>, dS = P (dO_s V^T - Delta) over
//     the joint softmax of forced and routed keys (its LSE saved by the forward) gives
//     dq = tau dS K, dK = tau dS^T q, dV = P^T dO_s.
// The forced keys are the same for every query: the forced part runs as dense attention backward
// (every token against the packed forced tokens).  Routed keys belong to one (block, head): their
// dq is taken per (block, head) and their dK / dV per (key block, head) over inverse routing lists,
// so every sum has a fixed order and the result is reproducible bit for bit.
//
// Matrix products use mma.sync m16n8k16 (bf16 operands, fp32 accumulation): each unit of work has
// 16 query rows (a pooled block of at most 16 tokens) or streams 64-row tiles against 64-key tiles.
#include "lsrm_common.cuh"

namespace lsrm {

lsrm_status launch_compress(const lsrm_nsa_desc& d, const int32_t* off, const void* q, const void* k, const void* v,
                            float* kc32, void* kc, float* vc32, void* vc, float* qc32, void* qc, cudaStream_t s,
                            const int32_t* kv_row);
lsrm_status launch_speed3r_forced(const lsrm_nsa_desc& d, const int32_t* off, const void* k, const void* v,
                                  uint32_t* bits, int* pre, int* total, void* kf, void* vf, uint32_t* status,
                                  cudaStream_t s);

namespace {

constexpr int kSbD = 64;            // head dim
constexpr float kLog2e = 1.4426950408889634f;

// byte offset of 16-byte chunk ch of row `row` in a swizzled [rows][64] bf16 tile (128-byte rows)
__device__ __forceinline__ uint32_t sb_swz(int row, int ch) { return (uint32_t)(row * 128 + ((ch ^ (row & 7)) << 4)); }

// copy `rows` rows (64 bf16 each) starting at row r0 of a [row][H][64] tensor (head h) into a
// swizzled tile; rows at or beyond n are zero-filled.  `lanes` threads share the copy.
__device__ __forceinline__ void sb_load_tile(unsigned char* tile, const uint16_t* x, long long r0, long long n,
                                             int H, int h, int rows, int tid, int lanes) {
  for (int e = tid; e < rows * 8; e += lanes) {
    const int r = e >> 3, ch = e & 7;
    const bool ok = r0 + r < n;
    const uint16_t* src = x + ((size_t)(ok ? r0 + r : 0) * H + h) * kSbD + ch * 8;
    cp_async16(tile + sb_swz(r, ch), src, ok);
  }
}

// A fragments (16 rows x 64) of rows [r0, r0 + 16) of a swizzled tile
__device__ __forceinline__ void sb_frag_a(uint32_t (&fa)[4][4], const unsigned char* tile, int r0, int lane) {
#pragma unroll
  for (int kt = 0; kt < 4; ++kt) {
    const int r = r0 + ((lane >> 3) & 1) * 8 + (lane & 7);
    const int ch = kt * 2 + (lane >> 4);
    ldmatrix_x4(fa[kt][0], fa[kt][1], fa[kt][2], fa[kt][3], smem_u32(tile) + sb_swz(r, ch));
  }
}

// acc[n] (+)= A (16 x 64, fragments) * Bt^T where Bt is a swizzled tile of nrows16 * 16 rows x 64
// (the n dimension runs over Bt's rows): the S = Q K^T pattern
template <int NT>
__device__ __forceinline__ void sb_mma_abt(float (&acc)[NT][4], const uint32_t (&fa)[4][4], const unsigned char* bt,
                                           int lane) {
#pragma unroll
  for (int kt = 0; kt < 4; ++kt)
#pragma unroll
    for (int np = 0; np < NT / 2; ++np) {
      uint32_t b0, b1, b2, b3;
      const int key = np * 16 + (lane >> 4) * 8 + (lane & 7);
      const int ch = kt * 2 + ((lane >> 3) & 1);
      ldmatrix_x4(b0, b1, b2, b3, smem_u32(bt) + sb_swz(key, ch));
      const uint32_t bb0[2] = {b0, b1}, bb1[2] = {b2, b3};
      mma_bf16_16816(acc[2 * np], fa[kt], bb0);
      mma_bf16_16816(acc[2 * np + 1], fa[kt], bb1);
    }
}

// acc[8] (+)= P (16 x 16*KT, fragments pa[KT]) * Bm where Bm is a swizzled tile of 16*KT rows x 64
// (the k dimension runs over Bm's rows): the O = P V pattern
template <int KT>
__device__ __forceinline__ void sb_mma_pb(float (&acc)[8][4], const uint32_t (&pa)[KT][4], const unsigned char* bm,
                                          int lane) {
#pragma unroll
  for (int kk = 0; kk < KT; ++kk)
#pragma unroll
    for (int dn = 0; dn < 4; ++dn) {
      uint32_t b0, b1, b2, b3;
      const int key = kk * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
      const int ch = dn * 2 + (lane >> 4);
      ldmatrix_x4_trans(b0, b1, b2, b3, smem_u32(bm) + sb_swz(key, ch));
      const uint32_t bb0[2] = {b0, b1}, bb1[2] = {b2, b3};
      mma_bf16_16816(acc[2 * dn], pa[kk], bb0);
      mma_bf16_16816(acc[2 * dn + 1], pa[kk], bb1);
    }
}

// accumulator tiles (n-tiles of 8 columns) -> A fragments over those columns, bf16
template <int NT>
__device__ __forceinline__ void sb_to_a(uint32_t (&pa)[NT / 2][4], const float (&x)[NT][4]) {
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    pa[n >> 1][(n & 1) * 2 + 0] = pack_bf16x2(x[n][0], x[n][1]);
    pa[n >> 1][(n & 1) * 2 + 1] = pack_bf16x2(x[n][2], x[n][3]);
  }
}

template <int NT>
__device__ __forceinline__ void sb_zero(float (&x)[NT][4]) {
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) x[n][e] = 0.f;
}

// ---- per-row preparation --------------------------------------------------------------------------
// 8 threads per (token, head) row, 8 dims each: dgates = (<dO, o_cmp>, <dO, o_slc>) (bf16),
// dO_s = g_slc dO (bf16), and rowc = (selected LSE in log2 units, Delta = g_slc <dO, o_slc>).
__global__ void sb_row_prep_kernel(const uint4* __restrict__ dout, const uint4* __restrict__ obr,
                                   const uint16_t* __restrict__ gates, const float* __restrict__ lse, long long rows,
                                   uint16_t* __restrict__ dgates, uint4* __restrict__ dos, float2* __restrict__ rowc) {
  const long long gid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  const long long row = gid >> 3;
  const int c = (int)(gid & 7);
  const bool act = row < rows;
  const long long rr = act ? row : 0;
  const uint4 o = dout[rr * 8 + c], oc = obr[(rr * 2 + 0) * 8 + c], os = obr[(rr * 2 + 1) * 8 + c];
  const uint32_t ow[4] = {o.x, o.y, o.z, o.w}, cw[4] = {oc.x, oc.y, oc.z, oc.w}, sw[4] = {os.x, os.y, os.z, os.w};
  const float g1 = bf16_to_f32(gates[rr * 2 + 1]);
  float d0 = 0.f, d1 = 0.f;
  uint32_t dw[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a0 = __uint_as_float(ow[i] << 16), a1 = __uint_as_float(ow[i] & 0xffff0000u);
    d0 += a0 * __uint_as_float(cw[i] << 16) + a1 * __uint_as_float(cw[i] & 0xffff0000u);
    d1 += a0 * __uint_as_float(sw[i] << 16) + a1 * __uint_as_float(sw[i] & 0xffff0000u);
    dw[i] = pack_bf16x2(g1 * a0, g1 * a1);
  }
#pragma unroll
  for (int m = 1; m < 8; m <<= 1) {
    d0 += __shfl_xor_sync(0xffffffffu, d0, m);
    d1 += __shfl_xor_sync(0xffffffffu, d1, m);
  }
  if (!act) return;
  dos[row * 8 + c] = make_uint4(dw[0], dw[1], dw[2], dw[3]);
  if (c == 0) {
    dgates[row * 2 + 0] = (uint16_t)(pack_bf16x2(d0, 0.f) & 0xffffu);
    dgates[row * 2 + 1] = (uint16_t)(pack_bf16x2(d1, 0.f) & 0xffffu);
    const float l = lse[row * 2 + 1];
    rowc[row] = make_float2(l == -INFINITY ? INFINITY : l * kLog2e, g1 * d1);
  }
}

// One warp per (block, head): Gbar = sum over the block's tokens of g_cmp dO (token order, fp32),
// Delta_bar = <Gbar, o_cmp> (o_cmp read from the block's first token), and the pooled LSE.
__global__ void sb_pool_prep_kernel(const int32_t* __restrict__ off, const uint16_t* __restrict__ dout,
                                    const uint16_t* __restrict__ obr, const uint16_t* __restrict__ gates,
                                    const float* __restrict__ lse, int B, int H, uint32_t* __restrict__ gbar16,
                                    float2* __restrict__ rowcb) {
  const long long w = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= (long long)B * H) return;
  const int a = (int)(w / H), h = (int)(w % H);
  const int t0 = off[a], t1 = off[a + 1];
  float g0 = 0.f, g1 = 0.f;
  for (int t = t0; t < t1; ++t) {
    const size_t row = (size_t)t * H + h;
    const float gc = bf16_to_f32(gates[row * 2 + 0]);
    const uint32_t x = reinterpret_cast<const uint32_t*>(dout + row * kSbD)[lane];
    g0 = fmaf(gc, __uint_as_float(x << 16), g0);
    g1 = fmaf(gc, __uint_as_float(x & 0xffff0000u), g1);
  }
  const size_t r0 = (size_t)t0 * H + h;
  const uint32_t ob = reinterpret_cast<const uint32_t*>(obr + (r0 * 2 + 0) * kSbD)[lane];
  float dl = g0 * __uint_as_float(ob << 16) + g1 * __uint_as_float(ob & 0xffff0000u);
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) dl += __shfl_xor_sync(0xffffffffu, dl, m);
  gbar16[w * 32 + lane] = pack_bf16x2(g0, g1);
  if (lane == 0) {
    const float l = lse[r0 * 2 + 0];
    rowcb[w] = make_float2(l == -INFINITY ? INFINITY : l * kLog2e, dl);
  }
}

// ---- dense attention backward (64-row tiles against 64-key tiles) -------------------------------
struct DenseBwd {
  const uint16_t* q;     // query rows [n_rows][H][64]
  const uint16_t* dout;  // their upstream gradient (already gated) [n_rows][H][64]
  const float2* rowc;    // (LSE log2 units, Delta) [n_rows][H]
  const uint16_t* k;     // keys [n_keys][H][64]
  const uint16_t* v;
  long long n_rows;
  int n_keys;
  const int* n_keys_dev;  // overrides n_keys when set
  int H;
  float scale_log2, tau;
  float* dq;  // [n_rows][H][64] = tau sum dS k          (dq kernel)
  float* dk;  // [n_keys][H][64] = tau sum dS^T q        (dkdv kernel; one partial per grid z of
  float* dv;  // [n_keys][H][64] = sum P^T dout            the query rows, split_stride apart)
  long long split_stride;
};

constexpr int kDbThreads = 128;  // 4 warps, 16 rows (or keys) each

struct DbSmem {
  unsigned char a[2][64 * 128];      // the CTA's own 64 rows: Q and dO (dq) or K and V (dkdv)
  unsigned char s[2][2][64 * 128];   // streamed tiles, two stages: K and V (dq) or Q and dO (dkdv)
  float2 rc[2][64];                  // (dkdv) the streamed rows' (LSE, Delta)
};

__global__ void __launch_bounds__(kDbThreads) sb_dense_dq_kernel(const DenseBwd p) {
  extern __shared__ __align__(128) unsigned char sb_smem[];
  DbSmem& S = *reinterpret_cast<DbSmem*>(sb_smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long r0 = (long long)blockIdx.x * 64;
  const int h = blockIdx.y;
  const int nk = p.n_keys_dev != nullptr ? *p.n_keys_dev : p.n_keys;
  sb_load_tile(S.a[0], p.q, r0, p.n_rows, p.H, h, 64, tid, kDbThreads);
  sb_load_tile(S.a[1], p.dout, r0, p.n_rows, p.H, h, 64, tid, kDbThreads);
  const int n_chunks = (nk + 63) / 64;
  if (n_chunks > 0) {
    sb_load_tile(S.s[0][0], p.k, 0, nk, p.H, h, 64, tid, kDbThreads);
    sb_load_tile(S.s[0][1], p.v, 0, nk, p.H, h, 64, tid, kDbThreads);
  }
  cp_async_commit();
  const int gq = lane >> 2, cq = lane & 3;
  float lse2[2], dlt[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const long long r = r0 + warp * 16 + gq + 8 * i;
    const float2 rc = r < p.n_rows ? p.rowc[(size_t)r * p.H + h] : make_float2(INFINITY, 0.f);
    lse2[i] = rc.x;
    dlt[i] = rc.y;
  }
  float dq[8][4];
  sb_zero(dq);
  uint32_t qa[4][4], da[4][4];
  for (int c = 0; c < n_chunks; ++c) {
    const int st = c & 1;
    if (c + 1 < n_chunks) {
      sb_load_tile(S.s[st ^ 1][0], p.k, (long long)(c + 1) * 64, nk, p.H, h, 64, tid, kDbThreads);
      sb_load_tile(S.s[st ^ 1][1], p.v, (long long)(c + 1) * 64, nk, p.H, h, 64, tid, kDbThreads);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (c == 0) {
      sb_frag_a(qa, S.a[0], warp * 16, lane);
      sb_frag_a(da, S.a[1], warp * 16, lane);
    }
    float s[8][4], dp[8][4];
    sb_zero(s);
    sb_zero(dp);
    sb_mma_abt<8>(s, qa, S.s[st][0], lane);
    sb_mma_abt<8>(dp, da, S.s[st][1], lane);
    const int nkc = min(64, nk - c * 64);
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = n * 8 + 2 * cq + (e & 1);
        const float pr = key < nkc ? fast_exp2(s[n][e] * p.scale_log2 - lse2[e >> 1]) : 0.f;
        s[n][e] = pr * (dp[n][e] - dlt[e >> 1]);  // dS
      }
    uint32_t pa[4][4];
    sb_to_a<8>(pa, s);
    sb_mma_pb<4>(dq, pa, S.s[st][0], lane);
    __syncthreads();  // the stage is overwritten by the next prefetch
  }
  cp_async_wait<0>();  // (no chunk at all: the row tiles' copies are still in flight)
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const long long r = r0 + warp * 16 + gq + 8 * i;
    if (r >= p.n_rows) continue;
    float* dst = p.dq + ((size_t)r * p.H + h) * kSbD;
#pragma unroll
    for (int n = 0; n < 8; ++n)
      *reinterpret_cast<float2*>(dst + n * 8 + 2 * cq) = make_float2(p.tau * dq[n][2 * i], p.tau * dq[n][2 * i + 1]);
  }
}

__global__ void __launch_bounds__(kDbThreads) sb_dense_dkdv_kernel(const DenseBwd p) {
  extern __shared__ __align__(128) unsigned char sb_smem[];
  DbSmem& S = *reinterpret_cast<DbSmem*>(sb_smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int k0 = blockIdx.x * 64, h = blockIdx.y;
  const int nk = p.n_keys_dev != nullptr ? *p.n_keys_dev : p.n_keys;
  if (k0 >= nk) return;
  sb_load_tile(S.a[0], p.k, k0, nk, p.H, h, 64, tid, kDbThreads);
  sb_load_tile(S.a[1], p.v, k0, nk, p.H, h, 64, tid, kDbThreads);
  // this CTA's share of the query-row chunks (grid z splits them; partial sums per split)
  const long long all_chunks = (p.n_rows + 63) / 64;
  const long long per = (all_chunks + gridDim.z - 1) / gridDim.z;
  const long long c_lo = blockIdx.z * per, c_hi = c_lo + per < all_chunks ? c_lo + per : all_chunks;
  const long long n_chunks = c_hi > c_lo ? c_hi - c_lo : 0;
  auto load_rows = [&](int st, long long cc) {
    const long long c = c_lo + cc;
    sb_load_tile(S.s[st][0], p.q, c * 64, p.n_rows, p.H, h, 64, tid, kDbThreads);
    sb_load_tile(S.s[st][1], p.dout, c * 64, p.n_rows, p.H, h, 64, tid, kDbThreads);
    if (tid < 64) {
      const long long r = c * 64 + tid;
      S.rc[st][tid] = r < p.n_rows ? p.rowc[(size_t)r * p.H + h] : make_float2(INFINITY, 0.f);
    }
  };
  if (n_chunks > 0) load_rows(0, 0);
  cp_async_commit();
  const int cq = lane & 3;
  float dk[8][4], dv[8][4];
  sb_zero(dk);
  sb_zero(dv);
  uint32_t ka[4][4], va[4][4];
  for (long long c = 0; c < n_chunks; ++c) {
    const int st = (int)(c & 1);
    if (c + 1 < n_chunks) load_rows(st ^ 1, c + 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (c == 0) {
      sb_frag_a(ka, S.a[0], warp * 16, lane);
      sb_frag_a(va, S.a[1], warp * 16, lane);
    }
    float s[8][4], dp[8][4];
    sb_zero(s);
    sb_zero(dp);
    sb_mma_abt<8>(s, ka, S.s[st][0], lane);   // S^T: keys x rows
    sb_mma_abt<8>(dp, va, S.s[st][1], lane);  // dP^T = V dO^T
    float pt[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 rc = S.rc[st][n * 8 + 2 * cq + (e & 1)];
        const float pr = fast_exp2(s[n][e] * p.scale_log2 - rc.x);
        pt[n][e] = pr;
        s[n][e] = pr * (dp[n][e] - rc.y);  // dS^T
      }
    uint32_t pa[4][4];
    sb_to_a<8>(pa, pt);
    sb_mma_pb<4>(dv, pa, S.s[st][1], lane);
    sb_to_a<8>(pa, s);
    sb_mma_pb<4>(dk, pa, S.s[st][0], lane);
    __syncthreads();
  }
  cp_async_wait<0>();
  const int gq = lane >> 2;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int kr = k0 + warp * 16 + gq + 8 * i;
    if (kr >= nk) continue;
    float* dkr = p.dk + blockIdx.z * p.split_stride + ((size_t)kr * p.H + h) * kSbD;
    float* dvr = p.dv + blockIdx.z * p.split_stride + ((size_t)kr * p.H + h) * kSbD;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      *reinterpret_cast<float2*>(dkr + n * 8 + 2 * cq) = make_float2(p.tau * dk[n][2 * i], p.tau * dk[n][2 * i + 1]);
      *reinterpret_cast<float2*>(dvr + n * 8 + 2 * cq) = make_float2(dv[n][2 * i], dv[n][2 * i + 1]);
    }
  }
}

// ---- routed part ------------------------------------------------------------------------------------
struct RoutedBwd {
  const int32_t* off;
  const uint16_t* q;      // [N][H][64]
  const uint16_t* k;
  const uint16_t* v;
  const uint16_t* dos;    // g_slc dO [N][H][64]
  const float2* rowc;     // [N][H]
  const int32_t* idx;     // [B][H][top_k]
  const uint32_t* fbits;  // forced blocks
  const float* dqf;       // forced part of dq [N][H][64] (tau included), or null
  const float* dqbar;     // [B][H][64]
  const float* dkbar;
  const float* dvbar;
  const int* inv_start;   // [B * H + 1]
  const int* inv_list;
  uint16_t* dq;           // outputs, bf16
  uint16_t* dk;
  uint16_t* dv;
  uint32_t* status;
  int B, H, top_k;
  float scale_log2, tau;
};

constexpr int kRbWarps = 4;

struct RbSmem {
  unsigned char q[kRbWarps][16 * 128];
  unsigned char d[kRbWarps][16 * 128];
  unsigned char k[kRbWarps][64 * 128];
  unsigned char v[kRbWarps][64 * 128];
};

// One warp per (block a, head h): dq of a's tokens over its routed keys, plus the forced part and
// the pooled branch's share dQbar / n_a.
__global__ void __launch_bounds__(kRbWarps * 32) sb_routed_dq_kernel(const RoutedBwd p) {
  extern __shared__ __align__(128) unsigned char sb_smem[];
  RbSmem& S = *reinterpret_cast<RbSmem*>(sb_smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long pair = (long long)blockIdx.x * kRbWarps + warp;
  if (pair >= (long long)p.B * p.H) return;
  const int h = (int)(pair / p.B), a = (int)(pair % p.B);
  const int H = p.H;
  const int t0 = p.off[a], n_a = min(16, p.off[a + 1] - t0);

  // routed blocks of (a, h), two per lane, and the exclusive prefix of their token counts
  int my_start[2] = {0, 0}, my_n[2] = {0, 0}, excl[2];
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int e = 32 * half + lane;
    if (e < p.top_k) {
      const int j = p.idx[((size_t)a * H + h) * p.top_k + e];
      if (j >= 0 && j < p.B) {
        my_start[half] = p.off[j];
        my_n[half] = p.off[j + 1] - my_start[half];
      } else if (j >= p.B) {
        raise_status(p.status, LSRM_ERR_BOUNDS);
      }
    }
  }
  int base = 0;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    int incl = my_n[half];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    excl[half] = base + incl - my_n[half];
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  const int nk = base;
  const int second0 = __shfl_sync(0xffffffffu, excl[1], 0);

  sb_load_tile(S.q[warp], p.q, t0, t0 + n_a, H, h, 16, lane, 32);
  sb_load_tile(S.d[warp], p.dos, t0, t0 + n_a, H, h, 16, lane, 32);
  cp_async_commit();
  cp_async_wait<0>();
  __syncwarp();
  uint32_t qa[4][4], da[4][4];
  sb_frag_a(qa, S.q[warp], 0, lane);
  sb_frag_a(da, S.d[warp], 0, lane);
  const int gq = lane >> 2, cq = lane & 3;
  float lse2[2], dlt[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int r = gq + 8 * i;
    const float2 rc = r < n_a ? p.rowc[(size_t)(t0 + r) * H + h] : make_float2(INFINITY, 0.f);
    lse2[i] = rc.x;
    dlt[i] = rc.y;
  }
  float dq[8][4];
  sb_zero(dq);
  const int n_chunks = (nk + 63) / 64;
  for (int c = 0; c < n_chunks; ++c) {
    __syncwarp();
    for (int e = lane; e < 64 * 8; e += 32) {
      const int kr = e >> 3, ch = e & 7;
      const int pos = c * 64 + kr;
      const bool ok = pos < nk;
      const bool hi = p.top_k > 32 && pos >= second0;
      int lo = 0;
#pragma unroll
      for (int step = 16; step > 0; step >>= 1) {
        const int pm0 = __shfl_sync(0xffffffffu, excl[0], lo + step);
        const int pm1 = __shfl_sync(0xffffffffu, excl[1], lo + step);
        if ((hi ? pm1 : pm0) <= pos) lo += step;
      }
      const int st0 = __shfl_sync(0xffffffffu, my_start[0], lo), pre0 = __shfl_sync(0xffffffffu, excl[0], lo);
      const int st1 = __shfl_sync(0xffffffffu, my_start[1], lo), pre1 = __shfl_sync(0xffffffffu, excl[1], lo);
      const int stt = hi ? st1 : st0, pre = hi ? pre1 : pre0;
      const long long u = ok ? (long long)stt + (pos - pre) : t0;
      const size_t src = ((size_t)u * H + h) * kSbD + ch * 8;
      cp_async16(S.k[warp] + sb_swz(kr, ch), p.k + src, ok);
      cp_async16(S.v[warp] + sb_swz(kr, ch), p.v + src, ok);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncwarp();
    float s[8][4], dp[8][4];
    sb_zero(s);
    sb_zero(dp);
    sb_mma_abt<8>(s, qa, S.k[warp], lane);
    sb_mma_abt<8>(dp, da, S.v[warp], lane);
    const int nkc = min(64, nk - c * 64);
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = n * 8 + 2 * cq + (e & 1);
        const float pr = key < nkc ? fast_exp2(s[n][e] * p.scale_log2 - lse2[e >> 1]) : 0.f;
        s[n][e] = pr * (dp[n][e] - dlt[e >> 1]);
      }
    uint32_t pa[4][4];
    sb_to_a<8>(pa, s);
    sb_mma_pb<4>(dq, pa, S.k[warp], lane);
  }
  const float inv_n = 1.f / (float)(p.off[a + 1] - t0);
  const float* qb = p.dqbar + ((size_t)a * H + h) * kSbD;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int r = gq + 8 * i;
    if (r >= n_a) continue;
    const size_t row = (size_t)(t0 + r) * H + h;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const int col = n * 8 + 2 * cq;
      float x0 = p.tau * dq[n][2 * i] + qb[col] * inv_n, x1 = p.tau * dq[n][2 * i + 1] + qb[col + 1] * inv_n;
      if (p.dqf != nullptr) {
        const float2 f = *reinterpret_cast<const float2*>(p.dqf + row * kSbD + col);
        x0 += f.x;
        x1 += f.y;
      }
      *reinterpret_cast<uint32_t*>(p.dq + row * kSbD + col) = pack_bf16x2(x0, x1);
    }
  }
}

// ---- routed dK, dV: per (key block j, head h), j not forced, over the query blocks that routed to j
// (the inverse list, ascending).  Lists of at most kListSeg entries are done by one warp, which
// writes the final rows; longer lists are cut into segments of kListSeg entries, one warp each,
// whose partial sums are added in segment order afterwards (routing concentrates on a few blocks,
// so some lists are thousands long).
struct RkSmem {
  unsigned char k[kRbWarps][16 * 128];
  unsigned char v[kRbWarps][16 * 128];
  unsigned char q[kRbWarps][2][16 * 128];
  unsigned char d[kRbWarps][2][16 * 128];
};

// dK, dV (without tau / the pooled share) of block j's 16 key rows from list entries [e_begin, e_end);
// the next entry's query rows are copied while the current one is computed
__device__ __forceinline__ void rk_range(const RoutedBwd& p, RkSmem& S, int warp, int lane, int j, int h,
                                         int e_begin, int e_end, float (&dk)[8][4], float (&dv)[8][4]) {
  const int H = p.H;
  const int u0 = p.off[j], n_j = min(16, p.off[j + 1] - u0);
  sb_load_tile(S.k[warp], p.k, u0, u0 + n_j, H, h, 16, lane, 32);
  sb_load_tile(S.v[warp], p.v, u0, u0 + n_j, H, h, 16, lane, 32);
  auto issue = [&](int e, int st) {
    const int a = p.inv_list[e];
    const int t0 = p.off[a], n_a = min(16, p.off[a + 1] - t0);
    sb_load_tile(S.q[warp][st], p.q, t0, t0 + n_a, H, h, 16, lane, 32);
    sb_load_tile(S.d[warp][st], p.dos, t0, t0 + n_a, H, h, 16, lane, 32);
  };
  if (e_begin < e_end) issue(e_begin, 0);
  cp_async_commit();
  cp_async_wait<0>();
  __syncwarp();
  uint32_t ka[4][4], va[4][4];
  sb_frag_a(ka, S.k[warp], 0, lane);
  sb_frag_a(va, S.v[warp], 0, lane);
  const int cq = lane & 3;
  for (int e = e_begin; e < e_end; ++e) {
    const int st = (e - e_begin) & 1;
    if (e + 1 < e_end) issue(e + 1, st ^ 1);
    cp_async_commit();
    const int a = p.inv_list[e];
    const int t0 = p.off[a], n_a = min(16, p.off[a + 1] - t0);
    // this lane's query columns: rows 2 cq + (0, 1) of each 8-row n-tile
    float2 rc[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        const int r = nt * 8 + 2 * cq + b;
        rc[nt][b] = r < n_a ? p.rowc[(size_t)(t0 + r) * H + h] : make_float2(INFINITY, 0.f);
      }
    cp_async_wait<1>();
    __syncwarp();
    float s[2][4], dp[2][4];
    sb_zero(s);
    sb_zero(dp);
    sb_mma_abt<2>(s, ka, S.q[warp][st], lane);   // S^T: 16 keys x 16 query rows
    sb_mma_abt<2>(dp, va, S.d[warp][st], lane);  // dP^T = V dO_s^T
    float pt[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const float2 c = rc[nt][x & 1];
        const float pr = fast_exp2(s[nt][x] * p.scale_log2 - c.x);
        pt[nt][x] = pr;
        s[nt][x] = pr * (dp[nt][x] - c.y);
      }
    uint32_t pa[1][4];
    sb_to_a<2>(pa, pt);
    sb_mma_pb<1>(dv, pa, S.d[warp][st], lane);
    sb_to_a<2>(pa, s);
    sb_mma_pb<1>(dk, pa, S.q[warp][st], lane);
    __syncwarp();  // stage st is refilled by the next iteration's copy
  }
  cp_async_wait<0>();
}

// final bf16 rows of block j: tau dK + dKbar / n_j, dV + dVbar / n_j
__device__ __forceinline__ void rk_write(const RoutedBwd& p, int lane, int j, int h, const float (&dk)[8][4],
                                         const float (&dv)[8][4]) {
  const int H = p.H;
  const int u0 = p.off[j], n_j = min(16, p.off[j + 1] - u0);
  const float inv_n = 1.f / (float)(p.off[j + 1] - u0);
  const float* kb = p.dkbar + ((size_t)j * H + h) * kSbD;
  const float* vb = p.dvbar + ((size_t)j * H + h) * kSbD;
  const int cq = lane & 3, gq = lane >> 2;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int r = gq + 8 * i;
    if (r >= n_j) continue;
    const size_t row = (size_t)(u0 + r) * H + h;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const int col = n * 8 + 2 * cq;
      *reinterpret_cast<uint32_t*>(p.dk + row * kSbD + col) =
          pack_bf16x2(p.tau * dk[n][2 * i] + kb[col] * inv_n, p.tau * dk[n][2 * i + 1] + kb[col + 1] * inv_n);
      *reinterpret_cast<uint32_t*>(p.dv + row * kSbD + col) =
          pack_bf16x2(dv[n][2 * i] + vb[col] * inv_n, dv[n][2 * i + 1] + vb[col + 1] * inv_n);
    }
  }
}

// one warp per (key block, head) whose list has at most kListSeg entries
__global__ void __launch_bounds__(kRbWarps * 32) sb_routed_dkdv_kernel(const RoutedBwd p) {
  extern __shared__ __align__(128) unsigned char sb_smem[];
  RkSmem& S = *reinterpret_cast<RkSmem*>(sb_smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long pair = (long long)blockIdx.x * kRbWarps + warp;
  if (pair >= (long long)p.B * p.H) return;
  const int h = (int)(pair / p.B), j = (int)(pair % p.B);
  if ((p.fbits[j >> 5] >> (j & 31)) & 1u) return;  // forced: written with the forced part
  const size_t li = (size_t)j * p.H + h;
  const int e0 = p.inv_start[li], e1 = p.inv_start[li + 1];
  if (e1 - e0 > kListSeg) return;  // segmented
  float dk[8][4], dv[8][4];
  sb_zero(dk);
  sb_zero(dv);
  rk_range(p, S, warp, lane, j, h, e0, e1, dk, dv);
  rk_write(p, lane, j, h, dk, dv);
}

// segments of the long lists: per list the number of segments (0 for short or forced lists), then
// per segment its list
__global__ void sb_seg_count_kernel(const int* __restrict__ inv_start, const uint32_t* __restrict__ fbits, int B,
                                    int H, int* seg_count, int* long_ids, int* n_long) {
  const long long li = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (li >= (long long)B * H) return;
  const int j = (int)(li / H);
  const int n = inv_start[li + 1] - inv_start[li];
  const bool forced = (fbits[j >> 5] >> (j & 31)) & 1u;
  seg_count[li] = (!forced && n > kListSeg) ? (n + kListSeg - 1) / kListSeg : 0;
  if (n > 64) long_ids[atomicAdd(n_long, 1)] = (int)li;  // sorted by the bitmap pass
}
__global__ void sb_seg_fill_kernel(const int* __restrict__ seg_count, const int* __restrict__ seg_start,
                                   long long n_lists, int* seg_list) {
  const long long li = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (li >= n_lists) return;
  for (int sgm = 0; sgm < seg_count[li]; ++sgm) seg_list[seg_start[li] + sgm] = (int)li;
}

// one warp per segment: the partial dK, dV of its entries, [segment][dK | dV][16 rows][64]
__global__ void __launch_bounds__(kRbWarps * 32) sb_routed_dkdv_seg_kernel(const RoutedBwd p, const int* seg_start,
                                                                           const int* seg_list, long long n_lists,
                                                                           float* seg_part) {
  extern __shared__ __align__(128) unsigned char sb_smem[];
  RkSmem& S = *reinterpret_cast<RkSmem*>(sb_smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long i = (long long)blockIdx.x * kRbWarps + warp;
  if (i >= seg_start[n_lists]) return;
  const int li = seg_list[i];
  const int j = li / p.H, h = li % p.H;
  const int sgm = (int)(i - seg_start[li]);
  const int e0 = p.inv_start[li] + sgm * kListSeg, e1 = min(p.inv_start[li + 1], e0 + kListSeg);
  float dk[8][4], dv[8][4];
  sb_zero(dk);
  sb_zero(dv);
  rk_range(p, S, warp, lane, j, h, e0, e1, dk, dv);
  float* out = seg_part + (size_t)i * 2 * 16 * kSbD;
  const int cq = lane & 3, gq = lane >> 2;
#pragma unroll
  for (int r2 = 0; r2 < 2; ++r2)
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const int r = gq + 8 * r2, col = n * 8 + 2 * cq;
      *reinterpret_cast<float2*>(out + r * kSbD + col) = make_float2(dk[n][2 * r2], dk[n][2 * r2 + 1]);
      *reinterpret_cast<float2*>(out + (16 + r) * kSbD + col) = make_float2(dv[n][2 * r2], dv[n][2 * r2 + 1]);
    }
}

// one warp per long list: its segments' partials added in segment order, then the final rows
__global__ void __launch_bounds__(kRbWarps * 32) sb_routed_dkdv_reduce_kernel(const RoutedBwd p, const int* seg_start,
                                                                              const float* seg_part) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long li = (long long)blockIdx.x * kRbWarps + warp;
  if (li >= (long long)p.B * p.H) return;
  const int s0 = seg_start[li], s1 = seg_start[li + 1];
  if (s1 == s0) return;
  const int j = (int)(li / p.H), h = (int)(li % p.H);
  const int cq = lane & 3, gq = lane >> 2;
  float dk[8][4], dv[8][4];
  sb_zero(dk);
  sb_zero(dv);
  for (int sg = s0; sg < s1; ++sg) {
    const float* in = seg_part + (size_t)sg * 2 * 16 * kSbD;
#pragma unroll
    for (int r2 = 0; r2 < 2; ++r2)
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const int r = gq + 8 * r2, col = n * 8 + 2 * cq;
        const float2 a = *reinterpret_cast<const float2*>(in + r * kSbD + col);
        const float2 b = *reinterpret_cast<const float2*>(in + (16 + r) * kSbD + col);
        dk[n][2 * r2] += a.x;
        dk[n][2 * r2 + 1] += a.y;
        dv[n][2 * r2] += b.x;
        dv[n][2 * r2 + 1] += b.y;
      }
  }
  rk_write(p, lane, j, h, dk, dv);
}

// ---- forced tokens: map of the packed copy, and the final dK, dV ----------------------------------
__global__ void sb_forced_map_kernel(const int32_t* __restrict__ off, const int32_t* __restrict__ forced,
                                     const int* __restrict__ pre, int B, int max_len, int2* __restrict__ fmap) {
  const int i = blockIdx.x;
  const int j = forced[i];
  if (j < 0 || j >= B) return;
  const int t0 = off[j], n = max(0, min(off[j + 1] - t0, max_len));
  for (int r = threadIdx.x; r < n; r += blockDim.x) fmap[pre[i] + r] = make_int2(t0 + r, j);
}

// one thread per (packed forced token, head, 8 dims): dk = the forced part's split partials summed
// in split order + dKbar / n_j (bf16)
__global__ void sb_forced_scatter_kernel(const int2* __restrict__ fmap, const int* __restrict__ ftotal,
                                         const int32_t* __restrict__ off, const float* __restrict__ dkf,
                                         const float* __restrict__ dvf, const float* __restrict__ dkbar,
                                         const float* __restrict__ dvbar, int H, long long cap, int n_split,
                                         long long split_stride, uint4* dk, uint4* dv) {
  const long long n = (long long)*ftotal * H * 8;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
    const long long uh = e >> 3;
    const int c = (int)(e & 7);
    const long long u = uh / H;
    const int h = (int)(uh % H);
    if (u >= cap) continue;
    const int2 m = fmap[u];
    const float inv_n = 1.f / (float)(off[m.y + 1] - off[m.y]);
    const float* a = dkf + (size_t)uh * kSbD + c * 8;
    const float* b = dvf + (size_t)uh * kSbD + c * 8;
    const float* ab = dkbar + ((size_t)m.y * H + h) * kSbD + c * 8;
    const float* bb = dvbar + ((size_t)m.y * H + h) * kSbD + c * 8;
    float sk[8], sv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      sk[i] = a[i];
      sv[i] = b[i];
    }
    for (int z = 1; z < n_split; ++z)
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        sk[i] += a[z * split_stride + i];
        sv[i] += b[z * split_stride + i];
      }
    uint32_t wk[4], wv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      wk[i] = pack_bf16x2(sk[2 * i] + ab[2 * i] * inv_n, sk[2 * i + 1] + ab[2 * i + 1] * inv_n);
      wv[i] = pack_bf16x2(sv[2 * i] + bb[2 * i] * inv_n, sv[2 * i + 1] + bb[2 * i + 1] * inv_n);
    }
    const size_t dst = ((size_t)m.x * H + h) * 8 + c;
    dk[dst] = make_uint4(wk[0], wk[1], wk[2], wk[3]);
    dv[dst] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
  }
}

// ---- inverse routing lists per (block, head): the query blocks that routed to it, ascending ---------
__global__ void sb_inv_count_kernel(const int32_t* __restrict__ idx, int B, int H, int k, int* count,
                                    uint32_t* status) {
  const long long n = (long long)B * H * k;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
    const int h = (int)((e / k) % H);
    const int j = idx[e];
    if (j < 0) continue;  // a row with fewer eligible blocks than k pads with -1
    if (j >= B) { raise_status(status, LSRM_ERR_BOUNDS); continue; }
    atomicAdd(count + (size_t)j * H + h, 1);
  }
}
constexpr int kSbScan = 1024;
__global__ void __launch_bounds__(kSbScan) sb_inv_scan_kernel(const int* count, int n, int* start) {
  __shared__ int part[kSbScan];
  const int per = (n + kSbScan - 1) / kSbScan;
  const int lo = min(n, (int)threadIdx.x * per), hi = min(n, lo + per);
  int s = 0;
  for (int i = lo; i < hi; ++i) s += count[i];
  part[threadIdx.x] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int i = 0; i < kSbScan; ++i) { const int c = part[i]; part[i] = acc; acc += c; }
    start[n] = acc;
  }
  __syncthreads();
  int acc = part[threadIdx.x];
  for (int i = lo; i < hi; ++i) { start[i] = acc; acc += count[i]; }
}
__global__ void sb_inv_fill_kernel(const int32_t* __restrict__ idx, int B, int H, int k, const int* start,
                                   int* cursor, int* list) {
  const long long n = (long long)B * H * k;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
    const int a = (int)(e / ((long long)H * k));
    const int h = (int)((e / k) % H);
    const int j = idx[e];
    if (j < 0 || j >= B) continue;
    const size_t li = (size_t)j * H + h;
    const int slot = atomicAdd(cursor + li, 1);
    list[start[li] + slot] = a;
  }
}
// ascending order of each list (a query block appears at most once per list): insertion sort of the
// lists of at most 64 entries here, one CTA per longer list below
__global__ void sb_inv_sort_kernel(const int* start, int n_lists, int* list) {
  const int li = blockIdx.x * blockDim.x + threadIdx.x;
  if (li >= n_lists) return;
  int* x = list + start[li];
  const int n = start[li + 1] - start[li];
  if (n > 64) return;
  for (int i = 1; i < n; ++i) {
    const int v = x[i];
    int j = i - 1;
    while (j >= 0 && x[j] > v) { x[j + 1] = x[j]; --j; }
    x[j + 1] = v;
  }
}

// a long list through a bitmap over the query blocks: set the entries' bits, then write the set bits
// in order (each thread owns a run of words; a scan of the per-thread counts places them)
constexpr int kSortThreads = 256;
__global__ void __launch_bounds__(kSortThreads) sb_inv_sort_long_kernel(const int* __restrict__ start,
                                                                        const int* __restrict__ long_ids,
                                                                        const int* __restrict__ n_long, int B,
                                                                        int* list) {
  extern __shared__ uint32_t bits[];
  __shared__ int part[kSortThreads];
  const int W = (B + 31) / 32;
  const int per = (W + kSortThreads - 1) / kSortThreads;
  const int w0 = min(W, (int)threadIdx.x * per), w1 = min(W, w0 + per);
  const int count = *n_long;
  for (int i = blockIdx.x; i < count; i += gridDim.x) {
    const int li = long_ids[i];
    int* x = list + start[li];
    const int n = start[li + 1] - start[li];
    for (int w = threadIdx.x; w < W; w += kSortThreads) bits[w] = 0u;
    __syncthreads();
    for (int e = threadIdx.x; e < n; e += kSortThreads) {
      const int a = x[e];
      atomicOr(&bits[a >> 5], 1u << (a & 31));
    }
    __syncthreads();
    int c = 0;
    for (int w = w0; w < w1; ++w) c += __popc(bits[w]);
    part[threadIdx.x] = c;
    __syncthreads();
    if (threadIdx.x == 0) {
      int acc = 0;
      for (int t = 0; t < kSortThreads; ++t) {
        const int v = part[t];
        part[t] = acc;
        acc += v;
      }
    }
    __syncthreads();
    int pos = part[threadIdx.x];
    for (int w = w0; w < w1; ++w) {
      uint32_t m = bits[w];
      while (m != 0u) {
        x[pos++] = w * 32 + (__ffs(m) - 1);
        m &= m - 1u;
      }
    }
    __syncthreads();  // the bitmap is cleared for the next list
  }
}

#define LSRM_TRY_BWD(x)             \
  do {                              \
    const lsrm_status _s = (x);     \
    if (_s != LSRM_OK) return _s;   \
  } while (0)

template <typename T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(reinterpret_cast<unsigned char*>(base) + off);
}

}  // namespace

lsrm_status launch_speed3r_backward(const lsrm_nsa_desc& d, const int32_t* off, const void* q, const void* k,
                                    const void* v, const void* gates, const int32_t* idx, const float* lse,
                                    const void* obr, const void* dout, void* dq, void* dk, void* dv, void* dgates,
                                    void* ws, uint32_t* status, cudaStream_t s) {
  if (d.head_dim != kSbD || d.max_block_len > 16 || d.top_k > 64 || d.n_q_heads != d.n_kv_heads || d.n_gates != 2)
    return LSRM_ERR_UNSUPPORTED;
  const Workspace w = workspace_layout(d);
  const PooledBwdWs b = pooled_bwd_layout(d);
  unsigned char* wb = at<unsigned char>(ws, w.bwd);
  const int B = d.n_blocks, H = d.n_q_heads;
  const long long N = d.n_tokens;
  const float tau = d.scale > 0 ? d.scale : 1.0f / sqrtf((float)d.head_dim);
  const float sl = tau * kLog2e;
  // forced bitmap, packed forced K / V and their prefix; pooled bf16 Q, K, V (block order)
  uint32_t* fbits = at<uint32_t>(ws, w.fbits);
  int* fpre = at<int>(ws, w.fpre);
  int* ftotal = at<int>(ws, w.ftotal);
  LSRM_TRY_BWD(launch_speed3r_forced(d, off, k, v, fbits, fpre, ftotal, at<void>(ws, w.kf), at<void>(ws, w.vf),
                                     status, s));
  void* qc16 = at<void>(ws, w.qc16);
  void* kc16 = at<void>(ws, w.kc16);
  void* vc16 = at<void>(ws, w.vc16);
  LSRM_TRY_BWD(launch_compress(d, off, q, k, v, nullptr, kc16, nullptr, vc16, nullptr, qc16, s, nullptr));
  // per-row and per-block constants
  float2* rowc = reinterpret_cast<float2*>(wb + b.rowc);
  float2* rowcb = reinterpret_cast<float2*>(wb + b.rowcb);
  uint16_t* dos = reinterpret_cast<uint16_t*>(wb + b.dos16);
  const long long rows = N * H;
  sb_row_prep_kernel<<<(unsigned)((rows * 8 + 255) / 256), 256, 0, s>>>(
      (const uint4*)dout, (const uint4*)obr, (const uint16_t*)gates, lse, rows, (uint16_t*)dgates, (uint4*)dos, rowc);
  sb_pool_prep_kernel<<<(unsigned)(((long long)B * H * 32 + 255) / 256), 256, 0, s>>>(
      off, (const uint16_t*)dout, (const uint16_t*)obr, (const uint16_t*)gates, lse, B, H,
      reinterpret_cast<uint32_t*>(wb + b.gbar16), rowcb);
  // pooled branch: dense backward of the B pooled queries over the B pooled keys, per head
  float* dqbar = reinterpret_cast<float*>(wb + b.dqbar);
  float* dkbar = reinterpret_cast<float*>(wb + b.dkbar);
  float* dvbar = reinterpret_cast<float*>(wb + b.dvbar);
  const size_t db_smem = sizeof(DbSmem);
  if (cudaFuncSetAttribute(sb_dense_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)db_smem) !=
          cudaSuccess ||
      cudaFuncSetAttribute(sb_dense_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)db_smem) !=
          cudaSuccess)
    return LSRM_ERR_CUDA;
  DenseBwd pb{};
  pb.q = (const uint16_t*)qc16;
  pb.dout = reinterpret_cast<const uint16_t*>(wb + b.gbar16);
  pb.rowc = rowcb;
  pb.k = (const uint16_t*)kc16;
  pb.v = (const uint16_t*)vc16;
  pb.n_rows = B;
  pb.n_keys = B;
  pb.H = H;
  pb.scale_log2 = sl;
  pb.tau = tau;
  pb.dq = dqbar;
  pb.dk = dkbar;
  pb.dv = dvbar;
  pb.split_stride = 0;
  const dim3 gblk((unsigned)((B + 63) / 64), (unsigned)H);
  sb_dense_dq_kernel<<<gblk, kDbThreads, db_smem, s>>>(pb);
  sb_dense_dkdv_kernel<<<gblk, kDbThreads, db_smem, s>>>(pb);
  // forced part of the selected branch: every token against the packed forced tokens
  const long long cap = (long long)(d.n_forced > 0 ? d.n_forced : 0) * d.max_block_len;
  float* dqf = nullptr;
  if (cap > 0) {
    dqf = reinterpret_cast<float*>(wb + b.dqf);
    DenseBwd pf{};
    pf.q = (const uint16_t*)q;
    pf.dout = dos;
    pf.rowc = rowc;
    pf.k = at<const uint16_t>(ws, w.kf);
    pf.v = at<const uint16_t>(ws, w.vf);
    pf.n_rows = N;
    pf.n_keys = (int)cap;
    pf.n_keys_dev = ftotal;
    pf.H = H;
    pf.scale_log2 = sl;
    pf.tau = tau;
    pf.dq = dqf;
    pf.dk = reinterpret_cast<float*>(wb + b.dkf);
    pf.dv = reinterpret_cast<float*>(wb + b.dvf);
    pf.split_stride = cap * H * kSbD;
    if ((N + 63) / 64 > INT32_MAX) return LSRM_ERR_UNSUPPORTED;
    sb_dense_dq_kernel<<<dim3((unsigned)((N + 63) / 64), (unsigned)H), kDbThreads, db_smem, s>>>(pf);
    sb_dense_dkdv_kernel<<<dim3((unsigned)((cap + 63) / 64), (unsigned)H, kForcedSplits), kDbThreads, db_smem, s>>>(
        pf);
  }
  // inverse routing lists
  const int n_lists = B * H;
  int* count = reinterpret_cast<int*>(wb + b.inv_count);
  int* cursor = reinterpret_cast<int*>(wb + b.inv_cursor);
  int* start = reinterpret_cast<int*>(wb + b.inv_start);
  int* list = reinterpret_cast<int*>(wb + b.inv_list);
  if (cudaMemsetAsync(count, 0, (size_t)n_lists * 4, s) != cudaSuccess ||
      cudaMemsetAsync(cursor, 0, (size_t)n_lists * 4, s) != cudaSuccess)
    return LSRM_ERR_CUDA;
  const long long n_idx = (long long)n_lists * d.top_k;
  const long long gi_want = (n_idx + 255) / 256 + 1;
  const unsigned gi = (unsigned)(gi_want < 148LL * 64 ? gi_want : 148LL * 64);
  sb_inv_count_kernel<<<gi, 256, 0, s>>>(idx, B, H, d.top_k, count, status);
  sb_inv_scan_kernel<<<1, kSbScan, 0, s>>>(count, n_lists, start);
  sb_inv_fill_kernel<<<gi, 256, 0, s>>>(idx, B, H, d.top_k, start, cursor, list);
  sb_inv_sort_kernel<<<(n_lists + 127) / 128, 128, 0, s>>>(start, n_lists, list);
  int* n_long = reinterpret_cast<int*>(wb + b.n_long);
  int* seg_count = reinterpret_cast<int*>(wb + b.seg_count);
  int* seg_start = reinterpret_cast<int*>(wb + b.seg_start);
  int* seg_list = reinterpret_cast<int*>(wb + b.seg_list);
  float* seg_part = reinterpret_cast<float*>(wb + b.seg_part);
  if (cudaMemsetAsync(n_long, 0, 4, s) != cudaSuccess) return LSRM_ERR_CUDA;
  sb_seg_count_kernel<<<(n_lists + 255) / 256, 256, 0, s>>>(start, fbits, B, H, seg_count,
                                                            reinterpret_cast<int*>(wb + b.long_ids), n_long);
  const size_t sort_smem = (size_t)((B + 31) / 32) * 4;
  if (sort_smem > 200 * 1024) return LSRM_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(sb_inv_sort_long_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sort_smem) !=
      cudaSuccess)
    return LSRM_ERR_CUDA;
  sb_inv_sort_long_kernel<<<148 * 2, kSortThreads, sort_smem, s>>>(start, reinterpret_cast<int*>(wb + b.long_ids),
                                                                   n_long, B, list);
  sb_inv_scan_kernel<<<1, kSbScan, 0, s>>>(seg_count, n_lists, seg_start);
  sb_seg_fill_kernel<<<(n_lists + 255) / 256, 256, 0, s>>>(seg_count, seg_start, n_lists, seg_list);
  // routed part: dq per (block, head); dK, dV per (non-forced key block, head)
  RoutedBwd pr{};
  pr.off = off;
  pr.q = (const uint16_t*)q;
  pr.k = (const uint16_t*)k;
  pr.v = (const uint16_t*)v;
  pr.dos = dos;
  pr.rowc = rowc;
  pr.idx = idx;
  pr.fbits = fbits;
  pr.dqf = dqf;
  pr.dqbar = dqbar;
  pr.dkbar = dkbar;
  pr.dvbar = dvbar;
  pr.inv_start = start;
  pr.inv_list = list;
  pr.dq = (uint16_t*)dq;
  pr.dk = (uint16_t*)dk;
  pr.dv = (uint16_t*)dv;
  pr.status = status;
  pr.B = B;
  pr.H = H;
  pr.top_k = d.top_k;
  pr.scale_log2 = sl;
  pr.tau = tau;
  const size_t rb_smem = sizeof(RbSmem), rk_smem = sizeof(RkSmem);
  if (cudaFuncSetAttribute(sb_routed_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rb_smem) !=
          cudaSuccess ||
      cudaFuncSetAttribute(sb_routed_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rk_smem) !=
          cudaSuccess ||
      cudaFuncSetAttribute(sb_routed_dkdv_seg_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rk_smem) !=
          cudaSuccess)
    return LSRM_ERR_CUDA;
  const long long pairs = (long long)B * H;
  const unsigned grb = (unsigned)((pairs + kRbWarps - 1) / kRbWarps);
  sb_routed_dq_kernel<<<grb, kRbWarps * 32, rb_smem, s>>>(pr);
  sb_routed_dkdv_kernel<<<grb, kRbWarps * 32, rk_smem, s>>>(pr);
  const long long seg_grid = ((long long)b.max_segs + kRbWarps - 1) / kRbWarps;
  if (seg_grid > INT32_MAX) return LSRM_ERR_UNSUPPORTED;
  sb_routed_dkdv_seg_kernel<<<(unsigned)seg_grid, kRbWarps * 32, rk_smem, s>>>(pr, seg_start, seg_list, pairs,
                                                                               seg_part);
  sb_routed_dkdv_reduce_kernel<<<grb, kRbWarps * 32, 0, s>>>(pr, seg_start, seg_part);
  // forced tokens: dK, dV of the forced part plus the pooled share
  if (cap > 0) {
    int2* fmap = reinterpret_cast<int2*>(wb + b.fmap);
    sb_forced_map_kernel<<<d.n_forced, 64, 0, s>>>(off, d.forced_blocks, fpre, B, d.max_block_len, fmap);
    sb_forced_scatter_kernel<<<148 * 8, 256, 0, s>>>(fmap, ftotal, off, reinterpret_cast<const float*>(wb + b.dkf),
                                                     reinterpret_cast<const float*>(wb + b.dvf), dkbar, dvbar, H, cap,
                                                     kForcedSplits, cap * H * kSbD, (uint4*)dk, (uint4*)dv);
  }
  return cudaGetLastError() == cudaSuccess ? LSRM_OK : LSRM_ERR_CUDA;
}

}  // namespace lsrm
