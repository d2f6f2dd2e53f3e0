// Speed3R pooled-query variant of the layer (Speed3R page, section 2.1 Global Sparse
// Attention, and section 2.2 for the always-selected reference frame and camera tokens).
//
// The selected branch of query token t (block a, head h) attends to the tokens of the forced
// blocks F (the same set for every query) and of the top-k routed blocks of (a, h).  It is
// computed in two parts whose softmaxes are merged exactly through their log-sum-exps:
//   forced part: dense attention of every token against the forced tokens, gathered once
//     into a contiguous [n_f][H][d] copy (tcgen05 kernel, launch_attn_dense);
//   routed part: here, one warp per (a, h) and up to 64 routed blocks, 16 query rows x (routed tokens) with mma.sync
//     m16n8k16 (the routed key set of (a, h) is shared by at most 16 rows, which is exactly
//     one MMA row tile).  Its epilogue merges in the forced part, adds the compressed branch
//     (pooled query, one output per block) and applies the two gates.
#include "lsrm_common.cuh"

namespace lsrm {

// ---- forced set: bitmap over blocks, prefix of token counts, gathered K / V -----------------------
__global__ void forced_bits_kernel(const int32_t* __restrict__ forced, int n_forced, int B, uint32_t* bits,
                                   uint32_t* status) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_forced; i += gridDim.x * blockDim.x) {
    const int j = forced[i];
    if (j < 0 || j >= B) { raise_status(status, LSRM_ERR_BOUNDS); continue; }
    atomicOr(bits + (j >> 5), 1u << (j & 31));
  }
}

// one thread: exclusive prefix of the forced blocks' token counts, and their total
// (a block longer than max_len would overrun the packed copy: it is flagged and clipped)
__global__ void forced_prefix_kernel(const int32_t* __restrict__ off, const int32_t* __restrict__ forced,
                                     int n_forced, int B, int max_len, int* pre, int* total, uint32_t* status) {
  if (blockIdx.x != 0 || threadIdx.x != 0) return;
  int acc = 0;
  for (int i = 0; i < n_forced; ++i) {
    pre[i] = acc;
    const int j = forced[i];
    if (j >= 0 && j < B) {
      int n = off[j + 1] - off[j];
      if (n > max_len || n < 0) {
        raise_status(status, LSRM_ERR_BOUNDS);
        n = n < 0 ? 0 : max_len;
      }
      acc += n;
    }
  }
  pre[n_forced] = acc;
  *total = acc;
}

// one CTA per forced block: copy its tokens' K and V rows (H * D bf16 each) to the packed copies
__global__ void forced_gather_kernel(const int32_t* __restrict__ off, const int32_t* __restrict__ forced,
                                     const int* __restrict__ pre, int B, int max_len, int row_u4,
                                     const uint4* __restrict__ k, const uint4* __restrict__ v, uint4* kf,
                                     uint4* vf) {
  const int i = blockIdx.x;
  const int j = forced[i];
  if (j < 0 || j >= B) return;
  const int t0 = off[j], n = max(0, min(off[j + 1] - t0, max_len)), dst0 = pre[i];
  for (int e = threadIdx.x; e < n * row_u4; e += blockDim.x) {
    const int r = e / row_u4, c = e % row_u4;
    kf[(size_t)(dst0 + r) * row_u4 + c] = k[(size_t)(t0 + r) * row_u4 + c];
    vf[(size_t)(dst0 + r) * row_u4 + c] = v[(size_t)(t0 + r) * row_u4 + c];
  }
}

// ---- routed part + merge + gated combine ----------------------------------------------------------
constexpr int kRtWarps = 4;
constexpr int kRtD = 64;
constexpr int kRtKeys = 64;

struct RoutedParams {
  const int32_t* off;
  const uint16_t* q;        // [N][H][64]
  const uint16_t* k;
  const uint16_t* v;
  const uint16_t* gates;    // [N][H][2] (cmp, slc)
  const int32_t* idx;       // [B][H][top_k]
  const float* o_forced;    // [N][H][64], forced part of the selected branch
  const float* lse_forced;  // [N][H]
  const float* o_blk;       // [B][H][64], compressed branch per block (pooled query)
  const float* lse_blk;     // [B][H]
  uint16_t* out;            // [N][H][64]
  float* lse_out;           // [N][H][2] (cmp, slc), optional
  uint16_t* obr;            // [N][H][2][64] bf16 branch outputs (cmp, slc) for the backward, optional
  uint32_t* status;
  int B, H, top_k;
  float scale_log2;
};

// byte offset of 16-byte chunk ch of row `row` in a swizzled [rows][64] bf16 tile (128-byte rows)
__device__ __forceinline__ uint32_t rt_swz(int row, int ch) { return (uint32_t)(row * 128 + ((ch ^ (row & 7)) << 4)); }

struct RtSmem {
  uint16_t q[kRtWarps][16 * kRtD];
  uint16_t kb[kRtWarps][kRtKeys * kRtD];
  uint16_t vb[kRtWarps][kRtKeys * kRtD];
};

__global__ void __launch_bounds__(kRtWarps * 32) speed3r_routed_kernel(const RoutedParams p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  RtSmem& S = *reinterpret_cast<RtSmem*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long pair = (long long)blockIdx.x * kRtWarps + warp;  // head-major: consecutive warps share a head
  if (pair >= (long long)p.B * p.H) return;
  const int h = (int)(pair / p.B), a = (int)(pair % p.B);
  const int t0 = p.off[a], n_a = min(16, p.off[a + 1] - t0);
  const int H = p.H;

  // routed blocks of (a, h): lane i holds blocks i and 32 + i (list entries in order); exclusive
  // prefix of their token counts over the whole list
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
  const int second0 = __shfl_sync(0xffffffffu, excl[1], 0);  // first key position of entry 32

  // Q rows of the block (zero beyond n_a)
  unsigned char* qs = reinterpret_cast<unsigned char*>(S.q[warp]);
  for (int e = lane; e < 16 * 8; e += 32) {
    const int r = e >> 3, ch = e & 7;
    const bool ok = r < n_a;
    const uint16_t* src = p.q + ((size_t)(t0 + (ok ? r : 0)) * H + h) * kRtD + ch * 8;
    cp_async16(qs + rt_swz(r, ch), src, ok);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncwarp();
  uint32_t qa[4][4];
#pragma unroll
  for (int kt = 0; kt < 4; ++kt) {
    const int r = ((lane >> 3) & 1) * 8 + (lane & 7);
    const int ch = kt * 2 + (lane >> 4);
    ldmatrix_x4(qa[kt][0], qa[kt][1], qa[kt][2], qa[kt][3], smem_u32(qs) + rt_swz(r, ch));
  }

  const int gq = lane >> 2, cq = lane & 3;
  float o[8][4];
#pragma unroll
  for (int n = 0; n < 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[n][e] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  unsigned char* ks = reinterpret_cast<unsigned char*>(S.kb[warp]);
  unsigned char* vs = reinterpret_cast<unsigned char*>(S.vb[warp]);
  const int n_chunks = (nk + kRtKeys - 1) / kRtKeys;
  for (int c = 0; c < n_chunks; ++c) {
    __syncwarp();  // the previous chunk's tiles are no longer read
    // token of every key position of the chunk: binary search of the routed-block prefix
    for (int e = lane; e < kRtKeys * 8; e += 32) {
      const int kr = e >> 3, ch = e & 7;
      const int pos = c * kRtKeys + kr;
      const bool ok = pos < nk;
      // the list entry holding position pos: the half first (entries 32.. start at second0), then
      // the largest lane of that half whose exclusive prefix <= pos (five fixed steps; every lane
      // joins each shuffle, reading both halves and keeping its own)
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
      const int st = hi ? st1 : st0, pre = hi ? pre1 : pre0;
      const long long u = ok ? (long long)st + (pos - pre) : t0;
      const size_t base = ((size_t)u * H + h) * kRtD + ch * 8;
      cp_async16(ks + rt_swz(kr, ch), p.k + base, ok);
      cp_async16(vs + rt_swz(kr, ch), p.v + base, ok);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncwarp();
    const int nkc = min(kRtKeys, nk - c * kRtKeys);
    float s[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[n][e] = 0.f;
#pragma unroll
    for (int kt = 0; kt < 4; ++kt)
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        const int key = np * 16 + (lane >> 4) * 8 + (lane & 7);
        const int ch = kt * 2 + ((lane >> 3) & 1);
        ldmatrix_x4(b0, b1, b2, b3, smem_u32(ks) + rt_swz(key, ch));
        const uint32_t bb0[2] = {b0, b1}, bb1[2] = {b2, b3};
        mma_bf16_16816(s[2 * np], qa[kt], bb0);
        mma_bf16_16816(s[2 * np + 1], qa[kt], bb1);
      }
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = n * 8 + 2 * cq + (e & 1);
        const float x = key < nkc ? s[n][e] * p.scale_log2 : -INFINITY;
        s[n][e] = x;
        mx[e >> 1] = fmaxf(mx[e >> 1], x);
      }
    float alpha[2], mref[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 1));
      mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 2));
      const float mn = fmaxf(m_run[i], mx[i]);
      alpha[i] = (mn == -INFINITY) ? 1.f : fast_exp2(m_run[i] - mn);
      m_run[i] = mn;
      mref[i] = (mn == -INFINITY) ? 0.f : mn;
      l_run[i] *= alpha[i];
    }
#pragma unroll
    for (int n = 0; n < 8; ++n)
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
      pa[n >> 1][(n & 1) * 2 + 0] = pack_bf16x2(pv[0], pv[1]);
      pa[n >> 1][(n & 1) * 2 + 1] = pack_bf16x2(pv[2], pv[3]);
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
      for (int dn = 0; dn < 4; ++dn) {
        uint32_t b0, b1, b2, b3;
        const int key = kk * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
        const int ch = dn * 2 + (lane >> 4);
        ldmatrix_x4_trans(b0, b1, b2, b3, smem_u32(vs) + rt_swz(key, ch));
        const uint32_t bb0[2] = {b0, b1}, bb1[2] = {b2, b3};
        mma_bf16_16816(o[2 * dn], pa[kk], bb0);
        mma_bf16_16816(o[2 * dn + 1], pa[kk], bb1);
      }
  }

  // epilogue: routed softmax -> merge with the forced part -> gated sum with the pooled branch
  const size_t blk = (size_t)a * H + h;
  const float lse_c = p.lse_blk[blk];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int r = gq + 8 * i;
    float l = l_run[i];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    if (r >= n_a) continue;
    const size_t row = (size_t)(t0 + r) * H + h;
    const float lf = p.lse_forced[row];                                  // natural log
    const float lr = l > 0.f ? (m_run[i] + __log2f(l)) * 0.6931471805599453f : -INFINITY;
    const float L = fmaxf(lf, lr);
    const float wf = lf == -INFINITY ? 0.f : __expf(lf - L);
    const float wr = lr == -INFINITY ? 0.f : __expf(lr - L);
    const float wsum = wf + wr;
    const float cf = wsum > 0.f ? wf / wsum : 0.f;
    const float cr = (wsum > 0.f && l > 0.f) ? wr / (wsum * l) : 0.f;  // routed O is unnormalised
    const float g_cmp = bf16_to_f32(p.gates[row * 2 + 0]), g_slc = bf16_to_f32(p.gates[row * 2 + 1]);
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const int col = n * 8 + 2 * cq;
      const float2 of = *reinterpret_cast<const float2*>(p.o_forced + row * kRtD + col);
      const float2 oc = *reinterpret_cast<const float2*>(p.o_blk + blk * kRtD + col);
      const float s0 = cf * of.x + cr * o[n][2 * i], s1 = cf * of.y + cr * o[n][2 * i + 1];
      *reinterpret_cast<uint32_t*>(p.out + row * kRtD + col) =
          pack_bf16x2(g_cmp * oc.x + g_slc * s0, g_cmp * oc.y + g_slc * s1);
      if (p.obr != nullptr) {
        *reinterpret_cast<uint32_t*>(p.obr + (row * 2 + 0) * kRtD + col) = pack_bf16x2(oc.x, oc.y);
        *reinterpret_cast<uint32_t*>(p.obr + (row * 2 + 1) * kRtD + col) = pack_bf16x2(s0, s1);
      }
    }
    if (p.lse_out != nullptr && cq == 0) {
      p.lse_out[row * 2 + 0] = lse_c;
      p.lse_out[row * 2 + 1] = wsum > 0.f ? L + __logf(wsum) : -INFINITY;
    }
  }
}

lsrm_status launch_speed3r_forced(const lsrm_nsa_desc& d, const int32_t* off, const void* k, const void* v,
                                  uint32_t* bits, int* pre, int* total, void* kf, void* vf, uint32_t* status,
                                  cudaStream_t s) {
  const size_t words = (size_t)d.n_blocks / 32 + 2;
  if (cudaMemsetAsync(bits, 0, words * 4, s) != cudaSuccess) return LSRM_ERR_CUDA;
  forced_bits_kernel<<<(d.n_forced + 255) / 256 + 1, 256, 0, s>>>(d.forced_blocks, d.n_forced, d.n_blocks, bits,
                                                                 status);
  if (off == nullptr) return cudaGetLastError() == cudaSuccess ? LSRM_OK : LSRM_ERR_CUDA;  // bitmap only
  forced_prefix_kernel<<<1, 32, 0, s>>>(off, d.forced_blocks, d.n_forced, d.n_blocks, d.max_block_len, pre, total,
                                        status);
  if (d.n_forced > 0) {
    const int row_u4 = d.n_kv_heads * d.head_dim * 2 / 16;
    forced_gather_kernel<<<d.n_forced, 256, 0, s>>>(off, d.forced_blocks, pre, d.n_blocks, d.max_block_len, row_u4,
                                                    (const uint4*)k, (const uint4*)v, (uint4*)kf, (uint4*)vf);
  }
  return cudaGetLastError() == cudaSuccess ? LSRM_OK : LSRM_ERR_CUDA;
}

// Largest L2 norm over the rows of x (rows of 64 floats, the fp32 pooled keys) as float bits (a
// positive float orders like its bits), the key side of the exact-ranking gate's error bound.
__global__ void rownorm_max_kernel(const float* __restrict__ x, long long rows, uint32_t* out) {
  float m = 0.f;
  for (long long r = (long long)blockIdx.x * blockDim.x + threadIdx.x; r < rows; r += (long long)gridDim.x * blockDim.x) {
    const float4* x4 = reinterpret_cast<const float4*>(x + r * 64);
    float s2 = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float4 v = __ldg(x4 + i);
      s2 = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, s2))));
    }
    m = fmaxf(m, sqrtf(s2));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float wm[32];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, wm[w]);
    if (!(m <= 3.0e38f)) m = 3.0e38f;  // a NaN or infinite mean: a huge (finite) bound
    atomicMax(out, __float_as_uint(m));
  }
}

lsrm_status launch_rownorm_max(const float* x, long long rows, uint32_t* out, cudaStream_t s) {
  if (cudaMemsetAsync(out, 0, sizeof(uint32_t), s) != cudaSuccess) return LSRM_ERR_CUDA;
  if (rows <= 0) return LSRM_OK;
  const long long want = (rows + 255) / 256;
  const unsigned blocks = (unsigned)(want < 148 * 8 ? want : 148 * 8);
  rownorm_max_kernel<<<blocks, 256, 0, s>>>(x, rows, out);
  return cudaGetLastError() == cudaSuccess ? LSRM_OK : LSRM_ERR_CUDA;
}

// Row order of the pooled keys for the routing passes: non-forced blocks first, in block order,
// then the forced blocks in block order (a stable partition, so among candidates row order is
// block order and ties still go to the lower block id).  One CTA: per-word forced counts, their
// exclusive prefix, then each block's row, the inverse map and the forced bitmap over rows.
__global__ void key_order_kernel(const uint32_t* __restrict__ bits, int B, int32_t* row_of_block,
                                 int32_t* block_of_row, uint32_t* bits_part) {
  extern __shared__ int pre[];  // [n_words + 1]
  const int n_words = (B + 31) / 32;
  for (int w = threadIdx.x; w < n_words; w += blockDim.x) pre[w + 1] = __popc(bits[w]);
  __syncthreads();
  if (threadIdx.x == 0) {
    pre[0] = 0;
    for (int w = 0; w < n_words; ++w) pre[w + 1] += pre[w];
  }
  __syncthreads();
  const int n_nf = B - pre[n_words];
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const uint32_t word = bits[b >> 5];
    const int below = pre[b >> 5] + __popc(word & ((1u << (b & 31)) - 1u));  // forced blocks below b
    const int r = ((word >> (b & 31)) & 1u) ? n_nf + below : b - below;
    row_of_block[b] = r;
    block_of_row[r] = b;
  }
  for (int w = threadIdx.x; w < B / 32 + 2; w += blockDim.x) {
    const int lo = 32 * w, s0 = max(lo, n_nf) - lo, s1 = min(lo + 32, B) - lo;
    uint32_t m = 0u;
    if (s1 > s0) {
      const uint32_t upto = s1 >= 32 ? 0xffffffffu : ((1u << s1) - 1u);
      m = upto & ~((1u << s0) - 1u);
    }
    bits_part[w] = m;
  }
}

lsrm_status launch_key_order(const lsrm_nsa_desc& d, const uint32_t* bits, int32_t* row_of_block,
                             int32_t* block_of_row, uint32_t* bits_part, cudaStream_t s) {
  const int n_words = (d.n_blocks + 31) / 32;
  key_order_kernel<<<1, 1024, (size_t)(n_words + 1) * sizeof(int), s>>>(bits, d.n_blocks, row_of_block,
                                                                        block_of_row, bits_part);
  return cudaGetLastError() == cudaSuccess ? LSRM_OK : LSRM_ERR_CUDA;
}

lsrm_status launch_speed3r_routed(const lsrm_nsa_desc& d, const int32_t* off, const void* q, const void* k,
                                  const void* v, const void* gates, const int32_t* idx, const float* o_forced,
                                  const float* lse_forced, const float* o_blk, const float* lse_blk, void* out,
                                  float* lse_out, uint32_t* status, cudaStream_t s, void* obr) {
  if (d.head_dim != kRtD || d.max_block_len > 16 || d.top_k > 64) return LSRM_ERR_UNSUPPORTED;
  RoutedParams p{};
  p.off = off;
  p.q = (const uint16_t*)q;
  p.k = (const uint16_t*)k;
  p.v = (const uint16_t*)v;
  p.gates = (const uint16_t*)gates;
  p.idx = idx;
  p.o_forced = o_forced;
  p.lse_forced = lse_forced;
  p.o_blk = o_blk;
  p.lse_blk = lse_blk;
  p.out = (uint16_t*)out;
  p.lse_out = lse_out;
  p.obr = (uint16_t*)obr;
  p.status = status;
  p.B = d.n_blocks;
  p.H = d.n_q_heads;
  p.top_k = d.top_k;
  const float tau = d.scale > 0 ? d.scale : 1.0f / sqrtf((float)d.head_dim);
  p.scale_log2 = tau * 1.4426950408889634f;
  const long long pairs = (long long)d.n_blocks * d.n_q_heads;
  const long long grid = (pairs + kRtWarps - 1) / kRtWarps;
  if (grid > 0x7FFFFFFFLL) return LSRM_ERR_UNSUPPORTED;
  const size_t smem = sizeof(RtSmem);
  if (cudaFuncSetAttribute(speed3r_routed_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return LSRM_ERR_CUDA;
  speed3r_routed_kernel<<<(unsigned)grid, kRtWarps * 32, smem, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? LSRM_OK : LSRM_ERR_CUDA;
}

// o_cmp of every token = its block's pooled output (and LSE): the standalone compressed-branch call
__global__ void pooled_broadcast_kernel(const int32_t* __restrict__ off, const float* __restrict__ o_blk,
                                       const float* __restrict__ lse_blk, int B, int H, int D, float* o_cmp,
                                       float* lse) {
  const int a = blockIdx.x;
  const int t0 = off[a], n = off[a + 1] - t0;
  for (int e = threadIdx.x; e < n * H * D; e += blockDim.x) {
    const int r = e / (H * D), hd = e % (H * D);
    o_cmp[(size_t)(t0 + r) * H * D + hd] = o_blk[(size_t)a * H * D + hd];
    if (lse != nullptr && hd % D == 0) lse[(size_t)(t0 + r) * H + hd / D] = lse_blk[(size_t)a * H + hd / D];
  }
}

lsrm_status launch_pooled_broadcast(const lsrm_nsa_desc& d, const int32_t* off, const float* o_blk,
                                    const float* lse_blk, float* o_cmp, float* lse, cudaStream_t s) {
  pooled_broadcast_kernel<<<d.n_blocks, 256, 0, s>>>(off, o_blk, lse_blk, d.n_blocks, d.n_q_heads, d.head_dim,
                                                     o_cmp, lse);
  return cudaGetLastError() == cudaSuccess ? LSRM_OK : LSRM_ERR_CUDA;
}

}  // namespace lsrm
