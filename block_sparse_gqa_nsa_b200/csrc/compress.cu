// S1 compression: per-block means of K and V (and Q for the pooled-query variant).
// LSRM page (hyper.ai "LSRM", 方法, equations k^cmp / v^cmp): the compressed key of a
// block is the average of its tokens' keys (the trained ResBlock before the pool is
// outside this library); Speed3R page (section 2.1, compression branch) pools Q too.
//
// Memory: tokens are block-major, so a block's rows of one tensor are one contiguous
// span of n_b * H * d bf16.  One CTA reads one (block, tensor) span with 16-byte loads
// (every thread a fixed 8-column slice, tokens strided over thread groups), reduces
// the token groups through shared memory and writes fp32 + bf16 means.  HBM bound:
// each input byte is read once.
#include "lsrm_common.cuh"

namespace lsrm {

constexpr int kCompressThreads = 256;

__global__ void __launch_bounds__(kCompressThreads)
compress_kernel(const int32_t* __restrict__ off, const uint16_t* __restrict__ x0, const uint16_t* __restrict__ x1,
                const uint16_t* __restrict__ x2, int32_t h0, int32_t h1, int32_t h2, int32_t d,
                float* o32_0, uint16_t* o16_0, float* o32_1, uint16_t* o16_1, float* o32_2, uint16_t* o16_2,
                const int32_t* __restrict__ kv_row) {
  extern __shared__ float red[];  // [groups][cols]
  const int b = blockIdx.x;
  const int which = blockIdx.y;
  const uint16_t* x = which == 0 ? x0 : (which == 1 ? x1 : x2);
  const int H = which == 0 ? h0 : (which == 1 ? h1 : h2);
  float* o32 = which == 0 ? o32_0 : (which == 1 ? o32_1 : o32_2);
  uint16_t* o16 = which == 0 ? o16_0 : (which == 1 ? o16_1 : o16_2);
  if (x == nullptr || (o32 == nullptr && o16 == nullptr)) return;
  const int cols = H * d;           // multiple of 8 (d in {32, 64})
  const int c8 = cols / 8;          // 16-byte column slices per token row
  const int t0 = off[b], t1 = off[b + 1];
  const int n = t1 - t0;
  // the K and V means may go to a permuted row (kv_row[b]); Q means stay at row b
  const int orow = (kv_row != nullptr && which < 2) ? kv_row[b] : b;
  const float inv_n = n > 0 ? 1.0f / (float)n : 0.0f;
  // process the columns in passes of at most kCompressThreads slices
  for (int cbase = 0; cbase < c8; cbase += kCompressThreads) {
    const int slices = min(c8 - cbase, kCompressThreads);
    const int groups = kCompressThreads / slices;
    const int tid = threadIdx.x;
    const int sl = tid % slices, grp = tid / slices;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (grp < groups) {
      const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t0 * cols) + cbase + sl;
      for (int t = grp; t < n; t += groups) {
        const uint4 u = __ldg(src + (size_t)t * c8);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] += __uint_as_float(w[i] << 16);
          acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
        }
      }
      float* r = red + (size_t)grp * slices * 8 + sl * 8;
#pragma unroll
      for (int i = 0; i < 8; ++i) r[i] = acc[i];
    }
    __syncthreads();
    // sum the token groups in a fixed order and write means
    for (int e = tid; e < slices * 8; e += kCompressThreads) {
      float s = 0.0f;
      for (int g = 0; g < groups; ++g) s += red[(size_t)g * slices * 8 + e];
      const float m = s * inv_n;
      const size_t oi = (size_t)orow * cols + (size_t)cbase * 8 + e;
      if (o32) o32[oi] = m;
      if (o16) o16[oi] = __bfloat16_as_ushort(__float2bfloat16_rn(m));
    }
    __syncthreads();
  }
}

lsrm_status launch_compress(const lsrm_nsa_desc& d, const int32_t* off, const void* q, const void* k, const void* v,
                            float* kc32, void* kc, float* vc32, void* vc, float* qc32, void* qc,
                            cudaStream_t stream, const int32_t* kv_row) {
  const int ny = (q != nullptr && (qc32 != nullptr || qc != nullptr)) ? 3 : 2;
  dim3 grid((unsigned)d.n_blocks, (unsigned)ny);
  const size_t smem = (size_t)kCompressThreads * 8 * sizeof(float);
  compress_kernel<<<grid, kCompressThreads, smem, stream>>>(
      off, (const uint16_t*)k, (const uint16_t*)v, (const uint16_t*)q, d.n_kv_heads, d.n_kv_heads, d.n_q_heads,
      d.head_dim, kc32, (uint16_t*)kc, vc32, (uint16_t*)vc, qc32, (uint16_t*)qc, kv_row);
  return cudaGetLastError() == cudaSuccess ? LSRM_OK : LSRM_ERR_CUDA;
}

}  // namespace lsrm
