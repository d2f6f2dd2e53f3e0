// S2 routing kernels: geometric (integer centroid distance) and score-based top-k.
//
// Geometric routing, LSRM page (hyper.ai "LSRM", 方法, 3D-aware block routing
// paragraph): every token carries a 3D position; a query block keeps the blocks
// whose centres are nearest in Euclidean distance.  Centres are integer block
// means (round half up) and distances exact int64, so the result is bit-exact.
//
// Score routing, same paragraph: standard NSA picks the KV blocks with the highest
// attention scores against the compressed keys.  Here the score of block j for
// query block a and KV group g is the sum over a's tokens and g's heads of the
// compressed-branch softmax probability of j.
//
// Top-k is done by k rounds of a block-wide arg-min/arg-max (warp shuffles, then
// shared memory across warps): round r returns the best candidate strictly after
// the one returned by round r-1 in the total order (key, index), so no per-candidate
// state is kept and ties always go to the lower block index.
#include <cooperative_groups.h>

#include "lsrm_common.cuh"

namespace lsrm {

constexpr int kRouteThreads = 256;
constexpr int kCoordLimit = 1 << 29;

// ---- centroids -----------------------------------------------------------------------------------
// One warp per block: c[b][axis] = floor((2 S + n) / (2 n)), S = sum of the block's coordinates.
__global__ void centroid_kernel(const int32_t* __restrict__ off, const int32_t* __restrict__ coords, int32_t B,
                                int32_t* __restrict__ cen, uint32_t* status) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= B) return;
  const int t0 = off[warp], t1 = off[warp + 1];
  long long s[3] = {0, 0, 0};
  bool bad = false;
  for (int t = t0 + lane; t < t1; t += 32) {
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      const int c = __ldg(coords + (size_t)t * 3 + a);
      bad |= (c > kCoordLimit) || (c < -kCoordLimit);
      s[a] += c;
    }
  }
#pragma unroll
  for (int a = 0; a < 3; ++a)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s[a] += __shfl_xor_sync(0xffffffffu, s[a], o);
  if (__any_sync(0xffffffffu, bad) && lane == 0) raise_status(status, LSRM_ERR_BOUNDS);
  if (lane < 3) {
    const long long n = t1 - t0;
    const long long num = 2 * s[lane] + n, den = 2 * n;
    long long qv = num / den;
    if ((num % den != 0) && (num < 0)) --qv;  // floor division
    cen[(size_t)warp * 3 + lane] = (int32_t)qv;
  }
}

struct DistKey {
  long long d;
  int j;
};
__device__ __forceinline__ bool key_less(const DistKey& a, const DistKey& b) {
  return a.d < b.d || (a.d == b.d && a.j < b.j);
}

// One CTA per query block; centroids read from shared memory when they fit.
template <bool SMEM_CEN>
__global__ void __launch_bounds__(kRouteThreads)
geo_topk_kernel(const int32_t* __restrict__ cen, int32_t B, int32_t k, int32_t* __restrict__ idx) {
  extern __shared__ int32_t s_cen[];
  __shared__ DistKey s_warp[kRouteThreads / 32];
  __shared__ DistKey s_last;
  const int a = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (SMEM_CEN) {
    for (int i = tid; i < B * 3; i += kRouteThreads) s_cen[i] = cen[i];
  }
  const int32_t* C = SMEM_CEN ? s_cen : cen;
  if (tid == 0) s_last = DistKey{-1, -1};
  __syncthreads();
  const long long ax = C[a * 3 + 0], ay = C[a * 3 + 1], az = C[a * 3 + 2];
  for (int r = 0; r < k; ++r) {
    const DistKey last = s_last;
    DistKey best{LLONG_MAX, INT_MAX};
    for (int j = tid; j < B; j += kRouteThreads) {
      const long long dx = C[j * 3 + 0] - ax, dy = C[j * 3 + 1] - ay, dz = C[j * 3 + 2] - az;
      const DistKey cand{dx * dx + dy * dy + dz * dz, j};
      if (key_less(last, cand) && key_less(cand, best)) best = cand;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      DistKey other{__shfl_xor_sync(0xffffffffu, best.d, o), __shfl_xor_sync(0xffffffffu, best.j, o)};
      if (key_less(other, best)) best = other;
    }
    if (lane == 0) s_warp[warp] = best;
    __syncthreads();
    if (tid == 0) {
      DistKey b = s_warp[0];
      for (int w = 1; w < kRouteThreads / 32; ++w)
        if (key_less(s_warp[w], b)) b = s_warp[w];
      idx[(size_t)a * k + r] = b.j;
      s_last = b;
    }
    __syncthreads();
  }
}

// One CTA per query block for B <= kRouteThreads * kGeoPer: each thread computes its candidates'
// distances once, keeps them in registers and sorts them by (distance, index) with a 19-comparator
// network, so a thread's best remaining candidate is always its first.  Each round the block takes
// the minimum of those heads (warp shuffle, then the eight warp winners through shared memory and
// a 3-step shuffle, one block barrier per round with the winners alternating between two shared
// buffers) and the thread that owned the winner drops it.  The selection is the same as taking, k
// times, the best candidate strictly after the previous winner.
constexpr int kGeoPer = 8;
__device__ __forceinline__ void key_cswap(DistKey& a, DistKey& b) {
  if (key_less(b, a)) {
    const DistKey t = a;
    a = b;
    b = t;
  }
}
__device__ __forceinline__ DistKey shfl_key(const DistKey& x, int src_or_mask, bool xor_mode) {
  DistKey y;
  y.d = xor_mode ? __shfl_xor_sync(0xffffffffu, x.d, src_or_mask) : __shfl_sync(0xffffffffu, x.d, src_or_mask);
  y.j = xor_mode ? __shfl_xor_sync(0xffffffffu, x.j, src_or_mask) : __shfl_sync(0xffffffffu, x.j, src_or_mask);
  return y;
}
__global__ void __launch_bounds__(kRouteThreads)
geo_topk_reg_kernel(const int32_t* __restrict__ cen, int32_t B, int32_t k, int32_t* __restrict__ idx) {
  static_assert(kGeoPer == 8 && kRouteThreads / 32 == 8, "the sorting network and the winner reduction are for 8");
  __shared__ DistKey s_warp[2][kRouteThreads / 32];
  const int a = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long ax = cen[a * 3 + 0], ay = cen[a * 3 + 1], az = cen[a * 3 + 2];
  DistKey key[kGeoPer];
#pragma unroll
  for (int i = 0; i < kGeoPer; ++i) {
    const int j = tid + i * kRouteThreads;
    if (j < B) {
      const long long dx = cen[j * 3 + 0] - ax, dy = cen[j * 3 + 1] - ay, dz = cen[j * 3 + 2] - az;
      key[i] = DistKey{dx * dx + dy * dy + dz * dz, j};
    } else {
      key[i] = DistKey{LLONG_MAX, INT_MAX};
    }
  }
  // Batcher's odd-even merge network for 8 inputs (19 comparators, depth 6)
  key_cswap(key[0], key[2]); key_cswap(key[1], key[3]); key_cswap(key[4], key[6]); key_cswap(key[5], key[7]);
  key_cswap(key[0], key[4]); key_cswap(key[1], key[5]); key_cswap(key[2], key[6]); key_cswap(key[3], key[7]);
  key_cswap(key[0], key[1]); key_cswap(key[2], key[3]); key_cswap(key[4], key[5]); key_cswap(key[6], key[7]);
  key_cswap(key[2], key[4]); key_cswap(key[3], key[5]);
  key_cswap(key[1], key[4]); key_cswap(key[3], key[6]);
  key_cswap(key[1], key[2]); key_cswap(key[3], key[4]); key_cswap(key[5], key[6]);
  for (int r = 0; r < k; ++r) {
    DistKey best = key[0];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const DistKey other = shfl_key(best, o, true);
      if (key_less(other, best)) best = other;
    }
    if (lane == 0) s_warp[r & 1][warp] = best;
    __syncthreads();
    DistKey b = lane < kRouteThreads / 32 ? s_warp[r & 1][lane] : DistKey{LLONG_MAX, INT_MAX};
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) {
      const DistKey other = shfl_key(b, o, true);
      if (key_less(other, b)) b = other;
    }
    b = shfl_key(b, 0, false);
    if (tid == 0) idx[(size_t)a * k + r] = b.j;
    if (key[0].j == b.j) {  // this thread owned the winner: drop it (indices are unique)
#pragma unroll
      for (int i = 0; i + 1 < kGeoPer; ++i) key[i] = key[i + 1];
      key[kGeoPer - 1] = DistKey{LLONG_MAX, INT_MAX};
    }
  }
}

lsrm_status launch_route_geometric(const lsrm_nsa_desc& d, const int32_t* off, const int32_t* coords, int32_t* cen,
                                   int32_t* idx, uint32_t* status, cudaStream_t stream) {
  const int B = d.n_blocks;
  centroid_kernel<<<(B * 32 + 255) / 256, 256, 0, stream>>>(off, coords, B, cen, status);
  const size_t smem = (size_t)B * 3 * sizeof(int32_t);
  if (B <= kRouteThreads * kGeoPer) {
    geo_topk_reg_kernel<<<B, kRouteThreads, 0, stream>>>(cen, B, d.top_k, idx);
  } else if (smem <= 48 * 1024) {
    geo_topk_kernel<true><<<B, kRouteThreads, smem, stream>>>(cen, B, d.top_k, idx);
  } else {
    geo_topk_kernel<false><<<B, kRouteThreads, 0, stream>>>(cen, B, d.top_k, idx);
  }
  return cudaGetLastError() == cudaSuccess ? LSRM_OK : LSRM_ERR_CUDA;
}

// ---- camera-projection routing ------------------------------------------------------------------
// LSRM page, 方法, 3D-aware routing paragraph: the query point (the query block's centroid) is
// projected into every view; the image blocks of the tiles near the projected tile are the
// candidates, ranked by the smallest squared distance from any of their tokens to the query point;
// volume blocks are ranked by centroid distance.  One CTA per query block:
//   1. k_vol rounds of "best volume block strictly after the previous winner" by (centroid
//      distance, id);
//   2. one slot per (view, neighbour tile): the projection h = P [c; 1] in int64, pixel =
//      floor(h0 / h2), floor(h1 / h2) for h2 > 0, tile = floor(pixel / tile_px); the slot holds the
//      tile's block (or -1); a bitmap over image blocks marks the candidates (a block reached twice
//      keeps one slot);
//   3. one warp per slot: the smallest token distance;
//   4. k_img rounds over the slots by (token distance, id), and, once they run out, over the
//      image blocks outside the bitmap by (centroid distance, id).
// Every distance is exact int64, so the result is bit-exact.
constexpr int kCamMaxSlots = 4096;

__device__ __forceinline__ DistKey block_min_key(DistKey best, DistKey* s_warp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const DistKey other = shfl_key(best, o, true);
    if (key_less(other, best)) best = other;
  }
  if (lane == 0) s_warp[warp] = best;
  __syncthreads();
  DistKey b = s_warp[0];
  for (int w = 1; w < kRouteThreads / 32; ++w)
    if (key_less(s_warp[w], b)) b = s_warp[w];
  __syncthreads();  // s_warp is reused by the next call
  return b;
}

__device__ __forceinline__ long long floor_div_ll(long long a, long long b) {  // b > 0
  long long q = a / b;
  if ((a % b != 0) && (a < 0)) --q;
  return q;
}

__global__ void __launch_bounds__(kRouteThreads)
camera_route_kernel(const int32_t* __restrict__ off, const int32_t* __restrict__ coords,
                    const int32_t* __restrict__ cen, int32_t B, int32_t n_vol, int32_t n_views,
                    const int32_t* __restrict__ proj, int32_t tiles_x, int32_t tiles_y, int32_t tile_px,
                    const int32_t* __restrict__ tile_block, int32_t radius, int32_t k_vol, int32_t k_img,
                    int32_t* __restrict__ idx, uint32_t* status) {
  extern __shared__ __align__(16) unsigned char cam_smem[];
  __shared__ DistKey s_warp[kRouteThreads / 32];
  const int side = 2 * radius + 1, per_view = side * side;
  const int n_slots = n_views * per_view;
  const int n_img = B - n_vol;
  long long* s_d = reinterpret_cast<long long*>(cam_smem);
  int32_t* s_blk = reinterpret_cast<int32_t*>(s_d + n_slots);
  uint32_t* s_bits = reinterpret_cast<uint32_t*>(s_blk + n_slots);
  const int n_words = (n_img + 31) / 32;
  const int a = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = k_vol + k_img;
  const long long ax = cen[a * 3 + 0], ay = cen[a * 3 + 1], az = cen[a * 3 + 2];
  auto cdist = [&](int j) {
    const long long dx = cen[j * 3 + 0] - ax, dy = cen[j * 3 + 1] - ay, dz = cen[j * 3 + 2] - az;
    return dx * dx + dy * dy + dz * dz;
  };
  const DistKey none{LLONG_MAX, INT_MAX};

  // 1. volume blocks by centroid distance
  DistKey last{-1, -1};
  for (int r = 0; r < k_vol; ++r) {
    DistKey best = none;
    for (int j = tid; j < n_vol; j += kRouteThreads) {
      const DistKey c{cdist(j), j};
      if (key_less(last, c) && key_less(c, best)) best = c;
    }
    last = block_min_key(best, s_warp);
    if (tid == 0) idx[(size_t)a * K + r] = last.j;
  }
  if (k_img == 0) return;

  // 2. candidate slots
  for (int i = tid; i < n_words; i += kRouteThreads) s_bits[i] = 0u;
  __syncthreads();
  for (int i = tid; i < n_slots; i += kRouteThreads) {
    const int v = i / per_view, e = i - v * per_view;
    const int32_t* P = proj + (size_t)v * 12;
    long long h[3];
#pragma unroll
    for (int r = 0; r < 3; ++r)
      h[r] = (long long)P[4 * r] * ax + (long long)P[4 * r + 1] * ay + (long long)P[4 * r + 2] * az + P[4 * r + 3];
    int b = -1;
    if (h[2] > 0) {
      const long long tx = floor_div_ll(floor_div_ll(h[0], h[2]), tile_px) + (e % side) - radius;
      const long long ty = floor_div_ll(floor_div_ll(h[1], h[2]), tile_px) + (e / side) - radius;
      if (tx >= 0 && ty >= 0 && tx < tiles_x && ty < tiles_y) {
        b = tile_block[((size_t)v * tiles_y + ty) * tiles_x + tx];
        if (b >= B || (b >= 0 && b < n_vol)) {
          raise_status(status, LSRM_ERR_BOUNDS);
          b = -1;
        } else if (b >= 0) {
          const uint32_t bit = 1u << ((b - n_vol) & 31);
          if (atomicOr(&s_bits[(b - n_vol) >> 5], bit) & bit) b = -1;  // reached before: one slot
        }
      }
    }
    s_blk[i] = b;
  }
  __syncthreads();

  // 3. smallest token distance of each candidate (one warp per slot)
  for (int i = warp; i < n_slots; i += kRouteThreads / 32) {
    const int b = s_blk[i];
    if (b < 0) continue;
    long long m = LLONG_MAX;
    for (int t = off[b] + lane; t < off[b + 1]; t += 32) {
      const long long dx = coords[(size_t)t * 3] - ax, dy = coords[(size_t)t * 3 + 1] - ay,
                      dz = coords[(size_t)t * 3 + 2] - az;
      m = min(m, dx * dx + dy * dy + dz * dz);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = min(m, (long long)__shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) s_d[i] = m;
  }
  __syncthreads();

  // 4. image blocks: the candidates, then the fill
  last = DistKey{-1, -1};
  bool fill = false;
  for (int r = 0; r < k_img; ++r) {
    DistKey best = none;
    if (!fill) {
      for (int i = tid; i < n_slots; i += kRouteThreads) {
        const int b = s_blk[i];
        if (b < 0) continue;
        const DistKey c{s_d[i], b};
        if (key_less(last, c) && key_less(c, best)) best = c;
      }
      best = block_min_key(best, s_warp);
      if (best.j == INT_MAX) {  // no candidate left: the fill starts from the beginning
        fill = true;
        last = DistKey{-1, -1};
      }
    }
    if (fill) {
      best = none;
      for (int j = n_vol + tid; j < B; j += kRouteThreads) {
        if ((s_bits[(j - n_vol) >> 5] >> ((j - n_vol) & 31)) & 1u) continue;
        const DistKey c{cdist(j), j};
        if (key_less(last, c) && key_less(c, best)) best = c;
      }
      best = block_min_key(best, s_warp);
    }
    last = best;
    if (tid == 0) idx[(size_t)a * K + k_vol + r] = best.j;
  }
}

size_t camera_route_smem(int B, int n_vol, int n_slots) {
  return (size_t)n_slots * (sizeof(long long) + sizeof(int32_t)) + (size_t)((B - n_vol + 31) / 32) * 4;
}

lsrm_status launch_route_camera(const lsrm_nsa_desc& d, const int32_t* off, const int32_t* coords, int32_t n_vol,
                                int32_t n_views, const int32_t* proj, int32_t tiles_x, int32_t tiles_y,
                                int32_t tile_px, const int32_t* tile_block, int32_t radius, int32_t k_vol,
                                int32_t* cen, int32_t* idx, uint32_t* status, cudaStream_t stream) {
  const int B = d.n_blocks;
  const long long side = 2LL * radius + 1;
  const long long n_slots = (long long)n_views * side * side;
  if (n_slots > kCamMaxSlots) return LSRM_ERR_UNSUPPORTED;
  const size_t smem = camera_route_smem(B, n_vol, (int)n_slots);
  if (smem > 200 * 1024) return LSRM_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(camera_route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return LSRM_ERR_CUDA;
  centroid_kernel<<<(B * 32 + 255) / 256, 256, 0, stream>>>(off, coords, B, cen, status);
  camera_route_kernel<<<B, kRouteThreads, smem, stream>>>(off, coords, cen, B, n_vol, n_views, proj, tiles_x, tiles_y,
                                                          tile_px, tile_block, radius, k_vol, d.top_k - k_vol, idx,
                                                          status);
  return cudaGetLastError() == cudaSuccess ? LSRM_OK : LSRM_ERR_CUDA;
}

// ---- score routing -------------------------------------------------------------------------------
// One CTA per (query block a, KV group g), fp32 throughout, one thread per query row (the row's q
// in registers; the compressed keys staged in shared memory in chunks of kScoreChunk and read
// as broadcasts).  Pass 1 forms each row's softmax max and normaliser over all B compressed keys
// (log2 units); pass 2 forms the probabilities chunk by chunk, each thread summing them over its
// rows, and the per-thread partial sums are added in a fixed order (threads in index order), so
// the scores are reproducible bit for bit.  Then k rounds of arg-max by (score desc, j asc).
constexpr int kScoreChunk = 32;  // compressed keys per chunk (one register per key per thread)
constexpr int kMaxScoreRows = 64 * 64;
constexpr int kMaxScoreSplits = 8;

// k rounds of "best key strictly after the previous winner" by (score desc, j asc) over s_score[B]
__device__ void score_topk_rounds(const float* s_score, int B, int k, int32_t* dst, float* s_bv, int* s_bj,
                                  float* s_lv, int* s_lj) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) { *s_lv = INFINITY; *s_lj = -1; }
  __syncthreads();
  for (int r = 0; r < k; ++r) {
    const float lv = *s_lv;
    const int lj = *s_lj;
    float bv = -INFINITY;
    int bj = INT_MAX;
    for (int j = tid; j < B; j += kRouteThreads) {
      const float v = s_score[j];
      const bool after_last = (v < lv) || (v == lv && j > lj);
      const bool better = (v > bv) || (v == bv && j < bj);
      if (after_last && better) { bv = v; bj = j; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
      if (ov > bv || (ov == bv && oj < bj)) { bv = ov; bj = oj; }
    }
    if (lane == 0) { s_bv[warp] = bv; s_bj[warp] = bj; }
    __syncthreads();
    if (tid == 0) {
      float v = s_bv[0];
      int j = s_bj[0];
      for (int w = 1; w < kRouteThreads / 32; ++w)
        if (s_bv[w] > v || (s_bv[w] == v && s_bj[w] < j)) { v = s_bv[w]; j = s_bj[w]; }
      dst[r] = j;
      *s_lv = v;
      *s_lj = j;
    }
    __syncthreads();
  }
}

// Sum of acc[kk] over the warp's lanes for every key kk, by a fixed butterfly: at each stage a lane
// keeps the half of its keys its lane bit selects and adds the partner's copy of that half, so lane l
// ends with key l; out[l] receives it.
__device__ __forceinline__ void warp_key_sums(float (&acc)[kScoreChunk], int lane, float* out) {
#pragma unroll
  for (int o = kScoreChunk / 2; o >= 1; o >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const float send = upper ? acc[i] : acc[i + o];
      const float keep = upper ? acc[i + o] : acc[i];
      acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  out[lane] = acc[0];
}

// One CTA per (query block a, KV group g, split of the block's rows).  The splits of one (a, g) form
// a thread-block cluster (grid z): each CTA leaves its per-key sums in its shared memory, and the
// cluster's first CTA adds them in split order through distributed shared memory and ranks.  Per
// key, the threads' partial sums are added by a fixed shuffle tree within each warp (lane l ends
// with key l) and then warp by warp, so the scores are reproducible bit for bit.
template <int D>
__global__ void __launch_bounds__(kRouteThreads)
score_route_kernel(const int32_t* __restrict__ off, const uint16_t* __restrict__ q, const float* __restrict__ kc32,
                   int32_t B, int32_t Hq, int32_t Hkv, int32_t k, float scale, int32_t* __restrict__ idx,
                   float* __restrict__ score_out, uint32_t* status) {
  extern __shared__ float smem[];
  float* s_k = smem;                                            // [kScoreChunk][D] compressed keys of the chunk
  float* s_wsum = s_k + kScoreChunk * D;                        // [warps][kScoreChunk] per-warp sums
  float* s_score = s_wsum + (kRouteThreads / 32) * kScoreChunk;  // [B]
  __shared__ float s_bv[kRouteThreads / 32];
  __shared__ int s_bj[kRouteThreads / 32];
  __shared__ float s_lv;
  __shared__ int s_lj;
  const int a = blockIdx.x, g = blockIdx.y, split = blockIdx.z, n_split = gridDim.z;
  const int G = Hq / Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = off[a];
  // a block longer than the descriptor allows: flag it and clip
  int rows = (off[a + 1] - t0) * G;
  if (rows > kMaxScoreRows) {
    if (tid == 0 && split == 0) raise_status(status, LSRM_ERR_BOUNDS);
    rows = kMaxScoreRows;
  }
  const int rows_per = (rows + n_split - 1) / n_split;
  const int r_lo = split * rows_per, r_hi = min(rows, r_lo + rows_per);
  const float sl2 = scale * 1.4426950408889634f;  // logits in log2 units
  const int nchunks = (B + kScoreChunk - 1) / kScoreChunk;
  constexpr int kRowsPerThread = kMaxScoreRows / kRouteThreads;
  // the CTA's per-key sums are in s_score: add the cluster's splits in order (first CTA), then rank
  auto finish = [&](float* sc) {
    if (n_split > 1) {
      cooperative_groups::cluster_group cluster = cooperative_groups::this_cluster();
      cluster.sync();  // every split's sums are in its shared memory
      if (split == 0) {
        for (int j = tid; j < B; j += kRouteThreads) {
          float sum = sc[j];
          for (int r = 1; r < n_split; ++r) sum += cluster.map_shared_rank(sc, r)[j];
          sc[j] = sum;
        }
      }
      cluster.sync();  // the other splits keep their shared memory until it has been read
      if (split != 0) return;
    }
    __syncthreads();
    if (score_out)
      for (int j = tid; j < B; j += kRouteThreads) score_out[((size_t)a * Hkv + g) * B + j] = sc[j];
    score_topk_rounds(sc, B, k, idx + ((size_t)a * Hkv + g) * k, s_bv, s_bj, &s_lv, &s_lj);
  };

  auto load_chunk = [&](int c) {
    __syncthreads();
    for (int e = tid; e < kScoreChunk * D; e += kRouteThreads) {
      const int kk = e / D, col = e % D;
      const int j = c * kScoreChunk + kk;
      s_k[e] = j < B ? kc32[((size_t)j * Hkv + g) * D + col] : 0.0f;
    }
    __syncthreads();
  };
  auto load_q = [&](int r, float* qv) {
    const int t = t0 + r / G, h = g * G + r % G;
    const uint4* src = reinterpret_cast<const uint4*>(q + ((size_t)t * Hq + h) * D);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      const uint4 u = __ldg(src + c);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        qv[8 * c + 2 * e] = __uint_as_float(w[e] << 16);
        qv[8 * c + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
      }
    }
  };
  // raw logits of one row against the chunk's keys (keys past B give -inf and are not computed)
  auto chunk_logits = [&](const float* qv, int c, float* sv) {
    const int nk = B - c * kScoreChunk;
#pragma unroll
    for (int kk = 0; kk < kScoreChunk; ++kk) {
      float s = 0.0f;
      if (kk < nk) {
#pragma unroll
        for (int cc = 0; cc < D; ++cc) s = fmaf(qv[cc], s_k[kk * D + cc], s);
      }
      sv[kk] = kk < nk ? s * sl2 : -INFINITY;
    }
  };

  // one chunk of keys and at most one row per thread: the logits are formed once and kept
  if (nchunks == 1 && r_hi - r_lo <= kRouteThreads) {
    float acc[kScoreChunk];
    const int r = r_lo + tid;
    float qv[D];
    if (r < r_hi) load_q(r, qv);  // issued before the keys' copy so the two loads overlap
    load_chunk(0);
    if (r < r_hi) {
      chunk_logits(qv, 0, acc);
      float mx = -INFINITY;
#pragma unroll
      for (int kk = 0; kk < kScoreChunk; ++kk) mx = fmaxf(mx, acc[kk]);
      float l = 0.0f;
#pragma unroll
      for (int kk = 0; kk < kScoreChunk; ++kk) {
        acc[kk] = exp2f(acc[kk] - mx);
        l += acc[kk];
      }
      const float li = 1.0f / l;
#pragma unroll
      for (int kk = 0; kk < kScoreChunk; ++kk) acc[kk] *= li;
    } else {
#pragma unroll
      for (int kk = 0; kk < kScoreChunk; ++kk) acc[kk] = 0.0f;
    }
    warp_key_sums(acc, lane, s_wsum + warp * kScoreChunk);
    __syncthreads();
    if (tid < kScoreChunk && tid < B) {
      float sum = 0.0f;
      for (int w = 0; w < kRouteThreads / 32; ++w) sum += s_wsum[w * kScoreChunk + tid];
      s_score[tid] = sum;
    }
    finish(s_score);
    return;
  }
  // pass 1: every row's max and normaliser (each thread its rows r = r_lo + tid, + 256, ...)
  float m[kRowsPerThread], linv[kRowsPerThread];
#pragma unroll
  for (int i = 0; i < kRowsPerThread; ++i) { m[i] = -INFINITY; linv[i] = 0.0f; }
  for (int c = 0; c < nchunks; ++c) {
    load_chunk(c);
#pragma unroll 1
    for (int i = 0; i < kRowsPerThread; ++i) {
      const int r = r_lo + tid + i * kRouteThreads;
      if (r >= r_hi) break;
      float qv[D], sv[kScoreChunk];
      load_q(r, qv);
      chunk_logits(qv, c, sv);
      float cm = -INFINITY;
#pragma unroll
      for (int kk = 0; kk < kScoreChunk; ++kk) cm = fmaxf(cm, sv[kk]);
      const float mn = fmaxf(m[i], cm);
      float l = m[i] == -INFINITY ? 0.0f : linv[i] * exp2f(m[i] - mn);  // linv holds the running sum here
#pragma unroll
      for (int kk = 0; kk < kScoreChunk; ++kk) l += exp2f(sv[kk] - mn);
      m[i] = mn;
      linv[i] = l;
    }
  }
#pragma unroll
  for (int i = 0; i < kRowsPerThread; ++i) linv[i] = linv[i] > 0.0f ? 1.0f / linv[i] : 0.0f;
  // pass 2: probabilities summed per key
  for (int c = 0; c < nchunks; ++c) {
    load_chunk(c);
    float acc[kScoreChunk];
#pragma unroll
    for (int kk = 0; kk < kScoreChunk; ++kk) acc[kk] = 0.0f;
#pragma unroll 1
    for (int i = 0; i < kRowsPerThread; ++i) {
      const int r = r_lo + tid + i * kRouteThreads;
      if (r >= r_hi) break;
      float qv[D], sv[kScoreChunk];
      load_q(r, qv);
      chunk_logits(qv, c, sv);
#pragma unroll
      for (int kk = 0; kk < kScoreChunk; ++kk) acc[kk] += exp2f(sv[kk] - m[i]) * linv[i];
    }
    warp_key_sums(acc, lane, s_wsum + warp * kScoreChunk);
    __syncthreads();
    if (tid < kScoreChunk) {
      const int j = c * kScoreChunk + tid;
      float sum = 0.0f;
      for (int w = 0; w < kRouteThreads / 32; ++w) sum += s_wsum[w * kScoreChunk + tid];
      if (j < B) s_score[j] = sum;
    }
  }
  finish(s_score);
}

size_t score_route_smem(int B, int D) {
  return (size_t)kScoreChunk * D * 4 + (size_t)(kRouteThreads / 32) * kScoreChunk * 4 + (size_t)B * 4;
}

// Small problems (few query blocks) split each block's rows over a cluster of up to 8 CTAs so that
// the GPU is filled.
template <int D>
lsrm_status launch_route_score_d(const lsrm_nsa_desc& d, const int32_t* off, const void* q, const float* kc32,
                                 int32_t* idx, float* score, uint32_t* status, cudaStream_t stream, size_t smem,
                                 int n_split) {
  if (cudaFuncSetAttribute(score_route_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return LSRM_ERR_CUDA;
  const float scale = d.scale > 0 ? d.scale : 1.0f / sqrtf((float)D);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)d.n_blocks, (unsigned)d.n_kv_heads, (unsigned)n_split);
  cfg.blockDim = dim3(kRouteThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = (unsigned)n_split;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, score_route_kernel<D>, off, (const uint16_t*)q, kc32, (int32_t)d.n_blocks,
                         (int32_t)d.n_q_heads, (int32_t)d.n_kv_heads, (int32_t)d.top_k, scale, idx, score,
                         status) != cudaSuccess)
    return LSRM_ERR_CUDA;
  return LSRM_OK;
}

lsrm_status launch_route_score(const lsrm_nsa_desc& d, const int32_t* off, const void* q, const float* kc32,
                               int32_t* idx, float* score, uint32_t* status, cudaStream_t stream) {
  const int B = d.n_blocks, D = d.head_dim;
  if ((size_t)d.max_block_len * (d.n_q_heads / d.n_kv_heads) > (size_t)kMaxScoreRows) return LSRM_ERR_UNSUPPORTED;
  const size_t smem = score_route_smem(B, D);
  if (smem > 200 * 1024) return LSRM_ERR_UNSUPPORTED;
  const long long ctas = (long long)B * d.n_kv_heads;
  const int max_rows = d.max_block_len * (d.n_q_heads / d.n_kv_heads);
  int n_split = (int)((148LL * 4 + ctas - 1) / ctas);
  n_split = min(n_split, min(kMaxScoreSplits, (max_rows + kRouteThreads - 1) / kRouteThreads));
  if (n_split < 1) n_split = 1;
  if (d.n_kv_heads > 65535 || n_split > 8) return LSRM_ERR_UNSUPPORTED;
  const lsrm_status st = D == 32 ? launch_route_score_d<32>(d, off, q, kc32, idx, score, status, stream, smem, n_split)
                                 : launch_route_score_d<64>(d, off, q, kc32, idx, score, status, stream, smem, n_split);
  if (st != LSRM_OK) return st;
  return cudaGetLastError() == cudaSuccess ? LSRM_OK : LSRM_ERR_CUDA;
}

// ---- gated combine ---------------------------------------------------------------------------------
// out[t,h,:] = sum_b gates[t,h,b] * o_b[t,h,:]  (bf16 out); one thread per 4 output columns.
__global__ void gate_combine_kernel(const float4* __restrict__ oc, const float4* __restrict__ os,
                                    const float4* __restrict__ ow, const uint16_t* __restrict__ gates,
                                    uint2* __restrict__ out, long long n_vec4, int d4, int ng) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n_vec4;
       i += (long long)gridDim.x * blockDim.x) {
    const long long row = i / d4;
    const uint16_t* g = gates + row * ng;
    const float g0 = bf16_to_f32(g[0]), g1 = bf16_to_f32(g[1]);
    const float4 a = oc[i], b = os[i];
    float4 r = make_float4(g0 * a.x + g1 * b.x, g0 * a.y + g1 * b.y, g0 * a.z + g1 * b.z, g0 * a.w + g1 * b.w);
    if (ow != nullptr && ng >= 3) {
      const float g2 = bf16_to_f32(g[2]);
      const float4 c = ow[i];
      r.x += g2 * c.x; r.y += g2 * c.y; r.z += g2 * c.z; r.w += g2 * c.w;
    }
    uint2 o;
    o.x = pack_bf16x2(r.x, r.y);
    o.y = pack_bf16x2(r.z, r.w);
    out[i] = o;
  }
}

lsrm_status launch_gate_combine(const lsrm_nsa_desc& d, const float* oc, const float* os, const float* ow,
                                const void* gates, void* out, cudaStream_t stream) {
  const long long n_vec4 = d.n_tokens * (long long)d.n_q_heads * d.head_dim / 4;
  const int threads = 256;
  const long long blocks = (n_vec4 + threads - 1) / threads;
  const int grid = (int)(blocks < 148LL * 32 ? blocks : 148LL * 32);
  gate_combine_kernel<<<grid, threads, 0, stream>>>((const float4*)oc, (const float4*)os, (const float4*)ow,
                                                    (const uint16_t*)gates, (uint2*)out, n_vec4, d.head_dim / 4,
                                                    d.n_gates);
  return cudaGetLastError() == cudaSuccess ? LSRM_OK : LSRM_ERR_CUDA;
}

}  // namespace lsrm
