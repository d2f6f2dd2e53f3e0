/*
 * lsrm_nsa.h — C ABI of the B200 (sm_100a) native-sparse-attention layer of the
 * Large Sparse Reconstruction Model (LSRM), plus its Speed3R pooled-query variant.
 *
 * The layer (LSRM page, hyper.ai "LSRM", section 方法):
 *   - active tokens are grouped into spatial blocks (8x8 image tiles, volume
 *     bricks; the block grouping paragraph);
 *   - compression: per-block mean of K and V (equations k^cmp, v^cmp; the
 *     ResBlock before the pool is a trained module and is not part of this ABI);
 *   - routing picks top-k KV blocks per query block, from compressed attention
 *     scores (standard NSA), from 3D distances between block centres, or for
 *     image blocks by projecting the query point into every view (the 3D-aware
 *     routing paragraph);
 *   - a compressed branch, a selected-block branch and an in-block window branch
 *     run softmax attention and a sigmoid-gated sum combines them (gate
 *     equations w = Sigmoid(Linear(x)); the gate VALUES are inputs here);
 *   - the dense blocks' decoupled self/cross gated mixture of the volume and
 *     image streams (the gated cross-attention equations).
 * Speed3R page (gist.science "Speed3R", section 2.1 Global Sparse Attention):
 *   Q/K/V are average-pooled per block, the pooled scores pick the top-k blocks,
 *   the reference frame and camera tokens are always selected (section 2.2), and
 *   a gate mixes the compressed and selected outputs.
 *
 * Notation: N tokens in block-major order; block b owns tokens off[b] .. off[b+1]-1
 * (n_b = off[b+1] - off[b], 1 <= n_b <= max_block_len <= 512: the pages' 8x8x8 volume
 * blocks next to 8x8 image tiles.  The backward, score routing beyond 4096 rows per block and
 * the pooled-query variant take blocks of at most 64 / 64 / 16 tokens and answer
 * LSRM_ERR_UNSUPPORTED otherwise).  Hq query heads,
 * Hkv KV heads, G = Hq / Hkv, query head h reads KV head h / G.  d = head_dim.
 * tau = scale (0 means 1/sqrt(d)).
 *
 * Layouts (all row-major, contiguous):
 *   q      bf16 [N][Hq][d]        k, v   bf16 [N][Hkv][d]
 *   gates  bf16 [N][Hq][n_gates]  order (cmp, slc, win); n_gates = 2 drops win
 *   off    int32 [B+1]            coords int32 [N][3] lattice coordinates
 *   out    bf16 [N][Hq][d]
 *   kc32/vc32 fp32 [B][Hkv][d], kc/vc bf16 [B][Hkv][d] (block means)
 *   qc32/qc fp32/bf16 [B][Hq][d]  (pooled queries, Speed3R only)
 *   idx    int32 [B][idx_heads][top_k]; idx_heads = 1 (geometric: one list per
 *          query block, shared by all KV heads) or Hkv (score routing)
 *   o_* / lse fp32 [N][Hq][d] / [N][Hq]  (per-branch outputs, natural-log LSE)
 *
 * Ownership and errors.  Every array pointer is DEVICE memory owned by the
 * caller; the library allocates nothing and keeps no global state (all scratch
 * lives in the caller's workspace, sized by lsrm_nsa_workspace_size and zeroed
 * once by lsrm_nsa_workspace_init), apart from the fixed centroid array of
 * lsrm_route_geometric_noalloc (see there).  The descriptor itself is host memory.
 * Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL = the
 * legacy default stream).  The return value reports argument validation and
 * launch errors only.  Faults found while running (a routed index outside
 * [0, B), a coordinate outside [-2^29, 2^29], a bounded wait that gave up) are
 * written to a status word in the workspace and read back, then cleared, by
 * lsrm_nsa_last_device_status.  No call traps, asserts or waits without bound.
 */
#ifndef LSRM_NSA_H
#define LSRM_NSA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LSRM_API __attribute__((visibility("default")))
#else
#define LSRM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LSRM_OK = 0,
  LSRM_ERR_INVALID_ARG = 1, /* a pointer, size or shape the call cannot accept */
  LSRM_ERR_UNSUPPORTED = 2, /* valid in principle, not built (e.g. head_dim not 32/64) */
  LSRM_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed */
  LSRM_ERR_TIMEOUT = 4,     /* a device-side bounded wait gave up */
  LSRM_ERR_BOUNDS = 5,      /* a device-side index/coordinate check failed; access skipped */
  LSRM_ERR_WORKSPACE = 6    /* workspace missing, misaligned or too small */
} lsrm_status;

/* route_mode of lsrm_nsa_forward */
enum { LSRM_ROUTE_GIVEN = 0, LSRM_ROUTE_SCORE = 1, LSRM_ROUTE_GEOMETRIC = 2, LSRM_ROUTE_ALL = 3 };

typedef struct {
  int64_t n_tokens;       /* N >= 1 */
  int32_t n_blocks;       /* B >= 1 */
  int32_t max_block_len;  /* upper bound of every n_b, 1..512 */
  int32_t n_q_heads;      /* Hq, multiple of n_kv_heads */
  int32_t n_kv_heads;     /* Hkv >= 1 */
  int32_t head_dim;       /* d in {32, 64} */
  int32_t top_k;          /* routed blocks per query block, 1..B */
  int32_t window;         /* even, 0 switches the window branch off */
  float scale;            /* softmax scale tau; 0 -> 1/sqrt(d) */
  int32_t pooled_q;       /* 0 LSRM layer, 1 Speed3R pooled-query variant (MHA, no window) */
  int32_t n_gates;        /* 3 (cmp, slc, win) or 2 (cmp, slc) */
  int32_t n_forced;       /* blocks every query selects (Speed3R), 0 for LSRM */
  const int32_t* forced_blocks; /* device int32 [n_forced], sorted, distinct */
} lsrm_nsa_desc;

/* Bytes of device workspace the calls below need for this descriptor (a
 * multiple of 256).  Pass the same workspace to every call of one layer. */
LSRM_API size_t lsrm_nsa_workspace_size(const lsrm_nsa_desc* desc);

/* Zero the workspace (status word included).  Call once after allocating it. */
LSRM_API lsrm_status lsrm_nsa_workspace_init(const lsrm_nsa_desc* desc, void* ws, size_t ws_bytes, void* stream);

/* S1 compression (LSRM page, equations k^cmp / v^cmp; Speed3R page 2.1 for the
 * pooled query): per-block means of K and V (and of Q when q != NULL), written
 * in fp32 and rounded to bf16.  Any output pointer may be NULL to skip it. */
LSRM_API lsrm_status lsrm_nsa_compress(const lsrm_nsa_desc* desc, const int32_t* off, const void* q_or_null,
                              const void* k, const void* v, float* kc32, void* kc, float* vc32, void* vc,
                              float* qc32_or_null, void* qc_or_null, void* ws, void* stream);

/* S2a score routing (LSRM page, routing paragraph: NSA picks KV blocks by their
 * attention scores against the compressed keys).  For query block a and KV
 * group g: Score[a,g,j] = sum over tokens t of a and heads h of g of
 * softmax_j(tau * q[t,h] . kc32[j,g]); idx[a][g][:] = the top_k j by
 * (Score desc, j asc).  score_or_null receives fp32 [B][Hkv][B] when given. */
LSRM_API lsrm_status lsrm_route_score_topk(const lsrm_nsa_desc* desc, const int32_t* off, const void* q, const float* kc32,
                                  int32_t* idx, float* score_or_null, void* ws, void* stream);

/* S2b geometric routing (LSRM page, routing paragraph: nearest blocks by 3D
 * Euclidean distance between block centres).  Centroid c[b] per axis =
 * floor((2*S + n_b) / (2*n_b)) with S the sum of the block's coordinates
 * (round half up); D[a,j] = sum over axes of (c[a]-c[j])^2 in int64;
 * idx[a][:] = the top_k j by (D asc, j asc).  coords must lie in [-2^29, 2^29]. */
LSRM_API lsrm_status lsrm_route_geometric(const lsrm_nsa_desc* desc, const int32_t* off, const int32_t* coords,
                                 int32_t* idx, void* ws, void* stream);

/* Camera-projection routing (LSRM page, 方法, 3D-aware routing paragraph: for
 * image blocks the query point is projected into every input view, the view's
 * nearby image blocks are retrieved and ranked by their smallest 3D distance to
 * the query point; volume blocks are ranked by the distance between centres).
 * The query point of block a is its centroid c_a (as lsrm_route_geometric).
 * Blocks [0, n_vol_blocks) are volume blocks, the rest image blocks.
 *   volume part: the k_vol volume blocks nearest to c_a by centroid distance,
 *     ties to the lower id;
 *   image part (k_img = top_k - k_vol): for each view v, h = proj[v] [c_a; 1]
 *     (int64); if h2 > 0 the projected tile is (floor(floor(h0/h2) / tile_px),
 *     floor(floor(h1/h2) / tile_px)) (x = column, y = row) and the blocks
 *     tile_block[v][y'][x'] of the tiles within Chebyshev distance `radius` of
 *     it inside the tiles_x x tiles_y grid are candidates (-1 entries hold no
 *     block); candidates are ranked by min over their tokens of the squared
 *     distance to c_a, ties to the lower id.  When fewer than k_img candidates
 *     exist, the remaining image blocks fill the list by centroid distance.
 * idx (device, int32 [B][top_k]) gets the volume part then the image part, each
 * in rank order; it serves as the shared index list (idx_heads = 1) of the
 * selected branch.  proj (device, int32 [n_views][3][4], any common scale per
 * view: only ratios matter) and tile_block (device, int32
 * [n_views][tiles_y][tiles_x]) are caller-owned; tile_block entries must be
 * image block ids or -1 (others raise LSRM_ERR_BOUNDS in the device status and
 * are skipped).  Errors: LSRM_ERR_INVALID_ARG for counts outside their ranges
 * (k_vol > n_vol_blocks, k_img > B - n_vol_blocks, tile_px < 1, radius < 0);
 * LSRM_ERR_UNSUPPORTED for more than 4096 (view, tile) neighbourhood slots
 * or more image blocks than the per-CTA bitmap holds (over a million).
 * Coordinates beyond +-2^29 raise LSRM_ERR_BOUNDS. */
LSRM_API lsrm_status lsrm_route_camera(const lsrm_nsa_desc* desc, const int32_t* off, const int32_t* coords,
                                       int32_t n_vol_blocks, int32_t n_views, const int32_t* proj,
                                       int32_t tiles_x, int32_t tiles_y, int32_t tile_px,
                                       const int32_t* tile_block, int32_t radius, int32_t k_vol, int32_t* idx,
                                       void* ws, void* stream);

/* Geometric routing that allocates nothing and takes no workspace, for callers that may
 * not allocate device memory at call time and have none to lend (for example a plugin in
 * a host framework whose memory pool owns the whole GPU, or a loop whose policy forbids
 * allocation after start-up).  The pages have no counterpart of this call; it accepts the
 * same descriptors as lsrm_route_geometric (the same checks, same status codes) and
 * computes exactly what it computes.  Its centroid scratch is a fixed array in the
 * library's own device memory (192 KiB, held on every GPU that loads the library until
 * the process exits), so n_blocks may be at most 16384; larger descriptors are rejected
 * with LSRM_ERR_WORKSPACE.  Every call looks up that array's address on the current
 * device (a host-side query that allocates nothing; no address is cached across calls, so
 * a device reset cannot leave a stale one).  The first call on a device may load the
 * library's device code there, so make it before any stream capture.  Every call shares
 * the one array: calls that may overlap on the GPU (different streams, or different host
 * threads on one device) race and must be serialised by the caller.
 * status_or_null (device uint32, may be NULL) receives LSRM_ERR_BOUNDS as bit
 * (1 << (LSRM_ERR_BOUNDS - 1)) OR-ed in when a coordinate lies outside [-2^29, 2^29];
 * the caller clears it. */
LSRM_API lsrm_status lsrm_route_geometric_noalloc(const lsrm_nsa_desc* desc, const int32_t* off,
                                                  const int32_t* coords, int32_t* idx, uint32_t* status_or_null,
                                                  void* stream);

/* Speed3R routing (Speed3R page 2.1 selection branch, 2.2 forced frame-0 and
 * camera blocks): per block a and head h, the top_k blocks j outside the forced
 * set by (tau * qc[a,h] . kc[j,h] desc, j asc).  qc / kc are the bf16 pooled
 * tensors [B][H][d] the tensor cores score with.  With qc32_or_null and
 * kc32_or_null (both or neither; fp32 [B][H][64], 16-byte aligned) the ranking is
 * that of the fp32 pooled means themselves: candidates are gathered from the bf16
 * logits with a gate widened by a bound on their error (2^-7 |qc32|_2 max_j |kc32_j|_2)
 * and ranked by fp32 dot products of the means; without them it is the ranking of
 * the bf16 operands, products accumulated in fp32.  idx is int32 [B][Hq][top_k]
 * (top_k at most 64, else LSRM_ERR_UNSUPPORTED; a row with fewer eligible blocks
 * pads with -1). */
LSRM_API lsrm_status lsrm_route_pooled_topk(const lsrm_nsa_desc* desc, const void* qc, const void* kc,
                                   const float* qc32_or_null, const float* kc32_or_null, int32_t* idx,
                                   void* ws, void* stream);

/* S3 compressed branch (LSRM page, k^cmp/v^cmp give the global coarse context;
 * Speed3R page 2.1 compression branch).  o_cmp[t,h] = sum_j softmax_j(tau *
 * q[t,h] . kc[j,g]) vc[j,g] over all B blocks; with pooled_q the query is
 * qc[beta(t),h] (pass it as q, shape [B][Hq][d]) and the block's output is
 * written to every token of the block.  kc/vc are bf16 block means. */
LSRM_API lsrm_status lsrm_nsa_cmp_attn(const lsrm_nsa_desc* desc, const int32_t* off, const void* q, const void* kc,
                              const void* vc, float* o_cmp, float* lse, void* ws, void* stream);

/* S4 selected branch (LSRM page: selected active blocks give fine detail;
 * Speed3R page 2.1 selection branch).  Softmax attention of q[t,h] over every
 * token of the blocks idx[beta(t)][g or 0][0..top_k-1] plus the forced blocks.
 * idx_heads is 1 or Hkv (see Layouts); rows must hold distinct block ids that
 * are not forced. */
LSRM_API lsrm_status lsrm_nsa_select_attn(const lsrm_nsa_desc* desc, const int32_t* off, const void* q, const void* k,
                                 const void* v, const int32_t* idx, int32_t idx_heads, float* o_slc, float* lse,
                                 void* ws, void* stream);

/* S5 window branch (LSRM page, sequence-parallel paragraph: window attention
 * runs locally inside whole blocks).  W(t) = { u in beta(t) : r(t) - w/2 <=
 * r(u) <= r(t) + w/2 - 1 }, r = position inside the block. */
LSRM_API lsrm_status lsrm_nsa_window_attn(const lsrm_nsa_desc* desc, const int32_t* off, const void* q, const void* k,
                                 const void* v, float* o_win, float* lse, void* ws, void* stream);

/* S6 gated combine (LSRM page, gate equations; Speed3R page 2.1 gated
 * aggregation): out = g_cmp o_cmp + g_slc o_slc (+ g_win o_win), bf16 out. */
LSRM_API lsrm_status lsrm_nsa_gate_combine(const lsrm_nsa_desc* desc, const float* o_cmp, const float* o_slc,
                                  const float* o_win_or_null, const void* gates, void* out, void* stream);

/* S3+S4+S5+S6 fused: the three attention branches and the gated combine in one
 * kernel (one CTA per query block, KV group and 128-row chunk), given the bf16
 * block means kc/vc (lsrm_nsa_compress) and the routing indices (idx_heads 1 or
 * Hkv; route_all = 1 selects every block and ignores idx).  Writes bf16 out and,
 * when lse_or_null is given, the per-branch LSE [N][Hq][n_gates].  For pooled_q
 * this call is not available (use lsrm_nsa_forward). */
LSRM_API lsrm_status lsrm_nsa_attend(const lsrm_nsa_desc* desc, const int32_t* off, const void* q, const void* k,
                                     const void* v, const void* kc, const void* vc, const void* gates,
                                     const int32_t* idx, int32_t idx_heads, int32_t route_all, void* out,
                                     float* lse_or_null, void* ws, void* stream);

/* Decoupled self/cross gated mixture (LSRM page, 方法: the dense transformer
 * blocks' gated cross-attention equations, o^x = w^{x-self} CrossAttn(x, x) +
 * w^{x-cross} CrossAttn(x, y) and o^y likewise with x and y swapped).  The
 * concatenated tokens hold two streams: blocks [0, n_blocks_x) are x (volume
 * tokens) and blocks [n_blocks_x, B) are y (image tokens).  For a token t of one
 * stream and head h (KV group g = h / (Hq/Hkv)):
 *   out[t,h] = gates[t,h,0] * softmax-attention of q[t,h] over every token of
 *              its own stream + gates[t,h,1] * the same over every token of the
 *              other stream,
 * one kernel launch (both attentions and the gated sum; an empty other stream
 * contributes 0).  q [N][Hq][d], k/v [N][Hkv][d], gates [N][Hq][2] (self,
 * cross), out [N][Hq][d], all bf16, 16-byte aligned; lse_or_null receives fp32
 * [N][Hq][2] (natural log; -inf for an empty stream).  desc: n_gates = 2,
 * pooled_q = 0, n_forced = 0; top_k and window are not used (top_k must still be
 * valid).  Blocks of any length up to 512 tokens.  Errors: LSRM_ERR_INVALID_ARG
 * for a bad descriptor, pointer, alignment or n_blocks_x outside [0, B];
 * LSRM_ERR_UNSUPPORTED when 128 is not a multiple of Hq/Hkv.  The gates are
 * inputs: the Sigmoid(Linear) that makes them is a trained layer. */
LSRM_API lsrm_status lsrm_nsa_mixture(const lsrm_nsa_desc* desc, const int32_t* off, int32_t n_blocks_x,
                                      const void* q, const void* k, const void* v, const void* gates, void* out,
                                      float* lse_or_null, void* ws, void* stream);

/* S7 the fused layer forward: compression, routing (route_mode), then the three
 * branches and the gated combine in one attention kernel whose epilogue writes
 * out.  route_mode: LSRM_ROUTE_GIVEN reads idx_inout as [B][Hkv][top_k];
 * LSRM_ROUTE_SCORE writes it as [B][Hkv][top_k]; LSRM_ROUTE_GEOMETRIC (coords
 * required) writes [B][top_k]; LSRM_ROUTE_ALL needs top_k == B and selects every
 * block (idx_inout may be NULL).  With a NULL idx_inout the indices live in the
 * workspace.  For pooled_q (top_k at most 64, blocks of at most 16 tokens,
 * head_dim 64) the routing is the Speed3R rule and idx_inout is
 * [B][Hq][top_k], ranked by the fp32 logits of the pooled means (as
 * lsrm_route_pooled_topk with fp32 inputs).
 * lse_or_null receives fp32 [N][Hq][n_gates] per-branch LSE (needed by the
 * backward).  obr_or_null (device, 16-byte aligned, caller-owned) receives the
 * normalised per-branch outputs o_b as bf16 [N][Hq][n_gates][d], the
 * activations that let the backward skip recomputing <dO, o_b>; it must be NULL
 * for pooled_q (LSRM_ERR_UNSUPPORTED otherwise). */
LSRM_API lsrm_status lsrm_nsa_forward(const lsrm_nsa_desc* desc, const int32_t* off, const void* q, const void* k,
                             const void* v, const void* gates, const int32_t* coords_or_null, int32_t route_mode,
                             void* out, int32_t* idx_inout, float* lse_or_null, void* obr_or_null, void* ws,
                             void* stream);

/* S10 backward of the layer with routing indices fixed:
 * dq, dgates [N][Hq][.], dk, dv [N][Hkv][d] (bf16) of L = sum(out * dout),
 * through the gated sum, the three softmax branches and the block mean.
 * lse is the forward's per-branch LSE.  idx_heads as in lsrm_nsa_select_attn.
 * obr_or_null: the forward's saved branch outputs (see lsrm_nsa_forward).  With
 * them dgates_b = <dO, o_b> and Delta_b = g_b dgates_b are read off directly and
 * every branch is streamed once; with NULL they are recomputed in an extra pass
 * over each branch (P dP summed in fp32).  dout and obr must be 16-byte aligned.
 * With pooled_q (the Speed3R layer, Speed3R page section 2: trained end to end)
 * idx is the forward's [B][Hq][top_k] routing (idx_heads = Hq), lse its
 * [N][Hq][2] output and obr_or_null is required (LSRM_ERR_INVALID_ARG without
 * it): the chain rule runs through the pooled query (dQbar / n_b to every token
 * of the block), the copy of the pooled output to the block's tokens, the joint
 * softmax of the forced and routed keys and the two gates; all sums have a fixed
 * order, so results are reproducible bit for bit. */
LSRM_API lsrm_status lsrm_nsa_backward(const lsrm_nsa_desc* desc, const int32_t* off, const void* q, const void* k,
                              const void* v, const void* gates, const int32_t* idx, int32_t idx_heads,
                              const float* lse, const void* obr_or_null, const void* dout, void* dq, void* dk,
                              void* dv, void* dgates, void* ws, void* stream);

/* Diagnostic (no counterpart in the pages): y[i] = 2^x[i] as the attention kernels' FMA-pipe
 * polynomial computes it (the exponentials of the softmax that do not go to the hardware ex2).
 * x and y are device float arrays of n elements (caller-owned); valid for x <= 127, and inputs
 * below -125 return about 2^-125.  Lets a test compare the polynomial with CUDA's exp2f over
 * its whole range; not part of the layer. */
LSRM_API lsrm_status lsrm_diag_exp2_poly(const float* x, float* y, int64_t n, void* stream);

/* Read (synchronising `stream`) and clear the device status word of the workspace. */
LSRM_API lsrm_status lsrm_nsa_last_device_status(void* ws, void* stream);

/* Static text for a status code. */
LSRM_API const char* lsrm_status_string(lsrm_status s);

#ifdef __cplusplus
}
#endif
#endif /* LSRM_NSA_H */
