"""Pins for the fp64 oracle: each check compares it with something other than itself —
a closed form, a library routine (torch's fp64 scaled_dot_product_attention, numpy
reductions and sorts), number theory, an invariant of the definition, or finite
differences — chosen so that a dropped term, a wrong sign or index, or a transposed
operand anywhere in the oracle fails at least one of them."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as O
from conftest import golden
from workloads import make_workload, lsrm_layout, speed3r_layout, bf16_bits_to_f32
from workloads.nsa_workloads import normal_bf16, f32_to_bf16_bits, speed3r_forced, sigmoid_normal_bf16


def f64(bits):
    return bf16_bits_to_f32(np.asarray(bits)).astype(np.float64)


def desc(w, **kw):
    args = dict(n_tokens=w.n_tokens, n_blocks=w.n_blocks, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                head_dim=w.head_dim, top_k=w.top_k, window=w.window, n_gates=w.n_gates, pooled_q=w.pooled_q)
    args.update(kw)
    return O.desc_for(**args)


def sdpa(q, k, v, mask=None, scale=None):
    """torch fp64 attention: q [T,H,d], k/v [S,Hk,d] with contiguous head groups."""
    G = q.shape[1] // k.shape[1]
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    kt = torch.from_numpy(k).repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
    vt = torch.from_numpy(v).repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
    m = None if mask is None else torch.from_numpy(mask)
    o = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=scale)
    return o[0].permute(1, 0, 2).numpy()


def small_layout_workload(sizes, hq=4, hkv=2, d=8, seed=0, k=2, w=4, ng=3):
    """A hand-made layout with the given block sizes (ragged allowed)."""
    off = np.zeros(len(sizes) + 1, dtype=np.int32)
    off[1:] = np.cumsum(sizes)
    n = int(off[-1])
    q = normal_bf16(seed, 0, (n, hq, d), 1.0)
    kk = normal_bf16(seed, 1, (n, hkv, d), 1.0)
    v = normal_bf16(seed, 2, (n, hkv, d), 1.0)
    g = sigmoid_normal_bf16(seed, 3, (n, hq, ng))
    D = O.desc_for(n, len(sizes), hq, hkv, d, k, w, n_gates=ng)
    return D, off, q, kk, v, g


# ------------------------------------------------------------------------------------------------
# S1 compression
# ------------------------------------------------------------------------------------------------

def test_compress_matches_numpy_reduceat_on_ragged_blocks():
    sizes = [3, 1, 7, 64, 2, 5]
    D, off, q, k, v, g = small_layout_workload(sizes)
    kc = O.compress(D, off, k, D.n_kv_heads)
    ref = np.add.reduceat(f64(k), off[:-1], axis=0) / np.array(sizes)[:, None, None]
    assert np.allclose(kc, ref, rtol=0, atol=1e-14)


def test_compress_of_constant_block_is_the_constant():
    sizes = [4, 9, 1]
    D, off, q, k, v, g = small_layout_workload(sizes)
    const = np.empty_like(k)
    for b in range(3):
        const[off[b]:off[b + 1]] = f32_to_bf16_bits(np.full((sizes[b],) + k.shape[1:], 0.25 * (b + 1), np.float32))
    kc = O.compress(D, off, const, D.n_kv_heads)
    for b in range(3):
        assert np.all(kc[b] == 0.25 * (b + 1))


# ------------------------------------------------------------------------------------------------
# S3/S4/S5 attention branches
# ------------------------------------------------------------------------------------------------

def test_every_branch_returns_a_constant_value_exactly():
    # softmax weights sum to 1 in every branch: a constant V comes back unchanged
    sizes = [5, 8, 3, 8]
    D, off, q, k, v, g = small_layout_workload(sizes, k=2, w=4)
    vconst = np.empty_like(v)
    vconst[...] = f32_to_bf16_bits(np.linspace(-1, 1, v.shape[2], dtype=np.float32))[None, None, :]
    idx = np.array([[0, 1], [1, 2], [2, 3], [3, 0]], dtype=np.int32)
    out, br, lse = O.forward(D, off, q, k, vconst, g, idx, want_branches=True)
    want = f64(vconst[0, 0])
    for b in range(3):
        assert np.allclose(br[:, :, b, :], want[None, None, :], atol=1e-12, rtol=0)


def test_dense_reduction_equals_sdpa():
    # k = B, gates (0, 1, 0): the layer is plain GQA softmax attention over all tokens
    w = make_workload("tiny", top_k=16)
    D = desc(w)
    idx = np.tile(np.arange(16, dtype=np.int32), (16, 1))
    gates = np.zeros_like(w.gates)
    gates[..., 1] = f32_to_bf16_bits(np.array([1.0], np.float32))[0]
    qb = np.array([0, 5, 11, 15], dtype=np.int32)
    out = O.forward(D, w.off, w.q, w.k, w.v, gates, idx, qblocks=qb)
    rows = np.concatenate([np.arange(w.off[b], w.off[b + 1]) for b in qb])
    ref = sdpa(f64(w.q)[rows], f64(w.k), f64(w.v))
    assert np.abs(out - ref).max() < 1e-12


def test_selected_branch_with_partial_selection_equals_sdpa_on_the_union():
    sizes = [6, 3, 8, 5, 7]
    D, off, q, k, v, g = small_layout_workload(sizes, hq=6, hkv=3, d=8, k=2)
    idx = np.array([[[4, 1], [0, 2], [3, 3]]] * 5, dtype=np.int32)  # per group; duplicates count once
    idx[2] = [[2, 0], [4, 3], [1, 2]]
    o, lse = O.select_attn(D, off, q, k, v, idx)
    qf, kf, vf = f64(q), f64(k), f64(v)
    for a in range(5):
        for g_ in range(3):
            blocks = sorted(set(idx[a, g_].tolist()))
            keys = np.concatenate([np.arange(off[j], off[j + 1]) for j in blocks])
            rows = np.arange(off[a], off[a + 1])
            ref = sdpa(qf[rows][:, 2 * g_:2 * g_ + 2], kf[keys][:, g_:g_ + 1], vf[keys][:, g_:g_ + 1])
            assert np.abs(o[rows][:, 2 * g_:2 * g_ + 2] - ref).max() < 1e-12
            # LSE: log-sum-exp of the scaled logits (torch.logsumexp)
            s = torch.einsum("thd,ud->thu", torch.from_numpy(qf[rows][:, 2 * g_:2 * g_ + 2]),
                             torch.from_numpy(kf[keys][:, g_])) / math.sqrt(8)
            assert np.abs(lse[rows][:, 2 * g_:2 * g_ + 2] - torch.logsumexp(s, -1).numpy()).max() < 1e-12


def test_single_block_compressed_branch_is_the_block_mean():
    sizes = [13]
    D, off, q, k, v, g = small_layout_workload(sizes, k=1)
    kc = O.compress(D, off, k, 2)
    vc = O.compress(D, off, v, 2)
    o, lse = O.cmp_attn(D, off, q, kc, vc)
    assert np.allclose(o, np.repeat(vc[0][None], 13, 0).repeat(2, axis=1), atol=1e-15)
    # one key: LSE = its logit
    qf = f64(q)
    logit = np.einsum("thd,thd->th", qf, np.repeat(kc[0][None], 13, 0).repeat(2, axis=1)) / math.sqrt(8)
    assert np.allclose(lse, logit, atol=1e-14)


def test_compressed_branch_equals_sdpa_over_block_means():
    w = make_workload("tiny")
    D = desc(w)
    kc = O.compress(D, w.off, w.k, 2)
    vc = O.compress(D, w.off, w.v, 2)
    o, _ = O.cmp_attn(D, w.off, w.q, kc, vc, qblocks=[3, 9])
    rows = np.r_[np.arange(192, 256), np.arange(576, 640)]
    # block means computed independently by numpy
    kn = f64(w.k).reshape(16, 64, 2, 32).mean(1)
    vn = f64(w.v).reshape(16, 64, 2, 32).mean(1)
    ref = sdpa(f64(w.q)[rows], kn, vn)
    assert np.abs(o - ref).max() < 1e-12


def test_wide_window_is_whole_block_attention():
    sizes = [7, 12, 1, 9]
    D, off, q, k, v, g = small_layout_workload(sizes, w=24)
    o, _ = O.window_attn(D, off, q, k, v)
    qf, kf, vf = f64(q), f64(k), f64(v)
    for a in range(4):
        r = np.arange(off[a], off[a + 1])
        assert np.abs(o[r] - sdpa(qf[r], kf[r], vf[r])).max() < 1e-12


def test_window_of_two_is_a_two_way_softmax():
    # w = 2 keeps r(u) in {r(t) - 1, r(t)}: the first token sees only itself; the others mix two values
    sizes = [5, 4]
    D, off, q, k, v, g = small_layout_workload(sizes, hq=2, hkv=1, d=4, w=2)
    o, _ = O.window_attn(D, off, q, k, v)
    qf, kf, vf = f64(q), f64(k), f64(v)
    tau = 0.5
    for a in range(2):
        t0 = off[a]
        assert np.array_equal(o[t0], np.repeat(vf[t0], 2, axis=0))
        for t in range(t0 + 1, off[a + 1]):
            for h in range(2):
                s_own = tau * qf[t, h] @ kf[t, 0]
                s_prev = tau * qf[t, h] @ kf[t - 1, 0]
                wprev = 1.0 / (1.0 + math.exp(s_own - s_prev))  # logistic form of a 2-way softmax
                want = wprev * vf[t - 1, 0] + (1 - wprev) * vf[t, 0]
                assert np.abs(o[t, h] - want).max() < 1e-14


def test_window_band_on_64_token_blocks():
    # w = 64 on a 64-token block: row r sees r' in [r-32, r+31]; the band width is 32..64 keys
    w = make_workload("tiny")
    D = desc(w)
    o, _ = O.window_attn(D, w.off, w.q, w.k, w.v, qblocks=[2])
    r = np.arange(128, 192)
    qf, kf, vf = f64(w.q)[r], f64(w.k)[r], f64(w.v)[r]
    pos = np.arange(64)
    mask = (pos[None, :] >= pos[:, None] - 32) & (pos[None, :] <= pos[:, None] + 31)
    assert mask.sum(1).min() == 32 and mask.sum(1).max() == 64
    # sdpa with a boolean mask over all heads: mask [T, S] broadcasts over heads
    ref = sdpa(qf, kf, vf, mask=mask[None])
    assert np.abs(o - ref).max() < 1e-12


def test_gated_combine_is_linear_in_the_gates():
    sizes = [4, 6, 5]
    D, off, q, k, v, g = small_layout_workload(sizes, k=2)
    idx = np.array([[0, 1], [1, 2], [2, 0]], dtype=np.int32)
    out, br, _ = O.forward(D, off, q, k, v, g, idx, want_branches=True)
    gf = f64(g)
    assert np.abs(out - np.einsum("thb,thbd->thd", gf, br)).max() < 1e-14
    # one-hot gates select a single branch
    for b in range(3):
        oh = np.zeros_like(g)
        oh[..., b] = f32_to_bf16_bits(np.array([1.0], np.float32))[0]
        ob = O.forward(D, off, q, k, v, oh, idx)
        assert np.abs(ob - br[:, :, b]).max() == 0.0


# ------------------------------------------------------------------------------------------------
# block permutation
# ------------------------------------------------------------------------------------------------

def _permute_blocks(off, perm, *tensors):
    sizes = np.diff(off)
    new_sizes = sizes[perm]
    new_off = np.zeros_like(off)
    new_off[1:] = np.cumsum(new_sizes)
    tok = np.concatenate([np.arange(off[b], off[b + 1]) for b in perm])
    return (new_off, tok) + tuple(t[tok] for t in tensors)


def test_block_permutation_equivariance_score_routing():
    w = make_workload("tiny")
    D = desc(w)
    kc = O.compress(D, w.off, w.k, 2)
    idx, score = O.route_score(D, w.off, w.q, kc)
    srt = np.sort(score, axis=2)[:, :, ::-1]
    assert (srt[:, :, 3] - srt[:, :, 4]).min() > 1e-9  # no ties at the k-th place
    out = O.forward(D, w.off, w.q, w.k, w.v, w.gates, idx)
    rng = np.random.default_rng(5)
    perm = rng.permutation(16)
    off2, tok, q2, k2, v2, g2 = _permute_blocks(w.off, perm, w.q, w.k, w.v, w.gates)
    kc2 = O.compress(D, off2, k2, 2)
    idx2, score2 = O.route_score(D, off2, q2, kc2)
    inv = np.argsort(perm)
    # routing permutes: new block i is old block perm[i]; its selected set maps through perm
    for i in range(16):
        for g_ in range(2):
            assert set(perm[idx2[i, g_]].tolist()) == set(idx[perm[i], g_].tolist())
    out2 = O.forward(D, off2, q2, k2, v2, g2, idx2)
    assert np.abs(out2 - out[tok]).max() < 1e-12
    assert inv.shape == (16,)


def test_block_permutation_equivariance_geometric_routing():
    w = make_workload("ragged_geo")
    D = desc(w)
    idx, cen = O.route_geometric(D, w.off, w.coords)
    rng = np.random.default_rng(11)
    perm = rng.permutation(w.n_blocks)
    off2, tok, c2 = _permute_blocks(w.off, perm, w.coords)
    idx2, cen2 = O.route_geometric(D, off2, c2)
    assert np.array_equal(cen2, cen[perm])
    # the multiset of selected distances is tie-invariant
    def dist(c, a, js):
        return sorted(((c[js] - c[a]) ** 2).sum(1).tolist())
    for i in range(w.n_blocks):
        assert dist(cen2, i, idx2[i]) == dist(cen, perm[i], idx[perm[i]])


# ------------------------------------------------------------------------------------------------
# S2b geometric routing
# ------------------------------------------------------------------------------------------------

def test_geometric_routing_matches_numpy_brute_force():
    for name in ("ragged_geo", "tiny_geo"):
        w = make_workload(name)
        D = desc(w)
        idx, cen = O.route_geometric(D, w.off, w.coords)
        sizes = np.diff(w.off).astype(np.int64)
        sums = np.add.reduceat(w.coords.astype(np.int64), w.off[:-1], axis=0)
        # round half up of sums / n with numpy's floor division
        c = np.floor_divide(2 * sums + sizes[:, None], 2 * sizes[:, None])
        assert np.array_equal(c, cen)
        d2 = ((c[:, None, :] - c[None, :, :]) ** 2).sum(-1)
        for a in range(w.n_blocks):
            order = np.lexsort((np.arange(w.n_blocks), d2[a]))  # distance asc, then index asc
            assert np.array_equal(order[: w.top_k], idx[a])


def test_geometric_routing_regular_grid_follows_three_square_counts():
    r3 = [int(x) for x in golden("r3_counts.txt")[0]]
    # a 9x9x9 grid of full bricks: the centre brick's neighbours by squared distance (in units of
    # the brick pitch, 64 lattice units) come in shells of r3(n)
    lay = lsrm_layout(36, 0, 8, None, None)
    B = lay.n_blocks
    assert B == 729
    D = O.desc_for(lay.n_tokens, B, 1, 1, 1, B, 0)
    idx, cen = O.route_geometric(D, lay.off, lay.coords)
    centre = 4 + 9 * (4 + 9 * 4)
    d = ((cen[idx[centre]] - cen[centre]) ** 2).sum(1)
    assert np.all(d % (64 * 64) == 0)
    n = d // (64 * 64)
    counts = np.bincount(n[n <= 16], minlength=17)
    assert counts.tolist() == r3[:17]
    # top-16: itself, the 6 face neighbours, then the 9 lowest-index of the 12 edge neighbours
    D16 = O.desc_for(lay.n_tokens, B, 1, 1, 1, 16, 0)
    idx16, _ = O.route_geometric(D16, lay.off, lay.coords)
    top = idx16[centre]
    assert top[0] == centre
    assert set(top[1:7].tolist()) == {centre + s for s in (1, -1, 9, -9, 81, -81)}
    edge = sorted(centre + a + b for a in (1, -1) for b in (9, -9)) + \
        sorted(centre + a + b for a in (1, -1) for b in (81, -81)) + \
        sorted(centre + a + b for a in (9, -9) for b in (81, -81))
    assert top[7:].tolist() == sorted(edge)[:9]


# ------------------------------------------------------------------------------------------------
# S2a score routing
# ------------------------------------------------------------------------------------------------

def test_score_routing_ties_and_a_dominant_block():
    w = make_workload("tiny")
    D = desc(w)
    kc = np.zeros((16, 2, 32))
    idx, score = O.route_score(D, w.off, w.q, kc)
    assert np.all(idx == np.arange(4)[None, None, :])            # all equal -> lowest indices
    assert np.allclose(score, 64 * 16 / 16.0)                     # uniform p = 1/16 summed over 1024 rows
    # make every query point along e0 and block 9's key large along e0 for group 1 only
    q = np.zeros_like(w.q)
    q[..., 0] = f32_to_bf16_bits(np.array([1.0], np.float32))[0]
    kc2 = np.zeros((16, 2, 32))
    kc2[9, 1, 0] = 5.0
    kc2[12, 1, 0] = 2.0
    idx2, _ = O.route_score(D, w.off, q, kc2)
    assert np.all(idx2[:, 1, :2] == [9, 12]) and np.all(idx2[:, 1, 2:] == [0, 1])
    assert np.all(idx2[:, 0, :] == np.arange(4))


def test_score_rows_sum_to_tokens_times_heads_per_group():
    w = make_workload("ragged_geo", top_k=3)
    D = desc(w)
    kc = O.compress(D, w.off, w.k, 2)
    idx, score = O.route_score(D, w.off, w.q, kc, qblocks=[0, 7, 61])
    n = np.diff(w.off)[[0, 7, 61]]
    assert np.allclose(score.sum(2), (n * 16)[:, None], rtol=0, atol=1e-9)
    for i in range(3):
        for g_ in range(2):
            order = np.lexsort((np.arange(w.n_blocks), -score[i, g_]))
            assert np.array_equal(order[:3], idx[i, g_])


# ------------------------------------------------------------------------------------------------
# Speed3R variant
# ------------------------------------------------------------------------------------------------

def test_speed3r_all_blocks_selected_is_dense_mha():
    w = make_workload("speed3r_small", n_frames=3)
    B = w.n_blocks
    forced = w.forced
    nonforced = np.setdiff1d(np.arange(B), forced).astype(np.int32)
    D = desc(w, top_k=len(nonforced))
    idx = np.tile(nonforced, (B, w.n_q_heads, 1)).astype(np.int32)
    gates = np.zeros_like(w.gates)
    gates[..., 1] = f32_to_bf16_bits(np.array([1.0], np.float32))[0]
    qb = np.array([0, 57, B - 1], dtype=np.int32)
    out = O.forward(D, w.off, w.q, w.k, w.v, gates, idx, forced=forced, qblocks=qb)
    rows = np.concatenate([np.arange(w.off[b], w.off[b + 1]) for b in qb])
    ref = sdpa(f64(w.q)[rows], f64(w.k), f64(w.v))
    assert np.abs(out - ref).max() < 1e-12


def test_speed3r_pooled_branch_and_routing():
    w = make_workload("speed3r_small", n_frames=4)
    D = desc(w)
    qc = O.compress(D, w.off, w.q, 16)
    kc = O.compress(D, w.off, w.k, 16)
    vc = O.compress(D, w.off, w.v, 16)
    qb = np.array([5, 101, 203, 300], dtype=np.int32)
    o, _ = O.cmp_attn(D, w.off, w.q, kc, vc, qc=qc, qblocks=qb)
    r0 = 0
    for b in qb:
        n = w.off[b + 1] - w.off[b]
        ref = sdpa(qc[b][None], kc, vc)[0]  # one pooled query per head over all block means
        assert np.abs(o[r0:r0 + n] - ref[None]).max() < 1e-12
        r0 += n
    idx, logits = O.route_pooled(D, qc, kc, w.forced, qblocks=qb, want_logits=True)
    ref_logits = np.einsum("hd,jhd->hj", qc[qb[1]], kc) / 8.0
    assert np.abs(logits[1] - ref_logits).max() < 1e-14
    forced = set(w.forced.tolist())
    for i in range(len(qb)):
        for h in range(16):
            assert not (set(idx[i, h].tolist()) & forced)
            lg = logits[i, h].copy()
            lg[list(forced)] = -np.inf
            order = np.lexsort((np.arange(w.n_blocks), -lg))
            assert np.array_equal(order[:32], idx[i, h])


def test_speed3r_routing_ties_go_to_the_lowest_non_forced_blocks():
    # Speed3R page, section 2.1 (top-k of the pooled logits) and 2.2 (frame 0 and the camera
    # blocks always selected, so never routed): with every pooled key equal, all logits of a row
    # tie and the routing must be the k lowest non-forced block ids; a block whose pooled key is
    # that key scaled up must come first whenever the row's logit on it is positive.
    w = make_workload("speed3r_small", n_frames=3)
    D = desc(w)
    rng = np.random.default_rng(11)
    qc = rng.standard_normal((w.n_blocks, 16, w.head_dim))
    u = rng.standard_normal((16, w.head_dim))
    kc = np.broadcast_to(u, (w.n_blocks, 16, w.head_dim)).copy()
    forced = set(w.forced.tolist())
    free = [b for b in range(w.n_blocks) if b not in forced]
    qb = np.array([0, 7, 150, w.n_blocks - 1], dtype=np.int32)
    idx, _ = O.route_pooled(D, qc, kc, w.forced, qblocks=qb)
    for i in range(len(qb)):
        for h in range(16):
            assert idx[i, h].tolist() == free[:32], (i, h)
    star = free[40]  # a late non-forced block
    kc[star] = 3.0 * u
    idx, _ = O.route_pooled(D, qc, kc, w.forced, qblocks=qb)
    for i, a in enumerate(qb):
        for h in range(16):
            lu = float(qc[a, h] @ u[h])
            if lu > 1e-9:
                assert idx[i, h, 0] == star and idx[i, h, 1:].tolist() == [b for b in free if b != star][:31]
            elif lu < -1e-9:
                assert star not in idx[i, h].tolist() and idx[i, h].tolist() == free[:32]


# ------------------------------------------------------------------------------------------------
# S10 backward
# ------------------------------------------------------------------------------------------------

def _fd_case(seed=0):
    sizes = [6, 4, 7, 5]
    D, off, q, k, v, g = small_layout_workload(sizes, hq=4, hkv=2, d=4, seed=seed, k=2, w=4)
    idx = np.array([[0, 2], [1, 3], [2, 0], [3, 1]], dtype=np.int32)
    rng = np.random.default_rng(seed)
    qf, kf, vf, gf = f64(q), f64(k), f64(v), f64(g)
    dout = rng.standard_normal(qf.shape)
    return D, off, qf, kf, vf, gf, idx, dout


def test_backward_matches_central_finite_differences():
    D, off, qf, kf, vf, gf, idx, dout = _fd_case()
    dq, dk, dv, dg = O.backward_f64(D, off, qf, kf, vf, gf, idx, dout)
    rng = np.random.default_rng(1)
    h = 1e-6
    arrays = {"q": (qf, dq), "k": (kf, dk), "v": (vf, dv), "g": (gf, dg)}
    for name, (x, grad) in arrays.items():
        for _ in range(12):
            i = tuple(rng.integers(0, s) for s in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[i] += h
            xm[i] -= h
            args = {"q": qf, "k": kf, "v": vf, "g": gf}
            ap = dict(args, **{name: xp})
            am = dict(args, **{name: xm})
            lp = O.loss_f64(D, off, ap["q"], ap["k"], ap["v"], ap["g"], idx, dout)
            lm = O.loss_f64(D, off, am["q"], am["k"], am["v"], am["g"], idx, dout)
            fd = (lp - lm) / (2 * h)
            assert abs(fd - grad[i]) < 1e-7 * max(1.0, abs(fd)), (name, i, fd, grad[i])


def test_gate_gradient_is_the_inner_product_with_the_branch_output():
    # out = sum_b g_b o_b with o_b independent of the gates, so dL/dg_b = <dO, o_b> for every
    # (token, head): the backward's gate gradient against the forward's own branch outputs, at
    # every entry (the identity the saved-output backward reads dgates from)
    D, off, qf, kf, vf, gf, idx, dout = _fd_case(5)
    _, _, _, dg = O.backward_f64(D, off, qf, kf, vf, gf, idx, dout)
    _, br, _ = O.forward_f64(D, off, qf, kf, vf, gf, idx, want_branches=True)
    ref = np.einsum("thd,thbd->thb", dout, br)
    assert np.abs(dg - ref).max() < 1e-12


def test_backward_compressed_only_spreads_the_block_gradient_evenly():
    D, off, qf, kf, vf, gf, idx, dout = _fd_case(3)
    g_cmp = np.zeros_like(gf)
    g_cmp[..., 0] = gf[..., 0]
    dq, dk, dv, dg = O.backward_f64(D, off, qf, kf, vf, g_cmp, idx, dout)
    for b in range(4):
        blk = slice(off[b], off[b + 1])
        assert np.abs(dk[blk] - dk[off[b]][None]).max() < 1e-15
        assert np.abs(dv[blk] - dv[off[b]][None]).max() < 1e-15


def test_backward_threads_agree_with_single_thread():
    w = make_workload("ragged_geo")
    D = desc(w)
    idx, _ = O.route_geometric(D, w.off, w.coords)
    dout = normal_bf16(0, 5, w.q.shape, 1.0)
    a = O.backward(D, w.off, w.q, w.k, w.v, w.gates, idx, dout, nthreads=1)
    b = O.backward(D, w.off, w.q, w.k, w.v, w.gates, idx, dout, nthreads=3)
    for x, y in zip(a, b):
        assert np.abs(x - y).max() < 1e-12 * max(1.0, np.abs(x).max())


def test_backward_query_block_lists_partition_the_gradient():
    # restricting the backward to a list of query blocks splits it by linearity: the key-side
    # gradients of a partition of the blocks add up to the full ones, and the query-side rows of
    # each listed block are the full rows
    D, off, qf, kf, vf, gf, idx, dout = _fd_case(5)
    full = O.backward_f64(D, off, qf, kf, vf, gf, idx, dout)
    part_a = O.backward_f64(D, off, qf, kf, vf, gf, idx, dout, qblocks=np.array([0, 2], np.int32))
    part_b = O.backward_f64(D, off, qf, kf, vf, gf, idx, dout, qblocks=np.array([1, 3], np.int32))
    for i in (1, 2):  # dk, dv
        assert np.abs(part_a[i] + part_b[i] - full[i]).max() < 1e-13 * max(1.0, np.abs(full[i]).max())
    for i in (0, 3):  # dq, dgates
        for b, part in ((0, part_a), (2, part_a), (1, part_b), (3, part_b)):
            blk = slice(off[b], off[b + 1])
            assert np.array_equal(part[i][blk], full[i][blk])
        assert not part_a[i][off[1]:off[2]].any()
