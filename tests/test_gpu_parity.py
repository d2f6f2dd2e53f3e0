"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Bars: geometric routing indices bit-exact; score routing equal wherever the
oracle's gap between the k-th and (k+1)-th score exceeds 1e-3 and otherwise
every chosen block within 1e-3 of the k-th score; attention outputs within
1e-2 max-abs and 5e-3 relative L2, per branch and for the fused layer output
(the output is compared with the oracle run on the GPU's own indices)."""
import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_gqa_nsa_b200 import nsa
from block_sparse_gqa_nsa_b200.build import build
from nsa_case import (DeviceCase, oracle_desc, assert_close, assert_grad_close, rows_for, to_np, i32, bf16_tensor,
                      check_pooled_routing)
from workloads import make_workload
from workloads.nsa_workloads import f32_to_bf16_bits

pytestmark = pytest.mark.gpu

GAP = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    nsa.load_library()


def _compress_dev(c: DeviceCase):
    w = c.w
    B, Hkv, d = w.n_blocks, w.n_kv_heads, w.head_dim
    kc32, vc32 = c.empty(B, Hkv, d), c.empty(B, Hkv, d)
    kc, vc = c.empty(B, Hkv, d, dtype=torch.bfloat16), c.empty(B, Hkv, d, dtype=torch.bfloat16)
    nsa.lsrm_nsa_compress(c.desc, c.off, None, c.k, c.v, kc32, kc, vc32, vc, ws=c.ws)
    return kc32, kc, vc32, vc


# ------------------------------------------------------------------------------------------------
# S1 compression
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["tiny", "ragged_geo", "speed3r_small", "sparse"])
def test_compress(name):
    w = make_workload(name)
    c = DeviceCase(w)
    D = oracle_desc(w)
    B, Hq, Hkv, d = w.n_blocks, w.n_q_heads, w.n_kv_heads, w.head_dim
    kc32, kc, vc32, vc = (c.empty(B, Hkv, d), c.empty(B, Hkv, d, dtype=torch.bfloat16), c.empty(B, Hkv, d),
                          c.empty(B, Hkv, d, dtype=torch.bfloat16))
    qc32, qc = c.empty(B, Hq, d), c.empty(B, Hq, d, dtype=torch.bfloat16)
    nsa.lsrm_nsa_compress(c.desc, c.off, c.q, c.k, c.v, kc32, kc, vc32, vc, qc32, qc, ws=c.ws)
    torch.cuda.synchronize()
    for gpu32, gpu16, x, H in ((kc32, kc, w.k, Hkv), (vc32, vc, w.v, Hkv), (qc32, qc, w.q, Hq)):
        ref = O.compress(D, w.off, x, H)
        g32 = to_np(gpu32)
        assert np.abs(g32 - ref).max() <= 1e-6 * max(1.0, np.abs(ref).max())
        # bf16 outputs are the fp32 means rounded to nearest even
        want16 = f32_to_bf16_bits(g32.astype(np.float32))
        got16 = gpu16.view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(got16, want16)


# ------------------------------------------------------------------------------------------------
# S2b geometric routing: bit-exact
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("name,k", [("tiny_geo", 8), ("ragged_geo", 5), ("ragged_geo", 1), ("ragged_geo", 62),
                                    ("sparse", 16)])
def test_geometric_routing_bit_exact(name, k):
    w = make_workload(name, top_k=k)
    c = DeviceCase(w)
    idx = c.empty(w.n_blocks, k, dtype=torch.int32)
    nsa.lsrm_route_geometric(c.desc, c.off, c.coords, idx, c.ws)
    assert nsa.lsrm_nsa_last_device_status(c.ws) == 0
    ref, _ = O.route_geometric(oracle_desc(w), w.off, w.coords)
    assert np.array_equal(to_np(idx), ref)


def test_geometric_routing_flags_out_of_range_coordinates():
    w = make_workload("ragged_geo")
    c = DeviceCase(w)
    bad = w.coords.copy()
    bad[7, 1] = (1 << 29) + 1
    idx = c.empty(w.n_blocks, w.top_k, dtype=torch.int32)
    nsa.lsrm_route_geometric(c.desc, c.off, i32(bad), idx, c.ws)
    assert nsa.lsrm_nsa_last_device_status(c.ws) == 5  # LSRM_ERR_BOUNDS
    assert nsa.lsrm_nsa_last_device_status(c.ws) == 0  # read clears it


# ------------------------------------------------------------------------------------------------
# S2a score routing: gap rule
# ------------------------------------------------------------------------------------------------

def check_score_routing(gpu_idx, ref_score, k):
    """gpu_idx [nq][Hkv][k]; ref_score [nq][Hkv][B] (oracle)."""
    n_checked = 0
    for a in range(gpu_idx.shape[0]):
        for g in range(gpu_idx.shape[1]):
            s = ref_score[a, g]
            order = np.lexsort((np.arange(len(s)), -s))
            sk = s[order[k - 1]]
            gap = sk - s[order[k]] if k < len(s) else np.inf
            chosen = gpu_idx[a, g]
            assert len(set(chosen.tolist())) == k
            if gap > GAP:
                assert set(chosen.tolist()) == set(order[:k].tolist()), (a, g)
                n_checked += 1
            assert np.all(s[chosen] >= sk - GAP), (a, g)
    return n_checked


@pytest.mark.parametrize("name,k", [("tiny", 4), ("tiny", 1), ("tiny", 16), ("ragged_geo", 5)])
def test_score_routing(name, k):
    w = make_workload(name, top_k=k)
    c = DeviceCase(w)
    kc32, kc, vc32, vc = _compress_dev(c)
    idx = c.empty(w.n_blocks, w.n_kv_heads, k, dtype=torch.int32)
    score = c.empty(w.n_blocks, w.n_kv_heads, w.n_blocks)
    nsa.lsrm_route_score_topk(c.desc, c.off, c.q, kc32, idx, score, c.ws)
    D = oracle_desc(w, top_k=k)
    kc_ref = O.compress(D, w.off, w.k, w.n_kv_heads)
    ref_idx, ref_score = O.route_score(D, w.off, w.q, kc_ref)
    assert np.abs(to_np(score) - ref_score).max() < 1e-4
    n = check_score_routing(to_np(idx), ref_score, k)
    if name == "tiny" and k == 4:
        assert n > 0  # the gap rule really compares some rows


# ------------------------------------------------------------------------------------------------
# S3/S4/S5 branches, one at a time
# ------------------------------------------------------------------------------------------------

def _branch_case(name, **kw):
    w = make_workload(name, **kw)
    c = DeviceCase(w)
    D = oracle_desc(w)
    return w, c, D


@pytest.mark.parametrize("name,kw", [("tiny", {}), ("ragged_geo", {}), ("tiny", {"head_dim": 64}),
                                     ("tiny", {"n_q_heads": 2, "n_kv_heads": 2}),
                                     ("tiny_geo", {"n_q_heads": 16, "n_kv_heads": 1})])
def test_branches(name, kw):
    w, c, D = _branch_case(name, **kw)
    N, Hq, d = w.n_tokens, w.n_q_heads, w.head_dim
    kc32, kc, vc32, vc = _compress_dev(c)
    # compressed
    o, lse = c.empty(N, Hq, d), c.empty(N, Hq)
    nsa.lsrm_nsa_cmp_attn(c.desc, c.off, c.q, kc, vc, o, lse, c.ws)
    kr, vr = O.compress(D, w.off, w.k, w.n_kv_heads), O.compress(D, w.off, w.v, w.n_kv_heads)
    ro, rl = O.cmp_attn(D, w.off, w.q, kr, vr)
    assert_close(to_np(o), ro, "cmp")
    assert np.abs(to_np(lse) - rl).max() < 2e-3
    # selected, with the oracle's geometric routing (per-group layout tested in the fused path)
    idx_ref, _ = O.route_geometric(D, w.off, w.coords)
    o2, lse2 = c.empty(N, Hq, d), c.empty(N, Hq)
    nsa.lsrm_nsa_select_attn(c.desc, c.off, c.q, c.k, c.v, i32(idx_ref), 1, o2, lse2, c.ws)
    ro2, rl2 = O.select_attn(D, w.off, w.q, w.k, w.v, idx_ref)
    assert_close(to_np(o2), ro2, "slc")
    assert np.abs(to_np(lse2) - rl2).max() < 2e-3
    # window
    o3, lse3 = c.empty(N, Hq, d), c.empty(N, Hq)
    nsa.lsrm_nsa_window_attn(c.desc, c.off, c.q, c.k, c.v, o3, lse3, c.ws)
    ro3, rl3 = O.window_attn(D, w.off, w.q, w.k, w.v)
    assert_close(to_np(o3), ro3, "win")
    assert np.abs(to_np(lse3) - rl3).max() < 2e-3
    # gated combine of the three GPU branches
    out = c.empty(N, Hq, d, dtype=torch.bfloat16)
    nsa.lsrm_nsa_gate_combine(c.desc, o, o2, o3, c.gates, out)
    ref = O.forward(D, w.off, w.q, w.k, w.v, w.gates, idx_ref)
    assert_close(to_np(out), ref, "combine")
    assert nsa.lsrm_nsa_last_device_status(c.ws) == 0


@pytest.mark.parametrize("w_", [2, 16, 128])
def test_window_widths(w_):
    w, c, D = _branch_case("ragged_geo", window=w_)
    o, lse = c.empty(w.n_tokens, w.n_q_heads, w.head_dim), c.empty(w.n_tokens, w.n_q_heads)
    nsa.lsrm_nsa_window_attn(c.desc, c.off, c.q, c.k, c.v, o, lse, c.ws)
    ro, _ = O.window_attn(D, w.off, w.q, w.k, w.v)
    assert_close(to_np(o), ro, f"win{w_}")


def test_selected_branch_flags_out_of_range_indices():
    w, c, D = _branch_case("ragged_geo")
    idx_ref, _ = O.route_geometric(D, w.off, w.coords)
    bad = idx_ref.copy()
    bad[3, 2] = w.n_blocks + 7
    bad[9, 0] = -1
    o = c.empty(w.n_tokens, w.n_q_heads, w.head_dim)
    nsa.lsrm_nsa_select_attn(c.desc, c.off, c.q, c.k, c.v, i32(bad), 1, o, None, c.ws)
    assert nsa.lsrm_nsa_last_device_status(c.ws) == 5
    # the other query blocks are unaffected
    ro, _ = O.select_attn(D, w.off, w.q, w.k, w.v, idx_ref)
    keep = np.setdiff1d(np.arange(w.n_blocks), [3, 9])
    rows = rows_for(w.off, keep)
    assert_close(to_np(o)[rows], ro[rows], "slc-others")


# ------------------------------------------------------------------------------------------------
# S7 fused forward
# ------------------------------------------------------------------------------------------------

def _forward(c: DeviceCase, mode, idx=None, obr=None):
    w = c.w
    out = c.empty(w.n_tokens, w.n_q_heads, w.head_dim, dtype=torch.bfloat16)
    lse = c.empty(w.n_tokens, w.n_q_heads, w.n_gates)
    if idx is None and mode != nsa.ROUTE_ALL:
        heads = 1 if mode == nsa.ROUTE_GEOMETRIC else w.n_kv_heads
        idx = c.empty(w.n_blocks, heads, c.top_k, dtype=torch.int32)
    nsa.lsrm_nsa_forward(c.desc, c.off, c.q, c.k, c.v, c.gates, c.coords, mode, out, idx, lse, c.ws, obr=obr)
    assert nsa.lsrm_nsa_last_device_status(c.ws) == 0
    return out, idx, lse


def _branch_outputs(c: DeviceCase):
    """bf16 [N][Hq][n_gates][d] buffer for the forward's saved branch outputs."""
    w = c.w
    return c.empty(w.n_tokens, w.n_q_heads, w.n_gates, w.head_dim, dtype=torch.bfloat16)


def test_fused_forward_tiny_score_routing():
    w = make_workload("tiny")
    c = DeviceCase(w)
    out, idx, lse = _forward(c, nsa.ROUTE_SCORE)
    D = oracle_desc(w)
    kc_ref = O.compress(D, w.off, w.k, w.n_kv_heads)
    _, ref_score = O.route_score(D, w.off, w.q, kc_ref)
    gidx = to_np(idx)
    check_score_routing(gidx, ref_score, w.top_k)
    ref, br, rl = O.forward(D, w.off, w.q, w.k, w.v, w.gates, gidx, want_branches=True)
    assert_close(to_np(out), ref, "out")
    assert np.abs(to_np(lse) - rl).max() < 2e-3


@pytest.mark.parametrize("name", ["tiny_geo", "ragged_geo"])
def test_fused_forward_geometric(name):
    w = make_workload(name)
    c = DeviceCase(w)
    out, idx, lse = _forward(c, nsa.ROUTE_GEOMETRIC)
    D = oracle_desc(w)
    ref_idx, _ = O.route_geometric(D, w.off, w.coords)
    assert np.array_equal(to_np(idx).reshape(w.n_blocks, -1), ref_idx)
    ref = O.forward(D, w.off, w.q, w.k, w.v, w.gates, ref_idx)
    assert_close(to_np(out), ref, "out")


def test_fused_forward_one_hot_gates_match_each_branch():
    # one-hot gates isolate each branch, so a small branch cannot hide inside the sum
    w = make_workload("tiny_geo")
    D = oracle_desc(w)
    ref_idx, _ = O.route_geometric(D, w.off, w.coords)
    _, br, _ = O.forward(D, w.off, w.q, w.k, w.v, w.gates, ref_idx, want_branches=True)
    for b in range(3):
        g = np.zeros_like(w.gates)
        g[..., b] = f32_to_bf16_bits(np.array([1.0], np.float32))[0]
        w.gates = g
        c = DeviceCase(w)
        out, _, _ = _forward(c, nsa.ROUTE_GEOMETRIC)
        assert_close(to_np(out), br[:, :, b], f"branch{b}")


def test_fused_forward_given_per_group_indices_k1():
    w = make_workload("tiny", top_k=1)
    c = DeviceCase(w)
    rng = np.random.default_rng(3)
    idx = rng.integers(0, w.n_blocks, size=(w.n_blocks, w.n_kv_heads, 1)).astype(np.int32)
    out, _, _ = _forward(c, nsa.ROUTE_GIVEN, i32(idx))
    ref = O.forward(oracle_desc(w, top_k=1), w.off, w.q, w.k, w.v, w.gates, idx)
    assert_close(to_np(out), ref, "out")


def test_fused_forward_sparse_stage_full_size_sampled():
    w = make_workload("sparse")
    c = DeviceCase(w)
    out, idx, lse = _forward(c, nsa.ROUTE_GEOMETRIC)
    D = oracle_desc(w)
    ref_idx, _ = O.route_geometric(D, w.off, w.coords)
    assert np.array_equal(to_np(idx).reshape(w.n_blocks, -1), ref_idx)
    rng = np.random.default_rng(0)
    qb = np.sort(np.r_[rng.choice(w.n_blocks, 6, replace=False), [0, w.n_blocks - 1]]).astype(np.int32)
    ref = O.forward(D, w.off, w.q, w.k, w.v, w.gates, ref_idx, qblocks=qb)
    assert_close(to_np(out)[rows_for(w.off, qb)], ref, "out")


def test_fused_forward_dense_equals_dense_gqa_sampled():
    w = make_workload("dense")
    c = DeviceCase(w)
    out, _, _ = _forward(c, nsa.ROUTE_ALL)
    D = oracle_desc(w)
    qb = np.array([0, 200], dtype=np.int32)
    idx = np.tile(np.arange(w.n_blocks, dtype=np.int32), (w.n_blocks, 1))
    ref = O.forward(D, w.off, w.q, w.k, w.v, w.gates, idx, qblocks=qb)
    assert_close(to_np(out)[rows_for(w.off, qb)], ref, "out")


# ------------------------------------------------------------------------------------------------
# S9 Speed3R pooled-query variant
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("n_frames", [3, 6])
def test_speed3r_forward_small(n_frames):
    w = make_workload("speed3r_small", n_frames=n_frames)
    c = DeviceCase(w)
    idx = c.empty(w.n_blocks, w.n_q_heads, w.top_k, dtype=torch.int32)
    out = c.empty(w.n_tokens, w.n_q_heads, w.head_dim, dtype=torch.bfloat16)
    lse = c.empty(w.n_tokens, w.n_q_heads, 2)
    nsa.lsrm_nsa_forward(c.desc, c.off, c.q, c.k, c.v, c.gates, None, nsa.ROUTE_SCORE, out, idx, lse, c.ws)
    assert nsa.lsrm_nsa_last_device_status(c.ws) == 0
    gidx = to_np(idx)
    check_pooled_routing(gidx, w, np.arange(w.n_blocks, dtype=np.int32), w.top_k)
    D = oracle_desc(w)
    ref, br, rl = O.forward(D, w.off, w.q, w.k, w.v, w.gates, gidx, forced=w.forced, want_branches=True)
    assert_close(to_np(out), ref, "out")
    assert np.abs(to_np(lse) - rl).max() < 2e-3
    # one-hot gates: each branch on its own
    for b in range(2):
        g = np.zeros_like(w.gates)
        g[..., b] = f32_to_bf16_bits(np.array([1.0], np.float32))[0]
        nsa.lsrm_nsa_forward(c.desc, c.off, c.q, c.k, c.v, bf16_tensor(g), None, nsa.ROUTE_GIVEN, out, idx, None,
                             c.ws)
        assert_close(to_np(out), br[:, :, b], f"branch{b}")


def test_speed3r_pooled_routing_and_compressed_branch_calls():
    w = make_workload("speed3r_small", n_frames=5)
    c = DeviceCase(w)
    B, H, d = w.n_blocks, w.n_q_heads, w.head_dim
    qc, kc, vc = (c.empty(B, H, d, dtype=torch.bfloat16) for _ in range(3))
    nsa.lsrm_nsa_compress(c.desc, c.off, c.q, c.k, c.v, None, kc, None, vc, None, qc, ws=c.ws)
    qc32, kc32 = c.empty(B, H, d), c.empty(B, H, d)
    nsa.lsrm_nsa_compress(c.desc, c.off, c.q, c.k, c.v, kc32, kc, None, vc, qc32, qc, ws=c.ws)
    idx = c.empty(B, H, w.top_k, dtype=torch.int32)
    # bf16-operand mode: the ranking of the operands given
    nsa.lsrm_route_pooled_topk(c.desc, qc, kc, idx, c.ws)
    check_pooled_routing(to_np(idx), w, np.arange(B, dtype=np.int32), w.top_k, qc=to_np(qc).astype(np.float64),
                         kc=to_np(kc).astype(np.float64))
    # exact mode: the ranking of the means
    nsa.lsrm_route_pooled_topk(c.desc, qc, kc, idx, c.ws, qc32=qc32, kc32=kc32)
    check_pooled_routing(to_np(idx), w, np.arange(B, dtype=np.int32), w.top_k)
    o, lse = c.empty(w.n_tokens, H, d), c.empty(w.n_tokens, H)
    nsa.lsrm_nsa_cmp_attn(c.desc, c.off, qc, kc, vc, o, lse, c.ws)
    D = oracle_desc(w)
    ro, rl = O.cmp_attn(D, w.off, w.q, O.compress(D, w.off, w.k, H), O.compress(D, w.off, w.v, H),
                        qc=O.compress(D, w.off, w.q, H))
    assert_close(to_np(o), ro, "cmp")
    assert np.abs(to_np(lse) - rl).max() < 2e-3
    assert nsa.lsrm_nsa_last_device_status(c.ws) == 0


def test_speed3r_full_size_sampled():
    w = make_workload("speed3r")
    c = DeviceCase(w)
    idx = c.empty(w.n_blocks, w.n_q_heads, w.top_k, dtype=torch.int32)
    out = c.empty(w.n_tokens, w.n_q_heads, w.head_dim, dtype=torch.bfloat16)
    nsa.lsrm_nsa_forward(c.desc, c.off, c.q, c.k, c.v, c.gates, None, nsa.ROUTE_SCORE, out, idx, None, c.ws)
    assert nsa.lsrm_nsa_last_device_status(c.ws) == 0
    gidx = to_np(idx)
    rng = np.random.default_rng(1)
    qb = np.sort(np.r_[rng.choice(w.n_blocks, 3, replace=False), [0, 101, w.n_blocks - 1]]).astype(np.int32)
    check_pooled_routing(gidx, w, qb, w.top_k)
    ref = O.forward(oracle_desc(w), w.off, w.q, w.k, w.v, w.gates, gidx, forced=w.forced, qblocks=qb)
    assert_close(to_np(out)[rows_for(w.off, qb)], ref, "out")


# ------------------------------------------------------------------------------------------------
# S10 backward (routing indices fixed; gradients of L = sum(out * dO))
# ------------------------------------------------------------------------------------------------

def _dout(w, seed=7):
    from workloads.nsa_workloads import normal_bf16
    return w.dout if w.dout is not None else normal_bf16(seed, 5, w.q.shape, 1.0)


def _gpu_backward(c: DeviceCase, idx_t, idx_heads, lse, dout_t, obr=None):
    w = c.w
    bf = torch.bfloat16
    dq = c.empty(w.n_tokens, w.n_q_heads, w.head_dim, dtype=bf)
    dk = c.empty(w.n_tokens, w.n_kv_heads, w.head_dim, dtype=bf)
    dv = c.empty(w.n_tokens, w.n_kv_heads, w.head_dim, dtype=bf)
    dg = c.empty(w.n_tokens, w.n_q_heads, w.n_gates, dtype=bf)
    nsa.lsrm_nsa_backward(c.desc, c.off, c.q, c.k, c.v, c.gates, idx_t, idx_heads, lse, dout_t, dq, dk, dv, dg, c.ws,
                          obr=obr)
    assert nsa.lsrm_nsa_last_device_status(c.ws) == 0
    return dq, dk, dv, dg


def _check_grads(got, ref, rows=None):
    for name, g, r in zip(("dq", "dk", "dv", "dgates"), got, ref):
        g = to_np(g)
        if rows is not None and name in ("dq", "dgates"):
            g, r = g[rows], r[rows]
        assert_grad_close(g, r, name)


@pytest.mark.parametrize("saved", [False, True])
@pytest.mark.parametrize("name,kw,mode", [
    ("backward_small", {}, "geom"),
    ("ragged_geo", {}, "geom"),
    ("tiny", {}, "score"),
    ("tiny", {"head_dim": 64}, "score"),
    ("tiny_geo", {"window": 0}, "geom"),
    ("tiny_geo", {"window": 2}, "geom"),
    ("ragged_geo", {"top_k": 1}, "geom"),
])
def test_backward_matches_oracle(name, kw, mode, saved):
    # saved: the forward keeps its branch outputs and the backward reads dgates from them
    w = make_workload(name, **kw)
    c = DeviceCase(w)
    obr = _branch_outputs(c) if saved else None
    out, idx, lse = _forward(c, nsa.ROUTE_GEOMETRIC if mode == "geom" else nsa.ROUTE_SCORE, obr=obr)
    heads = 1 if mode == "geom" else w.n_kv_heads
    gidx = to_np(idx).reshape(w.n_blocks, heads, w.top_k)
    dout = _dout(w)
    got = _gpu_backward(c, idx, heads, lse, bf16_tensor(dout), obr=obr)
    ref_idx = gidx[:, 0, :] if heads == 1 else gidx
    ref = O.backward(oracle_desc(w), w.off, w.q, w.k, w.v, w.gates, ref_idx, dout, nthreads=8)
    _check_grads(got, ref)


def test_saved_branch_outputs_match_single_branch_oracle():
    # the forward's saved o_b equals the oracle layer with a one-hot gate on branch b
    w = make_workload("ragged_geo")
    c = DeviceCase(w)
    obr = _branch_outputs(c)
    _, idx, _ = _forward(c, nsa.ROUTE_GEOMETRIC, obr=obr)
    D = oracle_desc(w)
    ref_idx = to_np(idx).reshape(w.n_blocks, -1)
    got = to_np(obr)
    for b in range(w.n_gates):
        one = np.zeros_like(w.gates)
        one[..., b] = f32_to_bf16_bits(np.array([1.0], np.float32))[0]
        ref = O.forward(D, w.off, w.q, w.k, w.v, one, ref_idx)
        assert_close(got[:, :, b, :], ref, f"o_{b}")


@pytest.mark.parametrize("saved", [False, True])
def test_backward_is_deterministic(saved):
    w = make_workload("backward_small")
    c = DeviceCase(w)
    obr = _branch_outputs(c) if saved else None
    _, idx, lse = _forward(c, nsa.ROUTE_GEOMETRIC, obr=obr)
    dout = bf16_tensor(_dout(w))
    a = _gpu_backward(c, idx, 1, lse, dout, obr=obr)
    b = _gpu_backward(c, idx, 1, lse, dout, obr=obr)
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))


def test_backward_compressed_only_gates_spread_block_gradient():
    # with the selected and window gates at zero only the block means receive gradient, so every
    # token of a block gets the same dK and dV
    w = make_workload("ragged_geo")
    g = w.gates.copy()
    g[..., 1:] = 0
    w.gates = g
    c = DeviceCase(w)
    _, idx, lse = _forward(c, nsa.ROUTE_GEOMETRIC)
    dq, dk, dv, dg = _gpu_backward(c, idx, 1, lse, bf16_tensor(_dout(w)))
    dk, dv = to_np(dk), to_np(dv)
    for b in range(w.n_blocks):
        blk = slice(w.off[b], w.off[b + 1])
        assert np.array_equal(dk[blk], np.broadcast_to(dk[w.off[b]], dk[blk].shape))
        assert np.array_equal(dv[blk], np.broadcast_to(dv[w.off[b]], dv[blk].shape))


@pytest.mark.parametrize("saved", [False, True])
def test_backward_sparse_stage_full_size(saved):
    """The backward workload (sparse stage, 121 344 tokens, dO ~ N(0, 1)) at full size:
    sampled query blocks exactly against the oracle restricted to them, key-side sums against
    identities that hold at any size, and sampled key blocks with the compressed gate at zero
    against the oracle over the query blocks that reach them."""
    w = make_workload("backward")
    c = DeviceCase(w)
    obr = _branch_outputs(c) if saved else None
    _, idx, lse = _forward(c, nsa.ROUTE_GEOMETRIC, obr=obr)
    gidx = to_np(idx).reshape(w.n_blocks, w.top_k)
    dout_t = bf16_tensor(w.dout)
    dq, dk, dv, dg = _gpu_backward(c, idx, 1, lse, dout_t, obr=obr)
    D = oracle_desc(w)
    rng = np.random.default_rng(2)
    qb = np.sort(np.r_[rng.choice(w.n_blocks, 2, replace=False), [w.n_blocks - 1]]).astype(np.int32)
    ref = O.backward(D, w.off, w.q, w.k, w.v, w.gates, gidx, w.dout, nthreads=len(qb), qblocks=qb)
    rows = rows_for(w.off, qb)
    assert_grad_close(to_np(dq)[rows], ref[0][rows], "dq")
    assert_grad_close(to_np(dg)[rows], ref[3][rows], "dgates")
    # sum_u dV[u, g] = sum over the group's rows of sum_b g_b dO (every branch's P sums to one);
    # sum_u dK[u, g] = 0 (every row of dS sums to zero)
    G = w.n_q_heads // w.n_kv_heads
    gsum = to_np(c.gates).sum(-1, keepdims=True) * to_np(dout_t)
    want_dv = gsum.reshape(w.n_tokens, w.n_kv_heads, G, w.head_dim).sum((0, 2))
    got_dv = to_np(dv).astype(np.float64).sum(0)
    assert np.abs(got_dv - want_dv).max() <= 1e-2 * np.abs(want_dv).max()
    dk64 = to_np(dk).astype(np.float64)
    assert np.abs(dk64.sum(0)).max() <= 1e-3 * np.abs(dk64).sum(0).max()
    # key blocks with the compressed gate at zero: dK, dV of block j come only from the query
    # blocks that routed to it and from j itself
    g = w.gates.copy()
    g[..., 0] = 0
    w.gates = g
    c.gates = bf16_tensor(g)
    dq, dk, dv, dg = _gpu_backward(c, idx, 1, lse, dout_t)
    for j in rng.choice(w.n_blocks, 2, replace=False):
        src = np.unique(np.r_[np.nonzero((gidx == j).any(1))[0], [j]]).astype(np.int32)
        ref = O.backward(D, w.off, w.q, w.k, w.v, g, gidx, w.dout, nthreads=6, qblocks=src)
        blk = slice(w.off[j], w.off[j + 1])
        assert_grad_close(to_np(dk)[blk], ref[1][blk], f"dk block {j}")
        assert_grad_close(to_np(dv)[blk], ref[2][blk], f"dv block {j}")


# ------------------------------------------------------------------------------------------------
# the online softmax's reference move (a later chunk's max exceeds the running reference by more
# than 2^8): one block's keys are scaled up so its scores jump late in the key stream
# ------------------------------------------------------------------------------------------------

def _set_block_keys(w, block, value):
    """Every key of `block` becomes `value` in every component: its scores (and its block mean's)
    reach many times the others' in log2 units, so the running reference has to move."""
    k = w.k.copy()
    k[w.off[block]:w.off[block + 1]] = f32_to_bf16_bits(np.array([value], np.float32))[0]
    w.k = k


def test_fused_forward_reference_moves_late_in_the_stream():
    w = make_workload("dense")      # 320 blocks: five compressed chunks, 320 selected chunks
    _set_block_keys(w, 300, 50.0)   # block 300: late in both the compressed and selected streams
    D = oracle_desc(w)
    qb = np.array([0, 150, 300], dtype=np.int32)
    idx = np.tile(np.arange(w.n_blocks, dtype=np.int32), (w.n_blocks, 1))
    for b in range(3):  # every branch on its own
        one = np.zeros_like(w.gates)
        one[..., b] = f32_to_bf16_bits(np.array([1.0], np.float32))[0]
        w.gates = one
        c = DeviceCase(w)
        o1, _, _ = _forward(c, nsa.ROUTE_ALL)
        ref = O.forward(D, w.off, w.q, w.k, w.v, one, idx, qblocks=qb)
        assert_close(to_np(o1)[rows_for(w.off, qb)], ref, f"branch{b}")


def test_speed3r_routing_with_a_late_dominant_block():
    w = make_workload("speed3r_small", n_frames=6)
    target = w.n_blocks - 3                      # a late, non-forced block
    assert target not in set(w.forced.tolist())
    _set_block_keys(w, target, 400.0)
    c = DeviceCase(w)
    idx = c.empty(w.n_blocks, w.n_q_heads, w.top_k, dtype=torch.int32)
    out = c.empty(w.n_tokens, w.n_q_heads, w.head_dim, dtype=torch.bfloat16)
    nsa.lsrm_nsa_forward(c.desc, c.off, c.q, c.k, c.v, c.gates, None, nsa.ROUTE_SCORE, out, idx, None, c.ws)
    assert nsa.lsrm_nsa_last_device_status(c.ws) == 0
    gidx = to_np(idx)
    for row in gidx.reshape(-1, w.top_k):
        assert len(set(row.tolist())) == w.top_k  # distinct: no candidate offered twice
    qb = np.arange(w.n_blocks, dtype=np.int32)
    # the dominant block's logits are ~400x the others' (bf16 rounding of the pooled queries alone
    # would move them by more than the 1e-3 gap): the forward ranks the fp32 means, so the plain
    # gap rule against the fp64 oracle holds
    check_pooled_routing(gidx, w, qb, w.top_k)
    ref = O.forward(oracle_desc(w), w.off, w.q, w.k, w.v, w.gates, gidx, forced=w.forced)
    assert_close(to_np(out), ref, "out")


def test_speed3r_routing_ties_break_by_block_id():
    # Two classes of non-forced blocks with bit-identical pooled keys: even blocks share one key
    # vector u, odd blocks the zero vector.  Every row then sees exactly equal logits inside each
    # class, so its top-k is fixed by the order (logit desc, block asc) alone: the k smallest ids
    # of the class whose logit is larger (with q.u clear of zero at operand precision).  Ties sit
    # exactly at the k-th logit, which is where a lower bound on it must still let them through.
    w = make_workload("speed3r_small", n_frames=6)
    forced = set(w.forced.tolist())
    rng = np.random.default_rng(7)
    u = f32_to_bf16_bits(rng.standard_normal(w.head_dim).astype(np.float32))
    k = w.k.copy()
    for b in range(w.n_blocks):
        if b in forced:
            continue
        k[w.off[b]:w.off[b + 1]] = u if b % 2 == 0 else 0
    w.k = k
    c = DeviceCase(w)
    idx = c.empty(w.n_blocks, w.n_q_heads, w.top_k, dtype=torch.int32)
    out = c.empty(w.n_tokens, w.n_q_heads, w.head_dim, dtype=torch.bfloat16)
    nsa.lsrm_nsa_forward(c.desc, c.off, c.q, c.k, c.v, c.gates, None, nsa.ROUTE_SCORE, out, idx, None, c.ws)
    assert nsa.lsrm_nsa_last_device_status(c.ws) == 0
    gidx = to_np(idx)
    D = oracle_desc(w)
    from workloads.nsa_workloads import bf16_bits_to_f32
    qc = O.compress(D, w.off, w.q, w.n_q_heads)  # the forward ranks the means themselves
    uf = bf16_bits_to_f32(u).astype(np.float64)
    even = [b for b in range(0, w.n_blocks, 2) if b not in forced]
    odd = [b for b in range(1, w.n_blocks, 2) if b not in forced]
    assert len(even) >= w.top_k and len(odd) >= w.top_k
    checked = 0
    for a in range(w.n_blocks):
        for h in range(w.n_q_heads):
            lu = float(np.dot(qc[a, h].astype(np.float64), uf)) * w.scale
            if abs(lu) < 1e-3:
                continue
            want = (even if lu > 0 else odd)[:w.top_k]
            assert gidx[a, h].tolist() == want, (a, h, lu)
            checked += 1
    assert checked > 0.9 * w.n_blocks * w.n_q_heads


@pytest.mark.parametrize("saved", [False, True])
def test_two_gate_layer_forward_and_backward(saved):
    # n_gates = 2: compressed and selected branches only (no window), forward and backward
    w = make_workload("ragged_geo")
    w.gates = np.ascontiguousarray(w.gates[..., :2])
    w.n_gates = 2
    c = DeviceCase(w)
    obr = _branch_outputs(c) if saved else None
    out, idx, lse = _forward(c, nsa.ROUTE_GEOMETRIC, obr=obr)
    D = oracle_desc(w)
    ref_idx, _ = O.route_geometric(D, w.off, w.coords)
    assert np.array_equal(to_np(idx).reshape(w.n_blocks, -1), ref_idx)
    assert_close(to_np(out), O.forward(D, w.off, w.q, w.k, w.v, w.gates, ref_idx), "out")
    dout = _dout(w)
    got = _gpu_backward(c, idx, 1, lse, bf16_tensor(dout), obr=obr)
    ref = O.backward(D, w.off, w.q, w.k, w.v, w.gates, ref_idx, dout, nthreads=8)
    _check_grads(got, ref)
