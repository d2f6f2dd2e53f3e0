"""Problem sizes beyond one grid dimension's 65535 limit: more than 65535 query blocks in the
LSRM layer (forward and backward), and the Speed3R variant at 1000 frames (101 000 blocks, the
sequence length of the Speed3R page's long-sequence experiments), each checked against the
oracle on sampled query blocks, among them blocks past index 65535."""
import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_gqa_nsa_b200 import nsa
from block_sparse_gqa_nsa_b200.build import build
from nsa_case import DeviceCase, oracle_desc, assert_close, assert_grad_close, rows_for, to_np, i32, bf16_tensor
from workloads import make_workload
from workloads.nsa_workloads import Layout, Workload, _tensors, normal_bf16

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    nsa.load_library()


def _many_blocks(n_blocks=70000, seed=3):
    # ragged blocks of 1-3 tokens, GQA 32/2, d 32, routing given (random distinct blocks)
    rng = np.random.default_rng(seed)
    sizes = rng.integers(1, 4, n_blocks)
    off = np.zeros(n_blocks + 1, dtype=np.int32)
    off[1:] = np.cumsum(sizes)
    lay = Layout(off=off, coords=None)
    q, k, v, g, dout = _tensors(lay, 32, 2, 32, 3, seed, 1.0 / np.sqrt(32.0), None, with_dout=True)
    w = Workload(name="many_blocks", layout=lay, n_q_heads=32, n_kv_heads=2, head_dim=32, top_k=4, window=2,
                 route="given", pooled_q=False, n_gates=3, q=q, k=k, v=v, gates=g, forced=np.zeros(0, np.int32),
                 dout=dout, seed=seed, description="70000 ragged blocks")
    idx = np.stack([rng.choice(n_blocks, 4, replace=False) for _ in range(n_blocks)]).astype(np.int32)
    return w, idx


def test_layer_forward_and_backward_past_65535_query_blocks():
    w, idx = _many_blocks()
    assert w.n_blocks > 65535
    c = DeviceCase(w)
    B, Hq, Hkv, d = w.n_blocks, w.n_q_heads, w.n_kv_heads, w.head_dim
    out = c.empty(w.n_tokens, Hq, d, dtype=torch.bfloat16)
    lse = c.empty(w.n_tokens, Hq, 3)
    gidx = i32(np.repeat(idx[:, None, :], Hkv, axis=1))  # the given-routing layout [B][Hkv][k]
    nsa.lsrm_nsa_forward(c.desc, c.off, c.q, c.k, c.v, c.gates, None, nsa.ROUTE_GIVEN, out, gidx, lse, c.ws)
    assert nsa.lsrm_nsa_last_device_status(c.ws) == 0
    D = oracle_desc(w)
    qb = np.array([0, 1234, 65534, 65535, 65536, 69998, B - 1], dtype=np.int32)
    rows = rows_for(w.off, qb)
    ref = O.forward(D, w.off, w.q, w.k, w.v, w.gates, idx, qblocks=qb)
    assert_close(to_np(out)[rows], ref, "out")
    # backward: the query-side gradients of the sampled blocks are exact per block
    dq = c.empty(w.n_tokens, Hq, d, dtype=torch.bfloat16)
    dk = c.empty(w.n_tokens, Hkv, d, dtype=torch.bfloat16)
    dv = c.empty(w.n_tokens, Hkv, d, dtype=torch.bfloat16)
    dg = c.empty(w.n_tokens, Hq, 3, dtype=torch.bfloat16)
    nsa.lsrm_nsa_backward(c.desc, c.off, c.q, c.k, c.v, c.gates, gidx, Hkv, lse, bf16_tensor(w.dout), dq, dk, dv,
                          dg, c.ws)
    assert nsa.lsrm_nsa_last_device_status(c.ws) == 0
    rdq, _, _, rdg = O.backward(D, w.off, w.q, w.k, w.v, w.gates, idx, w.dout, nthreads=8, qblocks=qb)
    assert_grad_close(to_np(dq)[rows], rdq[rows], "dq")
    assert_grad_close(to_np(dg)[rows], rdg[rows], "dgates")


def test_speed3r_forward_at_1000_frames_sampled():
    w = make_workload("speed3r_small", n_frames=1000)
    assert w.n_blocks > 65535
    c = DeviceCase(w)
    idx = c.empty(w.n_blocks, w.n_q_heads, w.top_k, dtype=torch.int32)
    out = c.empty(w.n_tokens, w.n_q_heads, w.head_dim, dtype=torch.bfloat16)
    nsa.lsrm_nsa_forward(c.desc, c.off, c.q, c.k, c.v, c.gates, None, nsa.ROUTE_SCORE, out, idx, None, c.ws)
    assert nsa.lsrm_nsa_last_device_status(c.ws) == 0
    gidx = to_np(idx)
    qb = np.array([0, 5, 101, 65535, 70001, w.n_blocks - 1], dtype=np.int32)
    # routing: validity and the gap rule against the oracle's fp64 pooled logits
    D = oracle_desc(w)
    qc = O.compress(D, w.off, w.q, w.n_q_heads)
    kc = O.compress(D, w.off, w.k, w.n_kv_heads)
    _, logits = O.route_pooled(D, qc, kc, w.forced, qblocks=qb, want_logits=True)
    forced = set(w.forced.tolist())
    for i, a in enumerate(qb):
        for h in range(w.n_q_heads):
            chosen = gidx[a, h].tolist()
            assert len(set(chosen)) == w.top_k and not (set(chosen) & forced)
            lg = logits[i, h].copy()
            lg[list(forced)] = -np.inf
            order = np.lexsort((np.arange(w.n_blocks), -lg))
            sk = lg[order[w.top_k - 1]]
            assert np.all(lg[chosen] >= sk - 1e-3)
            if sk - lg[order[w.top_k]] > 1e-3:
                assert set(chosen) == set(order[:w.top_k].tolist())
    ref = O.forward(D, w.off, w.q, w.k, w.v, w.gates, gidx, forced=w.forced, qblocks=qb)
    assert_close(to_np(out)[rows_for(w.off, qb)], ref, "out")
