"""Speed3R routing with a raised Top-K (Speed3R page, long-sequence experiments: the test-time
adaptation raises Top-K).  Above 48 the streaming top-k of the pooled compressed pass keeps a full
candidate buffer and replaces its worst entry, and the routed part reads two routed blocks per
lane; both are checked against the fp64 oracle with the plain gap rule, ties included."""
import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_gqa_nsa_b200 import nsa
from block_sparse_gqa_nsa_b200.build import build
from nsa_case import DeviceCase, assert_close, check_pooled_routing, oracle_desc, to_np
from workloads import make_workload
from workloads.nsa_workloads import bf16_bits_to_f32, f32_to_bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    nsa.load_library()


def _forward(c, w):
    idx = c.empty(w.n_blocks, w.n_q_heads, w.top_k, dtype=torch.int32)
    out = c.empty(w.n_tokens, w.n_q_heads, w.head_dim, dtype=torch.bfloat16)
    lse = c.empty(w.n_tokens, w.n_q_heads, 2)
    nsa.lsrm_nsa_forward(c.desc, c.off, c.q, c.k, c.v, c.gates, None, nsa.ROUTE_SCORE, out, idx, lse, c.ws)
    torch.cuda.synchronize()
    assert nsa.lsrm_nsa_last_device_status(c.ws) == 0
    return to_np(idx), to_np(out), to_np(lse)


@pytest.mark.parametrize("k", [40, 48, 49, 64])
def test_speed3r_forward_with_raised_top_k(k):
    w = make_workload("speed3r_small", n_frames=6, top_k=k)
    c = DeviceCase(w)
    gidx, out, lse = _forward(c, w)
    check_pooled_routing(gidx, w, np.arange(w.n_blocks, dtype=np.int32), k)
    ref, _, rl = O.forward(oracle_desc(w), w.off, w.q, w.k, w.v, w.gates, gidx, forced=w.forced,
                           want_branches=True)
    assert_close(out, ref, f"out k={k}")
    assert np.abs(lse - rl).max() < 2e-3


def test_speed3r_top_64_bf16_operand_mode():
    w = make_workload("speed3r_small", n_frames=5, top_k=64)
    c = DeviceCase(w)
    B, H, d = w.n_blocks, w.n_q_heads, w.head_dim
    qc, kc, vc = (c.empty(B, H, d, dtype=torch.bfloat16) for _ in range(3))
    nsa.lsrm_nsa_compress(c.desc, c.off, c.q, c.k, c.v, None, kc, None, vc, None, qc, ws=c.ws)
    idx = c.empty(B, H, 64, dtype=torch.int32)
    nsa.lsrm_route_pooled_topk(c.desc, qc, kc, idx, c.ws)
    torch.cuda.synchronize()
    check_pooled_routing(to_np(idx), w, np.arange(B, dtype=np.int32), 64, qc=to_np(qc).astype(np.float64),
                         kc=to_np(kc).astype(np.float64))


def test_speed3r_top_64_ties_break_by_block_id():
    # even non-forced blocks share one key vector, odd ones the zero vector: every row's top-64 is
    # the 64 lowest ids of the class with the larger logit, so a full buffer meets exact ties
    w = make_workload("speed3r_small", n_frames=6, top_k=64)
    forced = set(w.forced.tolist())
    rng = np.random.default_rng(11)
    u = f32_to_bf16_bits(rng.standard_normal(w.head_dim).astype(np.float32))
    k = w.k.copy()
    for b in range(w.n_blocks):
        if b not in forced:
            k[w.off[b]:w.off[b + 1]] = u if b % 2 == 0 else 0
    w.k = k
    c = DeviceCase(w)
    gidx, _, _ = _forward(c, w)
    qc = O.compress(oracle_desc(w), w.off, w.q, w.n_q_heads)
    uf = bf16_bits_to_f32(u).astype(np.float64)
    even = [b for b in range(0, w.n_blocks, 2) if b not in forced]
    odd = [b for b in range(1, w.n_blocks, 2) if b not in forced]
    checked = 0
    for a in range(w.n_blocks):
        for h in range(w.n_q_heads):
            lu = float(np.dot(qc[a, h], uf)) * w.scale
            if abs(lu) < 1e-3:
                continue
            assert gidx[a, h].tolist() == (even if lu > 0 else odd)[:64], (a, h, lu)
            checked += 1
    assert checked > 0.9 * w.n_blocks * w.n_q_heads


def test_speed3r_top_k_above_64_is_unsupported():
    w = make_workload("speed3r_small", n_frames=3, top_k=65)
    c = DeviceCase(w)
    with pytest.raises(nsa.NsaError) as e:
        _forward(c, w)
    assert e.value.status == 2  # LSRM_ERR_UNSUPPORTED
