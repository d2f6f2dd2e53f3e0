"""Backward of the Speed3R pooled-query layer on the GPU (lsrm_nsa_backward with pooled_q) against
the fp64 oracle's chain rule (Speed3R page, section 2: the model trains end to end), on the
forward's own routing indices, with the gradient bounds of the LSRM backward."""
import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_gqa_nsa_b200 import nsa
from block_sparse_gqa_nsa_b200.build import build
from nsa_case import DeviceCase, assert_close, assert_grad_close, bf16_tensor, oracle_desc, to_np
from workloads import make_workload
from workloads.nsa_workloads import STREAM_DOUT, normal_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    nsa.load_library()


def _forward(c, w):
    N, B, H, d = w.n_tokens, w.n_blocks, w.n_q_heads, w.head_dim
    idx = c.empty(B, H, w.top_k, dtype=torch.int32)
    out = c.empty(N, H, d, dtype=torch.bfloat16)
    lse = c.empty(N, H, 2)
    obr = c.empty(N, H, 2, d, dtype=torch.bfloat16)
    nsa.lsrm_nsa_forward(c.desc, c.off, c.q, c.k, c.v, c.gates, None, nsa.ROUTE_SCORE, out, idx, lse, c.ws, obr=obr)
    torch.cuda.synchronize()
    assert nsa.lsrm_nsa_last_device_status(c.ws) == 0
    return idx, out, lse, obr


def _backward(c, w, idx, lse, obr, dout):
    N, H, d = w.n_tokens, w.n_q_heads, w.head_dim
    dq, dk, dv = (c.empty(N, H, d, dtype=torch.bfloat16) for _ in range(3))
    dg = c.empty(N, H, 2, dtype=torch.bfloat16)
    nsa.lsrm_nsa_backward(c.desc, c.off, c.q, c.k, c.v, c.gates, idx, H, lse, dout, dq, dk, dv, dg, c.ws, obr=obr)
    torch.cuda.synchronize()
    assert nsa.lsrm_nsa_last_device_status(c.ws) == 0
    return dq, dk, dv, dg


@pytest.mark.parametrize("n_frames,k", [(3, 32), (5, 64)])
def test_speed3r_backward_matches_oracle(n_frames, k):
    w = make_workload("speed3r_small", n_frames=n_frames, top_k=k)
    c = DeviceCase(w)
    idx, out, lse, obr = _forward(c, w)
    gidx = to_np(idx)
    # the saved branch outputs are the oracle's branches (bf16)
    _, br, _ = O.forward(oracle_desc(w), w.off, w.q, w.k, w.v, w.gates, gidx, forced=w.forced, want_branches=True)
    assert_close(to_np(obr), br, "saved branch outputs")
    dout_np = normal_bf16(3, STREAM_DOUT, (w.n_tokens, w.n_q_heads, w.head_dim), 1.0)
    dout = bf16_tensor(dout_np)
    dq, dk, dv, dg = _backward(c, w, idx, lse, obr, dout)
    rq, rk, rv, rg = O.backward_pooled(oracle_desc(w), w.off, w.q, w.k, w.v, w.gates, gidx, w.forced, dout_np,
                                       nthreads=8)
    assert_grad_close(to_np(dg), rg, "dgates")
    assert_grad_close(to_np(dq), rq, "dq")
    assert_grad_close(to_np(dk), rk, "dk")
    assert_grad_close(to_np(dv), rv, "dv")
    # fixed summation orders: a second run gives the same bits
    dq2, dk2, dv2, dg2 = _backward(c, w, idx, lse, obr, dout)
    for a, b in ((dq, dq2), (dk, dk2), (dv, dv2), (dg, dg2)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_speed3r_backward_argument_checks():
    w = make_workload("speed3r_small", n_frames=3)
    c = DeviceCase(w)
    idx, out, lse, obr = _forward(c, w)
    N, H, d = w.n_tokens, w.n_q_heads, w.head_dim
    dout = c.empty(N, H, d, dtype=torch.bfloat16)
    dq, dk, dv = (c.empty(N, H, d, dtype=torch.bfloat16) for _ in range(3))
    dg = c.empty(N, H, 2, dtype=torch.bfloat16)
    with pytest.raises(nsa.NsaError) as e:  # the saved branch outputs are required
        nsa.lsrm_nsa_backward(c.desc, c.off, c.q, c.k, c.v, c.gates, idx, H, lse, dout, dq, dk, dv, dg, c.ws)
    assert e.value.status == 1
    with pytest.raises(nsa.NsaError) as e:  # per-head routing lists
        nsa.lsrm_nsa_backward(c.desc, c.off, c.q, c.k, c.v, c.gates, idx, 1, lse, dout, dq, dk, dv, dg, c.ws,
                              obr=obr)
    assert e.value.status == 1
