"""Parity of the self/cross gated mixture (lsrm_nsa_mixture, one kernel launch) with the fp64
oracle (LSRM page, 方法: the dense blocks' gated cross-attention equations).

Bars as for the fused layer: outputs within 1e-2 max-abs and 5e-3 relative L2; LSE within 1e-3
absolute.  Cases: the tiny and the ragged (voxel-exact shell) layouts in full, the dense-stage
shape (20480 tokens) on sampled blocks of both streams, empty streams, MHA at d = 64, and the
argument checks."""
import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_gqa_nsa_b200 import nsa
from block_sparse_gqa_nsa_b200.build import build
from nsa_case import DeviceCase, assert_close, rows_for, to_np
from workloads import make_workload

pytestmark = pytest.mark.gpu

LSE_ATOL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    nsa.load_library()


def _odesc(w):
    return O.desc_for(w.n_tokens, w.n_blocks, w.n_q_heads, w.n_kv_heads, w.head_dim, 1, 0, n_gates=2)


def _run(c, bx):
    w = c.w
    out = c.empty(w.n_tokens, w.n_q_heads, w.head_dim, dtype=torch.bfloat16)
    lse = c.empty(w.n_tokens, w.n_q_heads, 2)
    nsa.lsrm_nsa_mixture(c.desc, c.off, bx, c.q, c.k, c.v, c.gates, out, lse, c.ws)
    torch.cuda.synchronize()
    assert nsa.lsrm_nsa_last_device_status(c.ws) == 0
    return to_np(out), to_np(lse)


def _check(w, got_out, got_lse, bx, qblocks=None):
    ref, _, ref_lse = O.mixture(_odesc(w), w.off, w.q, w.k, w.v, w.gates, bx, qblocks=qblocks, want_branches=True)
    rows = np.arange(w.n_tokens) if qblocks is None else rows_for(w.off, qblocks)
    assert_close(got_out[rows], ref, f"{w.name} out")
    g, r = got_lse[rows], ref_lse
    assert np.array_equal(np.isneginf(g), np.isneginf(r)), f"{w.name}: -inf LSE pattern"
    fin = np.isfinite(r)
    assert np.abs(g[fin] - r[fin]).max() <= LSE_ATOL, f"{w.name}: lse"


@pytest.mark.parametrize("name", ["mixture_small", "mixture_ragged"])
def test_mixture_matches_oracle(name):
    w = make_workload(name)
    c = DeviceCase(w)
    out, lse = _run(c, w.n_blocks_x)
    _check(w, out, lse, w.n_blocks_x)


def test_mixture_dense_stage_shape_sampled_blocks():
    w = make_workload("mixture")
    c = DeviceCase(w)
    out, lse = _run(c, w.n_blocks_x)
    bx, B = w.n_blocks_x, w.n_blocks
    qblocks = [0, bx // 2, bx - 1, bx, (bx + B) // 2, B - 1]  # both streams, both ends of each
    _check(w, out, lse, bx, qblocks)


@pytest.mark.parametrize("which", ["all_x", "all_y"])
def test_mixture_with_an_empty_stream(which):
    w = make_workload("mixture_small")
    c = DeviceCase(w)
    bx = w.n_blocks if which == "all_x" else 0
    out, lse = _run(c, bx)
    _check(w, out, lse, bx)
    assert np.all(np.isneginf(lse[..., 1]))


def test_mixture_mha_d64():
    w = make_workload("mixture_ragged", n_q_heads=4, n_kv_heads=4, head_dim=64)
    c = DeviceCase(w)
    out, lse = _run(c, w.n_blocks_x)
    _check(w, out, lse, w.n_blocks_x)


def test_mixture_argument_checks():
    w = make_workload("mixture_small")
    c = DeviceCase(w)
    out = c.empty(w.n_tokens, w.n_q_heads, w.head_dim, dtype=torch.bfloat16)
    with pytest.raises(nsa.NsaError) as e:
        nsa.lsrm_nsa_mixture(c.desc, c.off, w.n_blocks + 1, c.q, c.k, c.v, c.gates, out, None, c.ws)
    assert e.value.status == 1  # LSRM_ERR_INVALID_ARG
    d3 = nsa.make_desc(w.n_tokens, w.n_blocks, w.max_block_len, w.n_q_heads, w.n_kv_heads, w.head_dim, 1, 0, 0.0,
                       False, 3)
    with pytest.raises(nsa.NsaError) as e:
        nsa.lsrm_nsa_mixture(d3, c.off, w.n_blocks_x, c.q, c.k, c.v, c.gates, out, None, c.ws)
    assert e.value.status == 1
