"""The pages' 8x8x8 volume blocks (LSRM page, 方法, block-grouping paragraph: image tokens in 8x8
blocks, volume tokens in 8x8x8 blocks), i.e. blocks of up to 512 tokens next to 64-token image
tiles, through the forward path: geometric routing bit-exact, each branch and the fused layer
against the oracle (a routed block of more than 64 tokens is several 64-key chunks; the window
band of a tile pair inside a long block spans one or two chunks).  The backward keeps blocks of
at most 64 tokens and says so."""
import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_gqa_nsa_b200 import nsa
from block_sparse_gqa_nsa_b200.build import build
from nsa_case import DeviceCase, oracle_desc, assert_close, rows_for, to_np, i32, bf16_tensor
from workloads import make_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    nsa.load_library()


@pytest.mark.parametrize("name", ["small_vol512", "ragged_vol512"])
def test_geometric_routing_on_512_token_blocks_is_bit_exact(name):
    w = make_workload(name)
    c = DeviceCase(w)
    idx = c.empty(w.n_blocks, w.top_k, dtype=torch.int32)
    nsa.lsrm_route_geometric(c.desc, c.off, c.coords, idx, c.ws)
    assert nsa.lsrm_nsa_last_device_status(c.ws) == 0
    ref, _ = O.route_geometric(oracle_desc(w), w.off, w.coords)
    assert np.array_equal(to_np(idx), ref)


@pytest.mark.parametrize("name,window", [("small_vol512", 64), ("small_vol512", 128), ("ragged_vol512", 64),
                                         ("ragged_vol512", 200)])
def test_window_branch_on_512_token_blocks(name, window):
    w = make_workload(name, window=window)
    c = DeviceCase(w)
    D = oracle_desc(w)
    o, lse = c.empty(w.n_tokens, w.n_q_heads, w.head_dim), c.empty(w.n_tokens, w.n_q_heads)
    nsa.lsrm_nsa_window_attn(c.desc, c.off, c.q, c.k, c.v, o, lse, c.ws)
    assert nsa.lsrm_nsa_last_device_status(c.ws) == 0
    ro, rl = O.window_attn(D, w.off, w.q, w.k, w.v)
    assert_close(to_np(o), ro, f"win{window}")
    assert np.abs(to_np(lse) - rl).max() < 2e-3


@pytest.mark.parametrize("name", ["small_vol512", "ragged_vol512"])
def test_selected_and_fused_forward_on_512_token_blocks(name):
    w = make_workload(name)
    c = DeviceCase(w)
    D = oracle_desc(w)
    idx_ref, _ = O.route_geometric(D, w.off, w.coords)
    # volume blocks (the long ones) first, then two image tiles
    qb = np.unique(np.r_[0, 1, w.layout.n_vol_blocks - 1, w.layout.n_vol_blocks, w.n_blocks - 1]).astype(np.int32)
    rows = rows_for(w.off, qb)
    o = c.empty(w.n_tokens, w.n_q_heads, w.head_dim)
    nsa.lsrm_nsa_select_attn(c.desc, c.off, c.q, c.k, c.v, i32(idx_ref), 1, o, None, c.ws)
    assert nsa.lsrm_nsa_last_device_status(c.ws) == 0
    ro, _ = O.select_attn(D, w.off, w.q, w.k, w.v, idx_ref, qblocks=qb)
    assert_close(to_np(o)[rows], ro, "slc")
    out = c.empty(w.n_tokens, w.n_q_heads, w.head_dim, dtype=torch.bfloat16)
    idx = c.empty(w.n_blocks, w.top_k, dtype=torch.int32)
    lse = c.empty(w.n_tokens, w.n_q_heads, 3)
    nsa.lsrm_nsa_forward(c.desc, c.off, c.q, c.k, c.v, c.gates, c.coords, nsa.ROUTE_GEOMETRIC, out, idx, lse, c.ws)
    assert nsa.lsrm_nsa_last_device_status(c.ws) == 0
    assert np.array_equal(to_np(idx), idx_ref)
    ref, _, rl = O.forward(D, w.off, w.q, w.k, w.v, w.gates, idx_ref, qblocks=qb, want_branches=True)
    assert_close(to_np(out)[rows], ref, "out")
    assert np.abs(to_np(lse)[rows] - rl).max() < 2e-3


@pytest.mark.slow
def test_sparse_stage_with_512_token_volume_blocks_sampled():
    w = make_workload("sparse_vol512")
    c = DeviceCase(w)
    out = c.empty(w.n_tokens, w.n_q_heads, w.head_dim, dtype=torch.bfloat16)
    idx = c.empty(w.n_blocks, w.top_k, dtype=torch.int32)
    nsa.lsrm_nsa_forward(c.desc, c.off, c.q, c.k, c.v, c.gates, c.coords, nsa.ROUTE_GEOMETRIC, out, idx, None, c.ws)
    assert nsa.lsrm_nsa_last_device_status(c.ws) == 0
    D = oracle_desc(w)
    idx_ref, _ = O.route_geometric(D, w.off, w.coords)
    assert np.array_equal(to_np(idx), idx_ref)
    nv = w.layout.n_vol_blocks
    qb = np.array([0, nv - 1, nv, w.n_blocks - 1], dtype=np.int32)
    ref = O.forward(D, w.off, w.q, w.k, w.v, w.gates, idx_ref, qblocks=qb)
    assert_close(to_np(out)[rows_for(w.off, qb)], ref, "out")


def test_backward_rejects_blocks_longer_than_64_tokens():
    w = make_workload("ragged_vol512")
    c = DeviceCase(w)
    bf = torch.bfloat16
    g = [c.empty(w.n_tokens, w.n_q_heads, w.head_dim, dtype=bf), c.empty(w.n_tokens, w.n_kv_heads, w.head_dim, dtype=bf),
         c.empty(w.n_tokens, w.n_kv_heads, w.head_dim, dtype=bf), c.empty(w.n_tokens, w.n_q_heads, 3, dtype=bf)]
    idx = c.empty(w.n_blocks, w.top_k, dtype=torch.int32).zero_()
    lse = c.empty(w.n_tokens, w.n_q_heads, 3).zero_()
    with pytest.raises(nsa.NsaError) as e:
        nsa.lsrm_nsa_backward(c.desc, c.off, c.q, c.k, c.v, c.gates, idx, 1, lse, c.q, *g, c.ws)
    assert e.value.status == 2  # LSRM_ERR_UNSUPPORTED
