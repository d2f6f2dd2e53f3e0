"""lsrm_route_geometric_noalloc: geometric routing for callers that cannot allocate device
memory (for example a plugin whose host framework's pool owns the whole GPU) and so have no
workspace to pass.  Its result must equal lsrm_route_geometric's bit for bit, call after
call, although every call reuses the same fixed scratch array inside the library.

This file is collected last on purpose, so that a run stopping at the first failure has
already run every other test."""
import numpy as np
import pytest
import torch

from block_sparse_gqa_nsa_b200 import nsa
from block_sparse_gqa_nsa_b200.build import build
from workloads import make_workload

pytestmark = pytest.mark.gpu


def _dev(w):
    off = torch.from_numpy(w.off.astype(np.int32)).cuda()
    coords = torch.from_numpy(w.coords.astype(np.int32)).cuda()
    desc = nsa.make_desc(w.n_tokens, w.n_blocks, w.max_block_len, w.n_q_heads, w.n_kv_heads, w.head_dim,
                         w.top_k, w.window, 0.0, False, w.n_gates)
    return off, coords, desc


def test_noalloc_routing_matches_workspace_routing_on_consecutive_calls():
    build()
    for name in ("sparse", "ragged_geo"):
        w = make_workload(name)
        off, coords, desc = _dev(w)
        ws = nsa.workspace(desc)
        ref = torch.empty(w.n_blocks, w.top_k, dtype=torch.int32, device="cuda")
        nsa.lsrm_route_geometric(desc, off, coords, ref, ws)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        for _ in range(2):  # the scratch keeps the previous call's centroids: results must not depend on it
            got = torch.full_like(ref, -7)
            nsa.lsrm_route_geometric_noalloc(desc, off, coords, got, status)
            torch.cuda.synchronize()
            assert torch.equal(got, ref), name
        assert int(status.item()) == 0


def test_noalloc_routing_rejects_too_many_blocks_and_reports_bad_coordinates():
    build()
    w = make_workload("ragged_geo")
    off, coords, desc = _dev(w)
    big = nsa.make_desc(20000 * 2, 20000, 2, 32, 2, 32, 4, 64)
    with pytest.raises(nsa.NsaError) as e:
        nsa.lsrm_route_geometric_noalloc(big, off, coords, torch.empty(1, dtype=torch.int32, device="cuda"))
    assert e.value.status == 6  # LSRM_ERR_WORKSPACE: beyond the fixed scratch
    # descriptors that lsrm_route_geometric rejects are rejected here too, with the same status
    ws = nsa.workspace(desc)
    idx0 = torch.empty(w.n_blocks, w.top_k, dtype=torch.int32, device="cuda")
    for bad_desc in (nsa.make_desc(w.n_tokens, w.n_blocks, 513, 32, 2, 32, w.top_k, 64),     # block > 512
                     nsa.make_desc(w.n_tokens, w.n_blocks, w.max_block_len, 32, 2, 48, w.top_k, 64),  # d = 48
                     nsa.make_desc(w.n_tokens, w.n_blocks, w.max_block_len, 32, 2, 32, w.top_k, 63)):  # odd w
        with pytest.raises(nsa.NsaError) as e_ref:
            nsa.lsrm_route_geometric(bad_desc, off, coords, idx0, ws)
        with pytest.raises(nsa.NsaError) as e_na:
            nsa.lsrm_route_geometric_noalloc(bad_desc, off, coords, idx0)
        assert e_na.value.status == e_ref.value.status
    bad = coords.clone()
    bad[3, 0] = (1 << 29) + 5
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx = torch.empty(w.n_blocks, w.top_k, dtype=torch.int32, device="cuda")
    nsa.lsrm_route_geometric_noalloc(desc, off, bad, idx, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 1 << (5 - 1)  # LSRM_ERR_BOUNDS bit
