"""Camera-projection routing on the GPU (lsrm_route_camera) against the fp64 oracle, bit for bit
(LSRM page, 方法, 3D-aware routing paragraph), and the layer run on its indices."""
import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_gqa_nsa_b200 import nsa
from block_sparse_gqa_nsa_b200.build import build
from nsa_case import DeviceCase, assert_close, i32, oracle_desc, rows_for, to_np
from workloads import camera_inputs, make_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    nsa.load_library()


def _route(c, proj, tiles, tile_px, radius, k_vol, k_img):
    w = c.w
    desc = nsa.make_desc(w.n_tokens, w.n_blocks, w.max_block_len, w.n_q_heads, w.n_kv_heads, w.head_dim,
                         k_vol + k_img, w.window, 0.0, False, w.n_gates)
    ws = nsa.workspace(desc)
    idx = torch.full((w.n_blocks, k_vol + k_img), -7, dtype=torch.int32, device="cuda")
    nsa.lsrm_route_camera(desc, c.off, c.coords, w.layout.n_vol_blocks, i32(proj), i32(tiles), tile_px, radius,
                          k_vol, idx, ws)
    torch.cuda.synchronize()
    return to_np(idx), nsa.lsrm_nsa_last_device_status(ws)


def _oracle(w, proj, tiles, tile_px, radius, k_vol, k_img):
    D = oracle_desc(w, top_k=k_vol + k_img)
    return O.route_camera(D, w.off, w.coords, w.layout.n_vol_blocks, proj, tiles, tile_px, radius, k_vol, k_img)


@pytest.mark.parametrize("name,radius,k_vol,k_img", [("sparse", 1, 8, 8), ("ragged_geo", 0, 4, 3),
                                                     ("ragged_geo", 1, 2, 5), ("ragged_geo", 8, 4, 6),
                                                     ("ragged_geo", 0, 1, 6), ("tiny_geo", 1, 0, 4)])
def test_camera_routing_bit_exact(name, radius, k_vol, k_img):
    w = make_workload(name)
    c = DeviceCase(w)
    proj, tiles, tile_px = camera_inputs(w.layout)
    got, st = _route(c, proj, tiles, tile_px, radius, k_vol, k_img)
    assert st == 0
    assert np.array_equal(got, _oracle(w, proj, tiles, tile_px, radius, k_vol, k_img))


def test_camera_routing_fill_and_cameras_that_see_nothing():
    w = make_workload("ragged_geo")
    c = DeviceCase(w)
    proj, tiles, tile_px = camera_inputs(w.layout)
    # half the views look away (depth negated): their tiles give no candidates
    proj2 = proj.copy()
    proj2[::2, 2] = -proj2[::2, 2]
    n_img = w.n_blocks - w.layout.n_vol_blocks
    for k_img in (3, n_img):  # the second asks for every image block: candidates, then the fill
        got, st = _route(c, proj2, tiles, tile_px, 0, 2, k_img)
        assert st == 0
        assert np.array_equal(got, _oracle(w, proj2, tiles, tile_px, 0, 2, k_img))


def test_camera_routing_argument_checks_and_bad_table_entries():
    w = make_workload("ragged_geo")
    c = DeviceCase(w)
    proj, tiles, tile_px = camera_inputs(w.layout)
    nv = w.layout.n_vol_blocks
    with pytest.raises(nsa.NsaError) as e:
        _route(c, proj, tiles, tile_px, 1, nv + 1, 0)
    assert e.value.status == 1  # LSRM_ERR_INVALID_ARG
    with pytest.raises(nsa.NsaError) as e:
        _route(c, proj, tiles, tile_px, 30, 1, 1)  # 2 views x 61^2 slots > 4096
    assert e.value.status == 2  # LSRM_ERR_UNSUPPORTED
    bad = tiles.copy()
    bad[bad >= 0] = 0  # a volume block in the tile table
    _, st = _route(c, proj, bad, tile_px, 1, 1, 1)
    assert st == 5  # LSRM_ERR_BOUNDS


def test_layer_on_camera_routed_indices():
    w = make_workload("tiny_geo")
    c = DeviceCase(w)
    proj, tiles, tile_px = camera_inputs(w.layout)
    k_vol, k_img = 4, 4
    idx_np, st = _route(c, proj, tiles, tile_px, 1, k_vol, k_img)
    assert st == 0
    k = k_vol + k_img
    desc = nsa.make_desc(w.n_tokens, w.n_blocks, w.max_block_len, w.n_q_heads, w.n_kv_heads, w.head_dim, k,
                         w.window, 0.0, False, w.n_gates)
    ws = nsa.workspace(desc)
    B, Hkv, d = w.n_blocks, w.n_kv_heads, w.head_dim
    kc, vc = (torch.empty(B, Hkv, d, dtype=torch.bfloat16, device="cuda") for _ in range(2))
    nsa.lsrm_nsa_compress(desc, c.off, None, c.k, c.v, None, kc, None, vc, ws=ws)
    out = torch.empty(w.n_tokens, w.n_q_heads, d, dtype=torch.bfloat16, device="cuda")
    nsa.lsrm_nsa_attend(desc, c.off, c.q, c.k, c.v, kc, vc, c.gates, i32(idx_np), 1, 0, out, None, ws)
    torch.cuda.synchronize()
    assert nsa.lsrm_nsa_last_device_status(ws) == 0
    qb = np.arange(0, B, max(1, B // 6))
    ref = O.forward(oracle_desc(w, top_k=k), w.off, w.q, w.k, w.v, w.gates, idx_np, qblocks=qb)
    assert_close(to_np(out)[rows_for(w.off, qb)], ref, "camera-routed layer")
