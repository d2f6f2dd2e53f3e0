"""Pins of the oracle's camera-projection routing (LSRM page, 方法, 3D-aware routing paragraph:
the query point is projected into every view, the view's nearby image blocks are retrieved and
ranked by their smallest 3D distance to the query point; volume blocks by centre distance).

* a hand-made case whose rows are worked out by hand below (projection, division by depth,
  tile floor, x/y order, the neighbourhood, the ranking by closest token, the fill by centroid
  distance, a camera that sees nothing);
* a brute force in numpy on a real small layout with a neighbourhood covering every tile, where
  every image block is a candidate;
* the layout generator's cameras: noise-free image tokens project back into their own tile.
"""
import numpy as np
import pytest

from oracle import oracle as O
from workloads import camera_inputs, lsrm_layout, make_workload

# hand-made layout: 4 volume blocks, then 6 image blocks, 2 tokens each (x, y, z lattice points)
_TOK = [
    [(2, 2, 0), (4, 4, 0)],      # 0 vol, centroid (3, 3, 0)
    [(30, 30, 0), (30, 30, 0)],  # 1 vol, centroid (30, 30, 0)
    [(10, 2, 0), (10, 2, 0)],    # 2 vol, centroid (10, 2, 0)
    [(60, 60, 60), (60, 60, 60)],  # 3 vol, centroid (60, 60, 60)
    [(1, 1, 1), (7, 7, 0)],      # 4 img, centroid (4, 4, 1)
    [(9, 1, 0), (5, 3, 0)],      # 5 img, centroid (7, 2, 0)
    [(2, 9, 0), (3, 12, 0)],     # 6 img, centroid (3, 11, 0)
    [(9, 9, 0), (15, 15, 0)],    # 7 img, centroid (12, 12, 0)
    [(28, 28, 0), (31, 31, 0)],  # 8 img, centroid (30, 30, 0)
    [(17, 2, 0), (20, 4, 0)],    # 9 img, centroid (19, 3, 0)
]
# one view: pixel = (floor(x / 2), floor(y / 2)) (depth 2), 4x4 tiles of 4 pixels: tile = floor(x / 8)
_PROJ = np.array([[[1, 0, 0, 0], [0, 1, 0, 0], [0, 0, 0, 2]]], dtype=np.int32)
_TILES = np.full((1, 4, 4), -1, dtype=np.int32)  # [view][ty][tx]
for (tx, ty), b in {(0, 0): 4, (1, 0): 5, (0, 1): 6, (1, 1): 7, (3, 3): 8, (2, 0): 9}.items():
    _TILES[0, ty, tx] = b


def _hand():
    off = np.zeros(len(_TOK) + 1, dtype=np.int32)
    off[1:] = np.cumsum([len(t) for t in _TOK])
    coords = np.array([p for blk in _TOK for p in blk], dtype=np.int32)
    D = O.desc_for(len(coords), len(_TOK), 2, 1, 32, 1, 0)
    return D, off, coords


def test_camera_routing_hand_worked_case():
    D, off, coords = _hand()
    idx = O.route_camera(D, off, coords, 4, _PROJ, _TILES, 4, 1, 2, 3)
    # block 0, point (3, 3, 0): pixel (1, 1), tile (0, 0); the 3x3 neighbourhood holds blocks 4, 5,
    # 6, 7; closest tokens 9, 4, 37, 72 -> 5, 4, 6.  Volume: 0 (d 0), 2 (d 50).
    assert idx[0].tolist() == [0, 2, 5, 4, 6]
    # block 1, point (30, 30, 0): pixel (15, 15), tile (3, 3) -> only block 8; then the fill by
    # centroid distance: 7 (648), 9 (850).  Volume: 1 (0), 2 (1184) ahead of 0 (1458).
    assert idx[1].tolist() == [1, 2, 8, 7, 9]
    # block 3, point (60, 60, 60): pixel (30, 30), tile (7, 7), outside the grid: all fill
    # (centroid distances to 8, 7, 9 ...: 2*30^2+60^2 = 5400, 2*48^2+60^2 = 8208, 41^2+57^2+60^2 = 8530)
    assert idx[3].tolist()[2:] == [8, 7, 9]
    # more image blocks asked than candidates: 5, 4, 6, 7, then 9 (256) and 8 (1458) by centroid
    idx6 = O.route_camera(D, off, coords, 4, _PROJ, _TILES, 4, 1, 2, 6)
    assert idx6[0].tolist() == [0, 2, 5, 4, 6, 7, 9, 8]
    # radius 0: block 2, point (10, 2, 0): pixel (5, 1), tile x 1, y 0 -> block 5 (not 6)
    idx0 = O.route_camera(D, off, coords, 4, _PROJ, _TILES, 4, 0, 2, 1)
    assert idx0[2].tolist() == [2, 0, 5]


def test_camera_routing_view_behind_the_points_gives_no_candidates():
    D, off, coords = _hand()
    proj = _PROJ.copy()
    proj[0, 2] = [0, 0, 1, -10]  # depth z - 10 < 0 for every point
    idx = O.route_camera(D, off, coords, 4, proj, _TILES, 4, 1, 2, 3)
    # only the fill: by centroid distance from (3, 3, 0): 4 (3), 5 (17), 6 (64)
    assert idx[0].tolist() == [0, 2, 4, 5, 6]


def test_camera_routing_rejects_counts_above_the_blocks():
    D, off, coords = _hand()
    with pytest.raises(ValueError):
        O.route_camera(D, off, coords, 4, _PROJ, _TILES, 4, 1, 5, 1)
    with pytest.raises(ValueError):
        O.route_camera(D, off, coords, 4, _PROJ, _TILES, 4, 1, 1, 7)


def test_camera_routing_equals_brute_force_when_every_tile_is_near():
    w = make_workload("ragged_geo")
    lay = w.layout
    proj, tiles, tile_px = camera_inputs(lay)
    nv, B = lay.n_vol_blocks, lay.n_blocks
    k_vol, k_img = 4, 3
    D = O.desc_for(w.n_tokens, B, 32, 2, 32, k_vol + k_img, 64)
    idx = O.route_camera(D, w.off, w.coords, nv, proj, tiles, tile_px, tiles.shape[1], k_vol, k_img)
    c = w.coords.astype(np.int64)
    off = w.off.astype(np.int64)
    n = np.diff(off)
    S = np.add.reduceat(c, off[:-1], axis=0)
    cen = np.floor_divide(2 * S + n[:, None], 2 * n[:, None])
    for a in range(B):
        dv = ((cen[:nv] - cen[a]) ** 2).sum(axis=1)
        vol = np.lexsort((np.arange(nv), dv))[:k_vol]
        dt = ((c - cen[a]) ** 2).sum(axis=1)
        mind = np.minimum.reduceat(dt, off[:-1])[nv:]
        img = nv + np.lexsort((np.arange(B - nv), mind))[:k_img]
        assert idx[a].tolist() == vol.tolist() + img.tolist(), a


def test_generator_cameras_project_noise_free_tokens_into_their_own_tile():
    lay = lsrm_layout(16, 4, 32, 8, (0.3, 0.45), True, noise_std=0.0)
    proj, tiles, tile_px = camera_inputs(lay)
    per_view = (tiles[0] >= 0).sum()
    c = lay.coords.astype(np.int64)
    for b in range(lay.n_vol_blocks, lay.n_blocks):
        v = (b - lay.n_vol_blocks) // per_view
        P = proj[v].astype(np.int64)
        h = c[lay.off[b]:lay.off[b + 1]] @ P[:, :3].T + P[:, 3]
        assert np.all(h[:, 2] > 0)
        tx = np.floor_divide(np.floor_divide(h[:, 0], h[:, 2]), tile_px)
        ty = np.floor_divide(np.floor_divide(h[:, 1], h[:, 2]), tile_px)
        assert np.all(tiles[v, ty, tx] == b), b
