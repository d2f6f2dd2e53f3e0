"""The seeded input generator: published test vectors, rounding, determinism, and the
token counts of the synthetic layouts."""
import ctypes
import math

import numpy as np
import pytest
import torch

from conftest import golden
from workloads import make_workload, lsrm_layout, speed3r_layout, gen_lib, bf16_bits_to_f32
from workloads.nsa_workloads import (normal_bf16, f32_to_bf16_bits, speed3r_forced, STREAM_Q,
                                     fibonacci_cameras)


def _u64(n):
    return np.zeros(n, dtype=np.uint64)


def test_splitmix64_reference_vector():
    out = _u64(3)
    gen_lib().nsa_gen_splitmix64(0, 3, out.ctypes.data)
    want = [int(x, 16) for x in golden("splitmix64.txt")[0]]
    assert [int(x) for x in out] == want


def test_xoshiro256ss_first_output_from_small_state():
    # xoshiro256**: output = rotl(s1 * 5, 7) * 9; from state (1, 2, 3, 4) that is rotl(10, 7) * 9 = 11520
    st = np.array([1, 2, 3, 4], dtype=np.uint64)
    out = _u64(2)
    gen_lib().nsa_gen_xoshiro_from_state(st.ctypes.data, 2, out.ctypes.data)
    assert int(out[0]) == 11520
    # second output from the state after one step: s = (7, 0, 262146, rotl(6, 45))
    # output = rotl(0 * 5, 7) * 9 = 0
    assert int(out[1]) == 0


def test_bf16_rounding_matches_torch():
    x = normal_bf16(3, 9, (200000,), 1.0)
    # re-derive: the generator rounds float32 values; torch's float32->bf16 cast is RNE too
    f = bf16_bits_to_f32(x)
    back = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(back, x)
    vals = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, 1e-30, 3.0e38], dtype=np.float32)
    ours = f32_to_bf16_bits(vals)
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_normals_are_standard_and_thread_independent():
    a = normal_bf16(7, STREAM_Q, (1 << 20,), 1.0)
    f = bf16_bits_to_f32(a).astype(np.float64)
    assert abs(f.mean()) < 5e-3 and abs(f.std() - 1.0) < 5e-3
    lib = gen_lib()
    b = np.empty(1 << 20, dtype=np.uint16)
    lib.nsa_gen_normal_bf16(7, STREAM_Q, b.size, 1.0, b.ctypes.data, 1)
    assert np.array_equal(a, b)
    c = np.empty(1 << 20, dtype=np.uint16)
    lib.nsa_gen_normal_bf16(8, STREAM_Q, c.size, 1.0, c.ctypes.data, 3)
    assert not np.array_equal(a, c)


def test_tiny_and_dense_layouts():
    t = make_workload("tiny")
    assert (t.n_tokens, t.n_blocks) == (1024, 16)
    assert t.layout.n_vol_blocks == 8 and t.layout.n_img_blocks == 8
    assert np.all(np.diff(t.off) == 64)
    d = make_workload("dense")
    assert (d.n_tokens, d.n_blocks, d.top_k) == (20480, 320, 320)
    g = bf16_bits_to_f32(d.gates)
    assert np.all(g[..., 0] == 0) and np.all(g[..., 1] == 1) and np.all(g[..., 2] == 0)


def test_sparse_stage_layout_counts():
    lay = lsrm_layout(64, 16, 64, 32, (0.35, 0.45), True, seed=0)
    assert lay.n_vol_blocks == 1384          # bricks touching the shell
    assert lay.n_img_blocks == 16 * 32       # 32 tiles kept per view
    assert lay.n_tokens == 1384 * 64 + 512 * 64 == 121344
    assert np.all(np.diff(lay.off) == 64)
    # the voxel-exact shell has 52976 voxels
    exact = lsrm_layout(64, 0, 64, None, (0.35, 0.45), False)
    assert exact.n_tokens == 52976 and exact.n_blocks == 1384
    # volume lattice coordinates are 16 * voxel + 8
    c = lay.coords[: 1384 * 64]
    assert np.all(c % 16 == 8)
    # image points lie near the r = 0.45 sphere: |16*64*(p+0.5) - 512| ~ 0.45 * 1024
    img = lay.coords[1384 * 64:].astype(np.float64)
    r = np.linalg.norm(img / 1024.0 - 0.5, axis=1)
    assert np.all(np.abs(r - 0.45) < 0.06)


def test_half_fov_gives_half_silhouette():
    # tan(theta) = tan(asin(0.45/2)) * sqrt(pi/2): the sphere's disc covers half the image square
    lay = lsrm_layout(16, 1, 64, None, None)
    t = lay.meta["tan_half_fov"]
    alpha = math.asin(0.45 / 2.0)
    assert abs(math.pi * math.tan(alpha) ** 2 / (4 * t * t) - 0.5) < 1e-12


def test_fibonacci_cameras_look_at_origin():
    pos, fwd, right, up = fibonacci_cameras(16, 2.0)
    assert np.allclose(np.linalg.norm(pos, axis=1), 2.0)
    assert np.allclose(fwd, -pos / 2.0)
    assert np.allclose((right * fwd).sum(1), 0) and np.allclose((up * fwd).sum(1), 0)


def test_speed3r_layout():
    lay = speed3r_layout(512)
    assert (lay.n_tokens, lay.n_blocks) == (701440, 51712)
    sz = np.diff(lay.off)[:101]
    assert sz[0] == 1 and sorted(np.bincount(sz)[[1, 4, 16]].tolist()) == [2, 18, 81]
    forced = speed3r_forced(lay)
    assert len(forced) == 101 + 511 and np.all(np.diff(forced) > 0)


def test_workloads_are_seeded():
    a = make_workload("tiny", seed=1)
    b = make_workload("tiny", seed=1)
    c = make_workload("tiny", seed=2)
    assert np.array_equal(a.q, b.q) and np.array_equal(a.gates, b.gates)
    assert not np.array_equal(a.q, c.q)
    s = bf16_bits_to_f32(a.q).astype(np.float64)
    assert abs(s.std() * math.sqrt(32) - 1.0) < 0.02


def test_mixture_workloads_split_the_streams_at_the_volume_blocks():
    for name, n, nx_blocks in (("mixture", 20480, 64), ("mixture_small", 1024, 8), ("mixture_ragged", 1472, 56)):
        w = make_workload(name)
        assert w.n_tokens == n and w.n_blocks_x == nx_blocks and w.n_gates == 2
        assert w.gates.shape == (n, w.n_q_heads, 2)
        # volume blocks come first: every volume token lies on the voxel lattice (16 i + 8)
        vol = w.coords[: w.off[w.n_blocks_x]]
        assert np.all(vol % 16 == 8)


def test_camera_inputs_tables_and_projection_shapes():
    lay = lsrm_layout(16, 4, 32, 8, (0.3, 0.45), True)
    from workloads import camera_inputs
    proj, tiles, tile_px = camera_inputs(lay)
    tpr = 32 // 8
    assert proj.shape == (4, 3, 4) and proj.dtype == np.int32 and tiles.shape == (4, tpr, tpr)
    assert tile_px == 8 and np.abs(proj).max() <= (1 << 23) + 1
    kept = tiles[tiles >= 0]
    # every image block appears exactly once, views in order
    assert sorted(kept.tolist()) == list(range(lay.n_vol_blocks, lay.n_blocks))
    assert (tiles >= 0).sum(axis=(1, 2)).tolist() == [8] * 4
