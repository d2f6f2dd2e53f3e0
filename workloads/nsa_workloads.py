"""Synthetic inputs shaped like the workloads of the LSRM and Speed3R pages.

Token layouts follow the block grouping of the LSRM page (hyper.ai, "LSRM",
section 方法, block grouping paragraph): active tokens are grouped into
spatial blocks, image tokens into 8x8 tiles and volume tokens into bricks.
Here bricks are 4x4x4 so that every block holds 64 tokens (the workload
definition fixes 64-token blocks; the page's 8x8x8 bricks are not used).

Tokens are stored block-major: block b owns tokens off[b] .. off[b+1]-1.
Volume blocks come first (bricks in raster order, x fastest; voxels inside a
brick also x fastest), then image tiles, view by view (kept tiles in raster
order, pixels inside a tile row-major).

Every token carries an integer 3D position on a lattice of 1/16 voxel of the
workload's grid G: volume voxel (i, j, k) -> 16*(i, j, k) + 8; an image point p
in world units (the grid spans [-0.5, 0.5]^3) -> floor(16*G*(p + 0.5) + 0.5).
An image token's point is where its pixel-centre ray first hits the sphere of
radius 0.45 (the outer shell radius), or the radial projection onto that sphere
of the ray's closest point to the origin when the ray misses, plus N(0, 0.01^2)
noise per axis, before quantisation.

The Speed3R layout (gist.science, "Speed3R", section 2.1, compression branch)
pools each frame's 37x37 patch grid with 4x4 windows, ceil-sized at the edge
(81 blocks of 16 tokens, 18 of 4, 1 of 1), and puts the frame's camera token
first as a 1-token block.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nsa_gen.c")
_LIB = os.path.join(_HERE, "libnsa_gen.so")

# stream ids of the seeded tensors (generation order)
STREAM_Q, STREAM_K, STREAM_V, STREAM_GATES, STREAM_NOISE, STREAM_DOUT = range(6)

_gen = None


def build_gen_lib(force: bool = False) -> str:
    """Compile the C generator in-tree (gcc, -O2, pthreads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def gen_lib():
    global _gen
    if _gen is None:
        lib = ctypes.CDLL(build_gen_lib())
        u64, i32, dbl, vp = ctypes.c_uint64, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
        lib.nsa_gen_normal_bf16.argtypes = [u64, u64, u64, dbl, vp, i32]
        lib.nsa_gen_sigmoid_normal_bf16.argtypes = [u64, u64, u64, vp, i32]
        lib.nsa_gen_normal_f64.argtypes = [u64, u64, u64, dbl, vp, i32]
        lib.nsa_gen_raw_u64.argtypes = [u64, u64, u64, u64, vp]
        lib.nsa_gen_splitmix64.argtypes = [u64, u64, vp]
        lib.nsa_gen_xoshiro_from_state.argtypes = [vp, u64, vp]
        for f in (lib.nsa_gen_normal_bf16, lib.nsa_gen_sigmoid_normal_bf16, lib.nsa_gen_normal_f64,
                  lib.nsa_gen_raw_u64, lib.nsa_gen_splitmix64, lib.nsa_gen_xoshiro_from_state):
            f.restype = i32
        _gen = lib
    return _gen


def _threads() -> int:
    return max(1, min(64, os.cpu_count() or 1))


def normal_bf16(seed: int, stream: int, shape, scale: float) -> np.ndarray:
    out = np.empty(int(np.prod(shape)), dtype=np.uint16)
    gen_lib().nsa_gen_normal_bf16(seed, stream, out.size, float(scale), out.ctypes.data, _threads())
    return out.reshape(shape)


def sigmoid_normal_bf16(seed: int, stream: int, shape) -> np.ndarray:
    out = np.empty(int(np.prod(shape)), dtype=np.uint16)
    gen_lib().nsa_gen_sigmoid_normal_bf16(seed, stream, out.size, out.ctypes.data, _threads())
    return out.reshape(shape)


def normal_f64(seed: int, stream: int, shape, scale: float) -> np.ndarray:
    out = np.empty(int(np.prod(shape)), dtype=np.float64)
    gen_lib().nsa_gen_normal_f64(seed, stream, out.size, float(scale), out.ctypes.data, _threads())
    return out.reshape(shape)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float32 exactly."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 bit patterns, nearest-even (for fixed inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


# --------------------------------------------------------------------------------------------
# layouts
# --------------------------------------------------------------------------------------------

@dataclass
class Layout:
    off: np.ndarray                    # int32 [B+1]
    coords: Optional[np.ndarray]       # int32 [N, 3] lattice coordinates, or None
    n_vol_blocks: int = 0
    n_img_blocks: int = 0
    meta: dict = field(default_factory=dict)

    @property
    def n_tokens(self) -> int:
        return int(self.off[-1])

    @property
    def n_blocks(self) -> int:
        return len(self.off) - 1


def fibonacci_cameras(n_views: int, dist: float):
    """Camera centres on a Fibonacci sphere of radius dist, each looking at the origin.
    Returns (pos [V,3], forward [V,3], right [V,3], up [V,3])."""
    golden = math.pi * (3.0 - math.sqrt(5.0))
    pos = np.zeros((n_views, 3))
    for i in range(n_views):
        y = 1.0 - 2.0 * (i + 0.5) / n_views
        rr = math.sqrt(max(0.0, 1.0 - y * y))
        phi = i * golden
        pos[i] = dist * np.array([math.cos(phi) * rr, y, math.sin(phi) * rr])
    fwd = -pos / np.linalg.norm(pos, axis=1, keepdims=True)
    world_up = np.array([0.0, 1.0, 0.0])
    right = np.cross(fwd, world_up)
    right /= np.linalg.norm(right, axis=1, keepdims=True)
    up = np.cross(right, fwd)
    return pos, fwd, right, up


def lsrm_layout(grid: int, n_views: int, view_res: int, keep_tiles: Optional[int] = None,
                shell: Optional[tuple] = None, brick_granular: bool = True, seed: int = 0,
                sphere_r: float = 0.45, cam_dist: float = 2.0, noise_std: float = 0.01,
                brick: int = 4, tile: int = 8) -> Layout:
    """Concatenated volume + image token layout of an LSRM NSA layer.

    grid: volume resolution G (G^3 voxels); shell=(r_in, r_out) keeps voxels whose
    centre radius lies in [r_in, r_out] (None keeps all); brick_granular keeps
    every voxel of a brick that touches the shell, so every brick is full.
    n_views cameras, view_res x view_res image tokens each, 8x8 tiles; keep_tiles
    tiles per view are kept (the ones whose centre ray passes closest to the
    origin, ties to the lower tile index; None keeps all)."""
    assert grid % brick == 0 and view_res % tile == 0
    nb = grid // brick
    centres = (np.arange(grid) + 0.5) / grid - 0.5
    if shell is None:
        active = np.ones((grid, grid, grid), dtype=bool)  # [z, y, x]
    else:
        z, y, x = np.meshgrid(centres, centres, centres, indexing="ij")
        r = np.sqrt(x * x + y * y + z * z)
        active = (r >= shell[0]) & (r <= shell[1])
    blocks_active = active.reshape(nb, brick, nb, brick, nb, brick).any(axis=(1, 3, 5))  # [bz,by,bx]
    if shell is not None and brick_granular:
        active = np.repeat(np.repeat(np.repeat(blocks_active, brick, 0), brick, 1), brick, 2)

    sizes, coords = [], []
    lz, ly, lx = np.meshgrid(np.arange(brick), np.arange(brick), np.arange(brick), indexing="ij")
    lx, ly, lz = lx.ravel(), ly.ravel(), lz.ravel()          # x fastest inside the brick
    for bz in range(nb):
        for by in range(nb):
            for bx in range(nb):
                if not blocks_active[bz, by, bx]:
                    continue
                i = bx * brick + lx
                j = by * brick + ly
                k = bz * brick + lz
                m = active[k, j, i]
                if not m.any():
                    continue
                sizes.append(int(m.sum()))
                coords.append(np.stack([16 * i[m] + 8, 16 * j[m] + 8, 16 * k[m] + 8], axis=1))
    n_vol_blocks = len(sizes)

    # images
    tan_half = math.tan(math.asin(sphere_r / cam_dist)) * math.sqrt(math.pi / 2.0)
    pos, fwd, right, up = fibonacci_cameras(n_views, cam_dist)
    tpr = view_res // tile
    tiles = [(tv, tu) for tv in range(tpr) for tu in range(tpr)]
    # exact integer rank: squared pixel offset of the tile centre from the image centre
    half2 = view_res  # twice the image centre in pixel units
    rad2 = [((2 * (tu * tile) + tile - half2) ** 2 + (2 * (tv * tile) + tile - half2) ** 2, t)
            for t, (tv, tu) in enumerate(tiles)]
    order = sorted(rad2)
    kept = sorted(t for _, t in order[: (keep_tiles if keep_tiles is not None else len(tiles))])
    img_pts = []
    py, px = np.meshgrid(np.arange(tile), np.arange(tile), indexing="ij")
    py, px = py.ravel(), px.ravel()  # row-major inside a tile
    for vi in range(n_views):
        for t in kept:
            tv, tu = tiles[t]
            u = tu * tile + px
            v = tv * tile + py
            xs = ((u + 0.5) / view_res * 2.0 - 1.0) * tan_half
            ys = (1.0 - (v + 0.5) / view_res * 2.0) * tan_half
            d = fwd[vi][None, :] + xs[:, None] * right[vi][None, :] + ys[:, None] * up[vi][None, :]
            d /= np.linalg.norm(d, axis=1, keepdims=True)
            o = pos[vi]
            b = d @ o                          # ray: o + s d ; |o + s d|^2 = R^2
            c = o @ o - sphere_r * sphere_r
            disc = b * b - c
            s_hit = -b - np.sqrt(np.maximum(disc, 0.0))
            hit = o[None, :] + s_hit[:, None] * d
            closest = o[None, :] - b[:, None] * d
            proj = sphere_r * closest / np.linalg.norm(closest, axis=1, keepdims=True)
            p = np.where((disc >= 0.0)[:, None], hit, proj)
            img_pts.append(p)
            sizes.append(tile * tile)
    n_img_blocks = len(sizes) - n_vol_blocks
    if img_pts:
        pts = np.concatenate(img_pts, axis=0)
        pts = pts + normal_f64(seed, STREAM_NOISE, pts.shape, noise_std)
        lat = np.floor(16.0 * grid * (pts + 0.5) + 0.5).astype(np.int64)
        coords.append(lat)
    off = np.zeros(len(sizes) + 1, dtype=np.int32)
    off[1:] = np.cumsum(sizes)
    coords_all = np.concatenate(coords, axis=0).astype(np.int32)
    assert coords_all.shape[0] == off[-1]
    return Layout(off=off, coords=coords_all, n_vol_blocks=n_vol_blocks, n_img_blocks=n_img_blocks,
                  meta=dict(grid=grid, n_views=n_views, view_res=view_res, keep_tiles=keep_tiles,
                            shell=shell, brick_granular=brick_granular, tan_half_fov=tan_half, tile=tile,
                            cam_pos=pos, cam_fwd=fwd, cam_right=right, cam_up=up, kept_tiles=kept))


def camera_inputs(layout: Layout, max_entry: int = 1 << 23):
    """The cameras of an LSRM layout as inputs of camera-projection routing.

    proj int32 [V][3][4]: per view a homogeneous projection of a lattice point c (the coords'
    units) to pixel coordinates, u = h0 / h2, v = h1 / h2 with h = P [c; 1] (h2 = depth along
    the view direction), the same pinhole model the image tokens were generated with (pixel
    (u, v) covers [u, u+1) x [v, v+1), rows from the top), scaled so that the largest entry is
    about max_entry and rounded to integers.  tile_block int32 [V][tiles][tiles]: the block id
    of each kept tile, -1 elsewhere.  tile_px: pixels per tile side.  Returns
    (proj, tile_block, tile_px)."""
    m = layout.meta
    G, R, tile, th = m["grid"], m["view_res"], m["tile"], m["tan_half_fov"]
    s = 1.0 / (16.0 * G)                     # lattice unit in world units; world = s c - 0.5
    V = m["n_views"]
    tpr = R // tile
    proj = np.zeros((V, 3, 4), dtype=np.int32)
    tile_block = np.full((V, tpr, tpr), -1, dtype=np.int32)
    kept = m["kept_tiles"]
    for v in range(V):
        pos, fwd, right, up = m["cam_pos"][v], m["cam_fwd"][v], m["cam_right"][v], m["cam_up"][v]
        rows = np.stack([0.5 * R * (right / th + fwd), 0.5 * R * (fwd - up / th), fwd])  # [3][3]
        o = -0.5 - pos                         # world offset of lattice point 0, relative to the camera
        P = np.concatenate([rows * s, (rows @ o)[:, None]], axis=1)
        proj[v] = np.rint(P * (max_entry / np.abs(P).max())).astype(np.int32)
        for r, t in enumerate(kept):
            tile_block[v, t // tpr, t % tpr] = layout.n_vol_blocks + v * len(kept) + r
    return proj, tile_block, tile


def speed3r_layout(n_frames: int, patch: int = 37, pool: int = 4) -> Layout:
    """Frame-by-frame Speed3R layout: a 1-token camera block, then the frame's
    patch grid pooled into ceil(patch/pool)^2 blocks in raster order."""
    nbx = -(-patch // pool)
    sizes = []
    for _ in range(n_frames):
        sizes.append(1)
        for by in range(nbx):
            for bx in range(nbx):
                h = min(pool, patch - by * pool)
                w = min(pool, patch - bx * pool)
                sizes.append(h * w)
    off = np.zeros(len(sizes) + 1, dtype=np.int32)
    off[1:] = np.cumsum(sizes)
    return Layout(off=off, coords=None, meta=dict(n_frames=n_frames, patch=patch, pool=pool,
                                                   blocks_per_frame=1 + nbx * nbx))


def speed3r_forced(layout: Layout) -> np.ndarray:
    """Blocks every query always selects (Speed3R page, section 2.2, VGGT variant):
    all blocks of frame 0 and the camera block of every frame; sorted, unique."""
    bpf = layout.meta["blocks_per_frame"]
    nf = layout.meta["n_frames"]
    forced = set(range(bpf)) | {f * bpf for f in range(nf)}
    return np.array(sorted(forced), dtype=np.int32)


# --------------------------------------------------------------------------------------------
# workloads
# --------------------------------------------------------------------------------------------

@dataclass
class Workload:
    name: str
    layout: Layout
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    top_k: int
    window: int
    route: str                 # "score" | "geom" | "all"
    pooled_q: bool
    n_gates: int
    q: np.ndarray              # uint16 bf16 bits [N, Hq, d]
    k: np.ndarray              # [N, Hkv, d]
    v: np.ndarray              # [N, Hkv, d]
    gates: np.ndarray          # [N, Hq, n_gates]
    forced: np.ndarray         # int32 sorted unique block ids (Speed3R), else empty
    dout: Optional[np.ndarray] = None
    seed: int = 0
    description: str = ""

    @property
    def off(self):
        return self.layout.off

    @property
    def coords(self):
        return self.layout.coords

    @property
    def n_tokens(self):
        return self.layout.n_tokens

    @property
    def n_blocks(self):
        return self.layout.n_blocks

    @property
    def max_block_len(self):
        return int(np.diff(self.layout.off).max())

    @property
    def scale(self):
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def n_blocks_x(self):
        """Blocks of the first stream (the volume tokens) in the self/cross mixture."""
        return int(self.layout.n_vol_blocks)


def _tensors(layout: Layout, hq: int, hkv: int, d: int, n_gates: int, seed: int, scale: float,
             fixed_gates=None, with_dout=False):
    n = layout.n_tokens
    q = normal_bf16(seed, STREAM_Q, (n, hq, d), scale)
    k = normal_bf16(seed, STREAM_K, (n, hkv, d), scale)
    v = normal_bf16(seed, STREAM_V, (n, hkv, d), scale)
    if fixed_gates is None:
        g = sigmoid_normal_bf16(seed, STREAM_GATES, (n, hq, n_gates))
    else:
        g = np.empty((n, hq, n_gates), dtype=np.uint16)
        g[...] = f32_to_bf16_bits(np.array(fixed_gates, dtype=np.float32))
    dout = normal_bf16(seed, STREAM_DOUT, (n, hq, d), 1.0) if with_dout else None
    return q, k, v, g, dout


WORKLOAD_NAMES = ("tiny", "dense", "sparse", "speed3r", "backward",
                  "tiny_geo", "ragged_geo", "speed3r_small", "backward_small",
                  "mixture", "mixture_small", "mixture_ragged")


def make_workload(name: str, seed: int = 0, **kw) -> Workload:
    """Named workloads.

    tiny      1024 tokens: 8^3 grid (8 bricks) + 2 views of 16x16 (8 tiles); GQA 32/2, d 32;
              top-4 by compressed score; window 64.
    dense     20480 tokens: 16^3 grid + 16 views of 32x32; k = all 320 blocks; gates (0, 1, 0)
              so that the layer equals dense GQA attention.
    sparse    the LSRM sparse stage: 1384 shell bricks of a 64^3 grid + 16 views of 64x64 with
              32 of 64 tiles kept per view; geometric top-16; window 64 (121344 tokens).
    speed3r   512 frames x (1 camera + 37x37 patches); MHA 16 heads, d 64; pooled-Q
              compression; top-32 plus forced blocks (frame 0, camera tokens); 2 gates.
    backward  the sparse workload plus an upstream gradient dO ~ N(0, 1).
    sparse_vol512 / small_vol512 / ragged_vol512: the pages' 8x8x8 volume blocks (512 tokens) with
              8x8 image tiles (the sparse stage, a small case, and a voxel-exact case of ragged blocks).
    small variants (test sizes): tiny_geo, ragged_geo (voxel-exact shell: partial blocks),
              speed3r_small, backward_small.
    mixture   the decoupled self/cross gated mixture at the dense-stage shape (16^3 volume tokens
              + 16 views of 32x32 image tokens, 20480 tokens); 2 gates (self, cross) ~ sigmoid(N(0,1)).
    mixture_small / mixture_ragged: the same on the tiny layout, and on the voxel-exact shell
              (ragged volume blocks).
    """
    d32 = 1.0 / math.sqrt(32.0)
    if name == "tiny":
        lay = lsrm_layout(8, 2, 16, None, None, seed=seed)
        hq, hkv, d, k, w, route = 32, 2, 32, 4, 64, "score"
        fixed, ng, sc, pooled = None, 3, d32, False
        desc = "1024 tokens (8^3 grid + 2 views 16x16), GQA 32/2, d 32, score top-4, window 64"
    elif name == "dense":
        lay = lsrm_layout(16, 16, 32, None, None, seed=seed)
        hq, hkv, d, k, w, route = 32, 2, 32, lay.n_blocks, 64, "all"
        fixed, ng, sc, pooled = (0.0, 1.0, 0.0), 3, d32, False
        desc = "20480 tokens (16^3 grid + 16 views 32x32), k = all 320 blocks, gates (0,1,0)"
    elif name in ("sparse", "backward"):
        lay = lsrm_layout(64, 16, 64, 32, (0.35, 0.45), True, seed=seed)
        hq, hkv, d, k, w, route = 32, 2, 32, 16, 64, "geom"
        fixed, ng, sc, pooled = None, 3, d32, False
        desc = ("121344 tokens (1384 shell bricks of 64^3 + 16 views 64x64, 32 tiles kept), "
                "geometric top-16, window 64")
    elif name == "tiny_geo":
        lay = lsrm_layout(16, 4, 32, 8, (0.3, 0.45), True, seed=seed)
        hq, hkv, d, k, w, route = 32, 2, 32, 8, 64, "geom"
        fixed, ng, sc, pooled = None, 3, d32, False
        desc = "small geometric-routing case (shell bricks of 16^3 + 4 views 32x32, 8 tiles kept)"
    elif name == "ragged_geo":
        lay = lsrm_layout(16, 2, 16, 3, (0.3, 0.45), False, seed=seed)
        hq, hkv, d, k, w, route = 32, 2, 32, 5, 64, "geom"
        fixed, ng, sc, pooled = None, 3, d32, False
        desc = "voxel-exact shell (partial blocks) + 2 views 16x16, 3 tiles kept, top-5"
    elif name in ("speed3r", "speed3r_small"):
        nf = 512 if name == "speed3r" else kw.pop("n_frames", 6)
        lay = speed3r_layout(nf)
        hq, hkv, d, k, w, route = 16, 16, 64, 32, 0, "score"
        fixed, ng, sc, pooled = None, 2, 1.0 / 8.0, True
        desc = f"{nf} frames x (1 camera + 37x37 patches), MHA 16 x 64, pooled-Q, top-32 + forced"
    elif name in ("sparse_vol512", "small_vol512", "ragged_vol512"):
        # the pages' 8x8x8 volume blocks (512 tokens) with 8x8 image tiles
        if name == "sparse_vol512":
            lay = lsrm_layout(64, 16, 64, 32, (0.35, 0.45), True, seed=seed, brick=8)
        elif name == "small_vol512":
            lay = lsrm_layout(16, 4, 32, 8, (0.3, 0.45), True, seed=seed, brick=8)
        else:
            lay = lsrm_layout(16, 2, 16, 3, (0.3, 0.45), False, seed=seed, brick=8)
        hq, hkv, d, k, w, route = 32, 2, 32, 16 if name == "sparse_vol512" else 4, 64, "geom"
        fixed, ng, sc, pooled = None, 3, d32, False
        desc = f"{name}: 8x8x8 volume blocks (512 tokens) + 8x8 image tiles, geometric top-{k}, window 64"
    elif name in ("mixture", "mixture_small", "mixture_ragged"):
        if name == "mixture":
            lay = lsrm_layout(16, 16, 32, None, None, seed=seed)
        elif name == "mixture_small":
            lay = lsrm_layout(8, 2, 16, None, None, seed=seed)
        else:
            lay = lsrm_layout(16, 2, 16, 3, (0.3, 0.45), False, seed=seed)
        hq, hkv, d, k, w, route = 32, 2, 32, 1, 0, "mixture"
        fixed, ng, sc, pooled = None, 2, d32, False
        desc = f"{name}: self/cross gated mixture of the volume and image streams ({lay.n_tokens} tokens)"
    elif name == "backward_small":
        lay = lsrm_layout(16, 4, 32, 8, (0.3, 0.45), True, seed=seed)
        hq, hkv, d, k, w, route = 32, 2, 32, 8, 64, "geom"
        fixed, ng, sc, pooled = None, 3, d32, False
        desc = "backward on the small geometric case"
    else:
        raise ValueError(f"unknown workload {name!r}")
    hq = kw.pop("n_q_heads", hq)
    hkv = kw.pop("n_kv_heads", hkv)
    d = kw.pop("head_dim", d)
    k = kw.pop("top_k", k)
    w = kw.pop("window", w)
    if kw:
        raise TypeError(f"unknown overrides {sorted(kw)}")
    q, kk, v, g, dout = _tensors(lay, hq, hkv, d, ng, seed, sc, fixed,
                                 with_dout=name in ("backward", "backward_small"))
    forced = speed3r_forced(lay) if pooled else np.zeros(0, dtype=np.int32)
    return Workload(name=name, layout=lay, n_q_heads=hq, n_kv_heads=hkv, head_dim=d, top_k=k,
                    window=w, route=route, pooled_q=pooled, n_gates=ng, q=q, k=kk, v=v, gates=g,
                    forced=forced, dout=dout, seed=seed, description=desc)
