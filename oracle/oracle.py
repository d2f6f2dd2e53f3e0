"""ORACLE — test infrastructure, not product code.

ctypes wrapper around liboracle_nsa.so (built from nsa_oracle.cpp with g++).
Every function takes numpy arrays: bf16 tensors as uint16 bit patterns, or
float64 arrays for the ``*_f64`` variants used by finite-difference checks.
Outputs are float64.  Query-side outputs cover the listed query blocks only,
compacted in list order (rows = tokens of qblocks[0], then qblocks[1], ...).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nsa_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle_nsa.so")

__all__ = ["build_oracle", "OracleDesc", "desc_for", "compress", "route_geometric", "route_score",
           "route_pooled", "cmp_attn", "select_attn", "window_attn", "forward", "backward", "loss_f64",
           "forward_f64", "backward_f64", "backward_pooled", "backward_pooled_f64", "loss_forced_f64", "mixture", "route_camera", "rows_of"]


class OracleDesc(ctypes.Structure):
    _fields_ = [("n_tokens", ctypes.c_int64), ("n_blocks", ctypes.c_int32),
                ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("window", ctypes.c_int32), ("scale", ctypes.c_double),
                ("pooled_q", ctypes.c_int32), ("n_gates", ctypes.c_int32)]


def build_oracle(force: bool = False) -> str:
    """Compile the oracle in-tree with g++ -O2 (plain C++17, no special flags)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-o", tmp, _SRC, "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build_oracle())
        vp = ctypes.c_void_p
        i32 = ctypes.c_int32
        P = ctypes.POINTER(OracleDesc)
        sig = {
            "oracle_compress": [P, vp, vp, i32, vp],
            "oracle_compress_f64": [P, vp, vp, i32, vp],
            "oracle_route_geometric": [P, vp, vp, vp, vp],
            "oracle_route_score": [P, vp, vp, vp, i32, vp, vp, vp],
            "oracle_route_pooled": [P, vp, vp, i32, vp, i32, vp, vp, vp],
            "oracle_cmp_attn": [P, vp, vp, vp, vp, vp, i32, vp, vp, vp],
            "oracle_select_attn": [P, vp, vp, vp, vp, vp, i32, i32, vp, i32, vp, vp, vp],
            "oracle_window_attn": [P, vp, vp, vp, vp, i32, vp, vp, vp],
            "oracle_forward": [P, vp, vp, vp, vp, vp, vp, i32, i32, vp, i32, vp, vp, vp, vp],
            "oracle_forward_f64": [P, vp, vp, vp, vp, vp, vp, i32, i32, vp, i32, vp, vp, vp, vp],
            "oracle_backward": [P, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, i32, vp, i32],
            "oracle_backward_f64": [P, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, i32, vp, i32],
            "oracle_loss_f64": [P, vp, vp, vp, vp, vp, vp, i32, vp],
            "oracle_loss_forced_f64": [P, vp, vp, vp, vp, vp, vp, i32, vp, i32, vp],
            "oracle_backward_pooled": [P, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp, i32],
            "oracle_backward_pooled_f64": [P, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp, i32],
            "oracle_mixture": [P, vp, vp, vp, vp, vp, i32, i32, vp, vp, vp, vp],
            "oracle_route_camera": [P, vp, vp, i32, i32, vp, i32, i32, i32, vp, i32, i32, i32, vp],
        }
        for name, args in sig.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = ctypes.c_double if name.startswith("oracle_loss") else ctypes.c_int
        _lib = lib
    return _lib


def desc_for(n_tokens: int, n_blocks: int, n_q_heads: int, n_kv_heads: int, head_dim: int, top_k: int,
             window: int, n_gates: int = 3, pooled_q: bool = False, scale: float = 0.0) -> OracleDesc:
    return OracleDesc(int(n_tokens), int(n_blocks), int(n_q_heads), int(n_kv_heads), int(head_dim),
                      int(top_k), int(window), float(scale), int(bool(pooled_q)), int(n_gates))


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def rows_of(off: np.ndarray, qblocks: Sequence[int]) -> int:
    off = np.asarray(off)
    qb = np.asarray(qblocks, dtype=np.int64)
    return int((off[qb + 1] - off[qb]).sum())


def _inputs(dtype, *arrs):
    return [_c(a, dtype) for a in arrs]


def compress(D: OracleDesc, off, x, n_heads: int) -> np.ndarray:
    """Block means [B][H][d] of a [N][H][d] tensor (bf16 bits, or float64)."""
    off = _c(off, np.int32)
    out = np.zeros((D.n_blocks, n_heads, D.head_dim))
    if np.asarray(x).dtype == np.float64:
        x = _c(x, np.float64)
        _L().oracle_compress_f64(ctypes.byref(D), _p(off), _p(x), n_heads, _p(out))
    else:
        x = _c(x, np.uint16)
        _L().oracle_compress(ctypes.byref(D), _p(off), _p(x), n_heads, _p(out))
    return out


def route_geometric(D: OracleDesc, off, coords):
    """Top-k nearest blocks by squared integer centroid distance: (idx [B][k], centroids [B][3])."""
    off, coords = _c(off, np.int32), _c(coords, np.int32)
    idx = np.zeros((D.n_blocks, D.top_k), dtype=np.int32)
    cen = np.zeros((D.n_blocks, 3), dtype=np.int64)
    _L().oracle_route_geometric(ctypes.byref(D), _p(off), _p(coords), _p(idx), _p(cen))
    return idx, cen


def route_score(D: OracleDesc, off, q, kc, qblocks=None):
    """Score routing: (idx [nq][Hkv][k], score [nq][Hkv][B]) for the listed query blocks."""
    qblocks = np.arange(D.n_blocks, dtype=np.int32) if qblocks is None else _c(qblocks, np.int32)
    off, q, kc = _c(off, np.int32), _c(q, np.uint16), _c(kc, np.float64)
    nq = len(qblocks)
    idx = np.zeros((nq, D.n_kv_heads, D.top_k), dtype=np.int32)
    score = np.zeros((nq, D.n_kv_heads, D.n_blocks))
    _L().oracle_route_score(ctypes.byref(D), _p(off), _p(q), _p(kc), nq, _p(qblocks), _p(idx), _p(score))
    return idx, score


def route_pooled(D: OracleDesc, qc, kc, forced, qblocks=None, want_logits=False):
    """Speed3R routing: (idx [nq][H][k], logits [nq][H][B] or None)."""
    qblocks = np.arange(D.n_blocks, dtype=np.int32) if qblocks is None else _c(qblocks, np.int32)
    qc, kc, forced = _c(qc, np.float64), _c(kc, np.float64), _c(forced, np.int32)
    nq = len(qblocks)
    idx = np.zeros((nq, D.n_q_heads, D.top_k), dtype=np.int32)
    logits = np.zeros((nq, D.n_q_heads, D.n_blocks)) if want_logits else None
    _L().oracle_route_pooled(ctypes.byref(D), _p(qc), _p(kc), len(forced), _p(forced), nq, _p(qblocks),
                             _p(idx), _p(logits))
    return idx, logits


def cmp_attn(D: OracleDesc, off, q, kc, vc, qc=None, qblocks=None):
    qblocks = np.arange(D.n_blocks, dtype=np.int32) if qblocks is None else _c(qblocks, np.int32)
    off, q = _c(off, np.int32), _c(q, np.uint16)
    kc, vc, qc = _c(kc, np.float64), _c(vc, np.float64), _c(qc, np.float64)
    rows = rows_of(off, qblocks)
    o = np.zeros((rows, D.n_q_heads, D.head_dim))
    lse = np.zeros((rows, D.n_q_heads))
    _L().oracle_cmp_attn(ctypes.byref(D), _p(off), _p(q), _p(kc), _p(vc), _p(qc), len(qblocks), _p(qblocks),
                         _p(o), _p(lse))
    return o, lse


def select_attn(D: OracleDesc, off, q, k, v, idx, forced=None, qblocks=None):
    """idx: [B][k] (shared by all groups) or [B][Hkv][k] (per group)."""
    qblocks = np.arange(D.n_blocks, dtype=np.int32) if qblocks is None else _c(qblocks, np.int32)
    off, q, k, v = _c(off, np.int32), _c(q, np.uint16), _c(k, np.uint16), _c(v, np.uint16)
    idx = _c(idx, np.int32)
    idx_heads = 1 if idx.ndim == 2 else idx.shape[1]
    forced = np.zeros(0, np.int32) if forced is None else _c(forced, np.int32)
    rows = rows_of(off, qblocks)
    o = np.zeros((rows, D.n_q_heads, D.head_dim))
    lse = np.zeros((rows, D.n_q_heads))
    _L().oracle_select_attn(ctypes.byref(D), _p(off), _p(q), _p(k), _p(v), _p(idx), idx_heads, len(forced),
                            _p(forced), len(qblocks), _p(qblocks), _p(o), _p(lse))
    return o, lse


def window_attn(D: OracleDesc, off, q, k, v, qblocks=None):
    qblocks = np.arange(D.n_blocks, dtype=np.int32) if qblocks is None else _c(qblocks, np.int32)
    off, q, k, v = _c(off, np.int32), _c(q, np.uint16), _c(k, np.uint16), _c(v, np.uint16)
    rows = rows_of(off, qblocks)
    o = np.zeros((rows, D.n_q_heads, D.head_dim))
    lse = np.zeros((rows, D.n_q_heads))
    _L().oracle_window_attn(ctypes.byref(D), _p(off), _p(q), _p(k), _p(v), len(qblocks), _p(qblocks), _p(o),
                            _p(lse))
    return o, lse


def _forward(fn, dtype, D, off, q, k, v, gates, idx, forced, qblocks, want_branches):
    qblocks = np.arange(D.n_blocks, dtype=np.int32) if qblocks is None else _c(qblocks, np.int32)
    off = _c(off, np.int32)
    q, k, v, gates = _inputs(dtype, q, k, v, gates)
    idx = _c(idx, np.int32)
    idx_heads = 1 if idx.ndim == 2 else idx.shape[1]
    forced = np.zeros(0, np.int32) if forced is None else _c(forced, np.int32)
    rows = rows_of(off, qblocks)
    out = np.zeros((rows, D.n_q_heads, D.head_dim))
    br = np.zeros((rows, D.n_q_heads, D.n_gates, D.head_dim)) if want_branches else None
    lse = np.zeros((rows, D.n_q_heads, D.n_gates)) if want_branches else None
    fn(ctypes.byref(D), _p(off), _p(q), _p(k), _p(v), _p(gates), _p(idx), idx_heads, len(forced), _p(forced),
       len(qblocks), _p(qblocks), _p(out), _p(br), _p(lse))
    return (out, br, lse) if want_branches else out


def forward(D, off, q, k, v, gates, idx, forced=None, qblocks=None, want_branches=False):
    """Layer output for the listed query blocks (all blocks by default).
    With want_branches: (out, branches [rows][Hq][n_gates][d], lse [rows][Hq][n_gates])."""
    return _forward(_L().oracle_forward, np.uint16, D, off, q, k, v, gates, idx, forced, qblocks, want_branches)


def forward_f64(D, off, q, k, v, gates, idx, forced=None, qblocks=None, want_branches=False):
    return _forward(_L().oracle_forward_f64, np.float64, D, off, q, k, v, gates, idx, forced, qblocks,
                    want_branches)


def _backward(fn, dtype, D, off, q, k, v, gates, idx, dout, nthreads, qblocks=None):
    off = _c(off, np.int32)
    q, k, v, gates, dout = _inputs(dtype, q, k, v, gates, dout)
    idx = _c(idx, np.int32)
    idx_heads = 1 if idx.ndim == 2 else idx.shape[1]
    N = D.n_tokens
    dq = np.zeros((N, D.n_q_heads, D.head_dim))
    dk = np.zeros((N, D.n_kv_heads, D.head_dim))
    dv = np.zeros((N, D.n_kv_heads, D.head_dim))
    dg = np.zeros((N, D.n_q_heads, D.n_gates))
    qb = None if qblocks is None else _c(qblocks, np.int32)
    n_qb = 0 if qb is None else len(qb)
    rc = fn(ctypes.byref(D), _p(off), _p(q), _p(k), _p(v), _p(gates), _p(idx), idx_heads, _p(dout), _p(dq),
            _p(dk), _p(dv), _p(dg), n_qb, _p(qb), int(nthreads))
    if rc != 0:
        raise ValueError("oracle backward: unsupported configuration")
    return dq, dk, dv, dg


def backward(D, off, q, k, v, gates, idx, dout, nthreads=1, qblocks=None):
    """(dq, dk, dv, dgates) of L = sum(O * dO) over all tokens, routing indices fixed.
    With qblocks only those query blocks contribute: dq and dgates of their rows are exact,
    dk and dv are the listed blocks' share, other rows of dq and dgates stay zero."""
    return _backward(_L().oracle_backward, np.uint16, D, off, q, k, v, gates, idx, dout, nthreads, qblocks)


def backward_f64(D, off, q, k, v, gates, idx, dout, nthreads=1, qblocks=None):
    return _backward(_L().oracle_backward_f64, np.float64, D, off, q, k, v, gates, idx, dout, nthreads, qblocks)


def loss_f64(D, off, q, k, v, gates, idx, dout) -> float:
    off = _c(off, np.int32)
    q, k, v, gates, dout = _inputs(np.float64, q, k, v, gates, dout)
    idx = _c(idx, np.int32)
    idx_heads = 1 if idx.ndim == 2 else idx.shape[1]
    return float(_L().oracle_loss_f64(ctypes.byref(D), _p(off), _p(q), _p(k), _p(v), _p(gates), _p(idx),
                                      idx_heads, _p(dout)))


def default_scale(head_dim: int) -> float:
    return 1.0 / math.sqrt(head_dim)


def _backward_pooled(fn, dtype, D, off, q, k, v, gates, idx, forced, dout, nthreads):
    off = _c(off, np.int32)
    q, k, v, gates, dout = _inputs(dtype, q, k, v, gates, dout)
    idx = _c(idx, np.int32)
    forced = np.zeros(0, np.int32) if forced is None else _c(forced, np.int32)
    N = D.n_tokens
    dq = np.zeros((N, D.n_q_heads, D.head_dim))
    dk = np.zeros((N, D.n_kv_heads, D.head_dim))
    dv = np.zeros((N, D.n_kv_heads, D.head_dim))
    dg = np.zeros((N, D.n_q_heads, D.n_gates))
    rc = fn(ctypes.byref(D), _p(off), _p(q), _p(k), _p(v), _p(gates), _p(idx), len(forced), _p(forced), _p(dout),
            _p(dq), _p(dk), _p(dv), _p(dg), int(nthreads))
    if rc != 0:
        raise ValueError("oracle pooled backward: unsupported configuration")
    return dq, dk, dv, dg


def backward_pooled(D, off, q, k, v, gates, idx, forced, dout, nthreads=1):
    """(dq, dk, dv, dgates) of L = sum(O * dO) for the Speed3R pooled-query layer (MHA, gates
    (cmp, slc)); idx [B][H][k] routing indices fixed, forced blocks joined to every selected set."""
    return _backward_pooled(_L().oracle_backward_pooled, np.uint16, D, off, q, k, v, gates, idx, forced, dout,
                            nthreads)


def backward_pooled_f64(D, off, q, k, v, gates, idx, forced, dout, nthreads=1):
    return _backward_pooled(_L().oracle_backward_pooled_f64, np.float64, D, off, q, k, v, gates, idx, forced, dout,
                            nthreads)


def loss_forced_f64(D, off, q, k, v, gates, idx, dout, forced) -> float:
    """L = sum(O * dO) with forced blocks joined to every selected set (pooled-query layer)."""
    off = _c(off, np.int32)
    q, k, v, gates, dout = _inputs(np.float64, q, k, v, gates, dout)
    idx = _c(idx, np.int32)
    idx_heads = 1 if idx.ndim == 2 else idx.shape[1]
    forced = _c(forced, np.int32)
    return float(_L().oracle_loss_forced_f64(ctypes.byref(D), _p(off), _p(q), _p(k), _p(v), _p(gates), _p(idx),
                                             idx_heads, _p(dout), len(forced), _p(forced)))


def mixture(D: OracleDesc, off, q, k, v, gates, bx: int, qblocks=None, want_branches=False):
    """Decoupled self/cross gated mixture (LSRM page, 方法, gated cross-attention equations):
    stream x = blocks [0, bx), stream y = blocks [bx, B); gates [N][Hq][2] = (w_self, w_cross).
    With want_branches: (out, branches [rows][Hq][2][d] = (self, cross), lse [rows][Hq][2])."""
    qblocks = np.arange(D.n_blocks, dtype=np.int32) if qblocks is None else _c(qblocks, np.int32)
    off = _c(off, np.int32)
    q, k, v, gates = _inputs(np.uint16, q, k, v, gates)
    rows = rows_of(off, qblocks)
    out = np.zeros((rows, D.n_q_heads, D.head_dim))
    br = np.zeros((rows, D.n_q_heads, 2, D.head_dim)) if want_branches else None
    lse = np.zeros((rows, D.n_q_heads, 2)) if want_branches else None
    rc = _L().oracle_mixture(ctypes.byref(D), _p(off), _p(q), _p(k), _p(v), _p(gates), int(bx), len(qblocks),
                             _p(qblocks), _p(out), _p(br), _p(lse))
    if rc != 0:
        raise ValueError("oracle_mixture: stream split outside [0, n_blocks]")
    return (out, br, lse) if want_branches else out


def route_camera(D: OracleDesc, off, coords, n_vol: int, proj, tile_block, tile_px: int, radius: int, k_vol: int,
                 k_img: int) -> np.ndarray:
    """Camera-projection routing (LSRM page, 方法, 3D-aware routing paragraph): idx [B][k_vol + k_img],
    the k_vol nearest volume blocks by centroid distance, then the k_img image blocks of the
    projected tile neighbourhoods nearest by their closest token.  proj int32 [V][3][4],
    tile_block int32 [V][tiles_y][tiles_x] (-1 = no block)."""
    off = _c(off, np.int32)
    coords = _c(coords, np.int32)
    proj = _c(proj, np.int32)
    tile_block = _c(tile_block, np.int32)
    V, ty, tx = tile_block.shape
    assert proj.shape == (V, 3, 4)
    idx = np.zeros((D.n_blocks, k_vol + k_img), dtype=np.int32)
    rc = _L().oracle_route_camera(ctypes.byref(D), _p(off), _p(coords), int(n_vol), int(V), _p(proj), int(tx),
                                  int(ty), int(tile_px), _p(tile_block), int(radius), int(k_vol), int(k_img),
                                  _p(idx))
    if rc != 0:
        raise ValueError("oracle_route_camera: k_vol / k_img above the block counts, or bad tile size / radius")
    return idx
