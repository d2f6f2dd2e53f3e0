"""Thin Python binding of liblsrm_nsa.so (the C ABI declared in include/lsrm_nsa.h).

Argument marshalling only: every function has the name of the C entry point it
calls, takes torch tensors that already live on the GPU (or None), passes their
device pointers and the current CUDA stream, and raises NsaError when the call
returns a status other than LSRM_OK.  All computation happens in the CUDA
kernels behind the ABI; there is no CPU path.  Importing works anywhere, but the
first call loads the library and fails loudly if it has not been built or no
GPU is present.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblsrm_nsa.so")

LSRM_OK = 0
STATUS = {0: "LSRM_OK", 1: "LSRM_ERR_INVALID_ARG", 2: "LSRM_ERR_UNSUPPORTED", 3: "LSRM_ERR_CUDA",
          4: "LSRM_ERR_TIMEOUT", 5: "LSRM_ERR_BOUNDS", 6: "LSRM_ERR_WORKSPACE"}
ROUTE_GIVEN, ROUTE_SCORE, ROUTE_GEOMETRIC, ROUTE_ALL = 0, 1, 2, 3

# every symbol include/lsrm_nsa.h declares
EXPORTS = ("lsrm_nsa_workspace_size", "lsrm_nsa_workspace_init", "lsrm_nsa_compress", "lsrm_route_score_topk",
           "lsrm_route_geometric", "lsrm_route_geometric_noalloc", "lsrm_route_camera", "lsrm_route_pooled_topk", "lsrm_nsa_cmp_attn", "lsrm_nsa_select_attn",
           "lsrm_nsa_window_attn", "lsrm_nsa_gate_combine", "lsrm_nsa_attend", "lsrm_nsa_mixture", "lsrm_nsa_forward", "lsrm_nsa_backward",
           "lsrm_nsa_last_device_status", "lsrm_status_string", "lsrm_diag_exp2_poly")


class NsaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {STATUS.get(status, status)}")
        self.status = status


class Desc(ctypes.Structure):
    """lsrm_nsa_desc (host struct)."""
    _fields_ = [("n_tokens", ctypes.c_int64), ("n_blocks", ctypes.c_int32), ("max_block_len", ctypes.c_int32),
                ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("window", ctypes.c_int32), ("scale", ctypes.c_float),
                ("pooled_q", ctypes.c_int32), ("n_gates", ctypes.c_int32), ("n_forced", ctypes.c_int32),
                ("forced_blocks", ctypes.c_void_p)]


def make_desc(n_tokens, n_blocks, max_block_len, n_q_heads, n_kv_heads, head_dim, top_k, window, scale=0.0,
              pooled_q=False, n_gates=3, forced: Optional[torch.Tensor] = None) -> Desc:
    if forced is not None and forced.numel() > 0:
        _check(forced, torch.int32, "forced")
        nf, fp = forced.numel(), forced.data_ptr()
    else:
        nf, fp = 0, None
    return Desc(int(n_tokens), int(n_blocks), int(max_block_len), int(n_q_heads), int(n_kv_heads), int(head_dim),
                int(top_k), int(window), float(scale), int(bool(pooled_q)), int(n_gates), nf, fp)


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load liblsrm_nsa.so; raise if it is missing (no fallback exists)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is not built; run `python -m block_sparse_gqa_nsa_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    D = ctypes.POINTER(Desc)
    sigs = {
        "lsrm_nsa_workspace_size": ([D], sz),
        "lsrm_nsa_workspace_init": ([D, vp, sz, vp], ctypes.c_int),
        "lsrm_nsa_compress": ([D, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp], ctypes.c_int),
        "lsrm_route_score_topk": ([D, vp, vp, vp, vp, vp, vp, vp], ctypes.c_int),
        "lsrm_route_geometric": ([D, vp, vp, vp, vp, vp], ctypes.c_int),
        "lsrm_route_geometric_noalloc": ([D, vp, vp, vp, vp, vp], ctypes.c_int),
        "lsrm_route_pooled_topk": ([D, vp, vp, vp, vp, vp, vp, vp], ctypes.c_int),
        "lsrm_nsa_cmp_attn": ([D, vp, vp, vp, vp, vp, vp, vp, vp], ctypes.c_int),
        "lsrm_nsa_select_attn": ([D, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp], ctypes.c_int),
        "lsrm_nsa_window_attn": ([D, vp, vp, vp, vp, vp, vp, vp, vp], ctypes.c_int),
        "lsrm_nsa_gate_combine": ([D, vp, vp, vp, vp, vp, vp], ctypes.c_int),
        "lsrm_nsa_attend": ([D, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, vp, vp, vp, vp], ctypes.c_int),
        "lsrm_nsa_mixture": ([D, vp, i32, vp, vp, vp, vp, vp, vp, vp, vp], ctypes.c_int),
        "lsrm_route_camera": ([D, vp, vp, i32, i32, vp, i32, i32, i32, vp, i32, i32, vp, vp, vp], ctypes.c_int),
        "lsrm_nsa_forward": ([D, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp], ctypes.c_int),
        "lsrm_nsa_backward": ([D, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp], ctypes.c_int),
        "lsrm_nsa_last_device_status": ([vp, vp], ctypes.c_int),
        "lsrm_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "lsrm_diag_exp2_poly": ([vp, vp, ctypes.c_int64, vp], ctypes.c_int),
    }
    for name, (args, res) in sigs.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    _lib = lib
    return lib


def _check(t: Optional[torch.Tensor], dtype, name: str, cuda: bool = True):
    if t is None:
        return
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if cuda and not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _call(name: str, *args):
    rc = getattr(load_library(), name)(*args)
    if rc != LSRM_OK:
        raise NsaError(name, rc)


def lsrm_nsa_workspace_size(desc: Desc) -> int:
    return int(load_library().lsrm_nsa_workspace_size(ctypes.byref(desc)))


def workspace(desc: Desc, device=None, stream=None) -> torch.Tensor:
    """Allocate (through torch) and zero the workspace the calls of this descriptor need."""
    n = lsrm_nsa_workspace_size(desc)
    if n == 0:
        raise NsaError("lsrm_nsa_workspace_size", 1)
    ws = torch.empty(n, dtype=torch.uint8, device=device or "cuda")
    lsrm_nsa_workspace_init(desc, ws, stream)
    return ws


def lsrm_nsa_workspace_init(desc: Desc, ws: torch.Tensor, stream=None):
    _check(ws, torch.uint8, "ws")
    _call("lsrm_nsa_workspace_init", ctypes.byref(desc), ws.data_ptr(), ws.numel(), _stream(stream))


def lsrm_nsa_compress(desc, off, q, k, v, kc32=None, kc=None, vc32=None, vc=None, qc32=None, qc=None, ws=None,
                      stream=None):
    for t, n, dt in ((off, "off", torch.int32), (q, "q", torch.bfloat16), (k, "k", torch.bfloat16),
                     (v, "v", torch.bfloat16), (kc32, "kc32", torch.float32), (kc, "kc", torch.bfloat16),
                     (vc32, "vc32", torch.float32), (vc, "vc", torch.bfloat16), (qc32, "qc32", torch.float32),
                     (qc, "qc", torch.bfloat16)):
        _check(t, dt, n)
    _call("lsrm_nsa_compress", ctypes.byref(desc), _ptr(off), _ptr(q), _ptr(k), _ptr(v), _ptr(kc32), _ptr(kc),
          _ptr(vc32), _ptr(vc), _ptr(qc32), _ptr(qc), _ptr(ws), _stream(stream))


def lsrm_route_score_topk(desc, off, q, kc32, idx, score=None, ws=None, stream=None):
    _check(off, torch.int32, "off"); _check(q, torch.bfloat16, "q"); _check(kc32, torch.float32, "kc32")
    _check(idx, torch.int32, "idx"); _check(score, torch.float32, "score")
    _call("lsrm_route_score_topk", ctypes.byref(desc), _ptr(off), _ptr(q), _ptr(kc32), _ptr(idx), _ptr(score),
          _ptr(ws), _stream(stream))


def lsrm_route_geometric(desc, off, coords, idx, ws, stream=None):
    _check(off, torch.int32, "off"); _check(coords, torch.int32, "coords"); _check(idx, torch.int32, "idx")
    _call("lsrm_route_geometric", ctypes.byref(desc), _ptr(off), _ptr(coords), _ptr(idx), _ptr(ws),
          _stream(stream))


def lsrm_route_geometric_noalloc(desc, off, coords, idx, status=None, stream=None):
    """Geometric routing without a workspace, for callers that cannot allocate device memory
    (its scratch is a fixed array inside the library; at most 16384 blocks; calls that
    overlap on the GPU race).  `status` is an optional one-element device tensor that receives
    the bounds bit.  The C entry point declares it uint32_t*; torch has no unsigned 32-bit
    tensor type, so it is passed as torch.int32, which has the same size and layout (the bit
    LSRM_ERR_BOUNDS sets, 1 << 4, reads the same in either type)."""
    _check(off, torch.int32, "off"); _check(coords, torch.int32, "coords"); _check(idx, torch.int32, "idx")
    _check(status, torch.int32, "status")
    _call("lsrm_route_geometric_noalloc", ctypes.byref(desc), _ptr(off), _ptr(coords), _ptr(idx), _ptr(status),
          _stream(stream))


def lsrm_route_pooled_topk(desc, qc, kc, idx, ws, stream=None, qc32=None, kc32=None):
    """Speed3R routing from the bf16 pooled tensors; with the fp32 means qc32 / kc32 the ranking is
    that of the fp32 means (the exact mode)."""
    _check(qc, torch.bfloat16, "qc"); _check(kc, torch.bfloat16, "kc"); _check(idx, torch.int32, "idx")
    _check(qc32, torch.float32, "qc32"); _check(kc32, torch.float32, "kc32")
    _call("lsrm_route_pooled_topk", ctypes.byref(desc), _ptr(qc), _ptr(kc), _ptr(qc32), _ptr(kc32), _ptr(idx),
          _ptr(ws), _stream(stream))


def lsrm_nsa_cmp_attn(desc, off, q, kc, vc, o_cmp, lse=None, ws=None, stream=None):
    _check(off, torch.int32, "off"); _check(q, torch.bfloat16, "q"); _check(kc, torch.bfloat16, "kc")
    _check(vc, torch.bfloat16, "vc"); _check(o_cmp, torch.float32, "o_cmp"); _check(lse, torch.float32, "lse")
    _call("lsrm_nsa_cmp_attn", ctypes.byref(desc), _ptr(off), _ptr(q), _ptr(kc), _ptr(vc), _ptr(o_cmp), _ptr(lse),
          _ptr(ws), _stream(stream))


def lsrm_nsa_select_attn(desc, off, q, k, v, idx, idx_heads, o_slc, lse=None, ws=None, stream=None):
    for t, n, dt in ((off, "off", torch.int32), (q, "q", torch.bfloat16), (k, "k", torch.bfloat16),
                     (v, "v", torch.bfloat16), (idx, "idx", torch.int32), (o_slc, "o_slc", torch.float32),
                     (lse, "lse", torch.float32)):
        _check(t, dt, n)
    _call("lsrm_nsa_select_attn", ctypes.byref(desc), _ptr(off), _ptr(q), _ptr(k), _ptr(v), _ptr(idx),
          int(idx_heads), _ptr(o_slc), _ptr(lse), _ptr(ws), _stream(stream))


def lsrm_nsa_window_attn(desc, off, q, k, v, o_win, lse=None, ws=None, stream=None):
    for t, n, dt in ((off, "off", torch.int32), (q, "q", torch.bfloat16), (k, "k", torch.bfloat16),
                     (v, "v", torch.bfloat16), (o_win, "o_win", torch.float32), (lse, "lse", torch.float32)):
        _check(t, dt, n)
    _call("lsrm_nsa_window_attn", ctypes.byref(desc), _ptr(off), _ptr(q), _ptr(k), _ptr(v), _ptr(o_win),
          _ptr(lse), _ptr(ws), _stream(stream))


def lsrm_nsa_gate_combine(desc, o_cmp, o_slc, o_win, gates, out, stream=None):
    for t, n, dt in ((o_cmp, "o_cmp", torch.float32), (o_slc, "o_slc", torch.float32),
                     (o_win, "o_win", torch.float32), (gates, "gates", torch.bfloat16), (out, "out", torch.bfloat16)):
        _check(t, dt, n)
    _call("lsrm_nsa_gate_combine", ctypes.byref(desc), _ptr(o_cmp), _ptr(o_slc), _ptr(o_win), _ptr(gates),
          _ptr(out), _stream(stream))


def lsrm_nsa_attend(desc, off, q, k, v, kc, vc, gates, idx, idx_heads, route_all, out, lse=None, ws=None,
                    stream=None):
    for t, n, dt in ((off, "off", torch.int32), (q, "q", torch.bfloat16), (k, "k", torch.bfloat16),
                     (v, "v", torch.bfloat16), (kc, "kc", torch.bfloat16), (vc, "vc", torch.bfloat16),
                     (gates, "gates", torch.bfloat16), (idx, "idx", torch.int32), (out, "out", torch.bfloat16),
                     (lse, "lse", torch.float32)):
        _check(t, dt, n)
    _call("lsrm_nsa_attend", ctypes.byref(desc), _ptr(off), _ptr(q), _ptr(k), _ptr(v), _ptr(kc), _ptr(vc),
          _ptr(gates), _ptr(idx), int(idx_heads), int(route_all), _ptr(out), _ptr(lse), _ptr(ws), _stream(stream))


def lsrm_route_camera(desc, off, coords, n_vol_blocks, proj, tile_block, tile_px, radius, k_vol, idx, ws,
                      stream=None):
    """Camera-projection routing: proj int32 [V][3][4], tile_block int32 [V][tiles_y][tiles_x]
    (device); idx int32 [B][top_k] = k_vol volume blocks, then top_k - k_vol image blocks."""
    for t, n, dt in ((off, "off", torch.int32), (coords, "coords", torch.int32), (proj, "proj", torch.int32),
                     (tile_block, "tile_block", torch.int32), (idx, "idx", torch.int32)):
        _check(t, dt, n)
    V, ty, tx = tile_block.shape
    if tuple(proj.shape) != (V, 3, 4):
        raise ValueError("proj: expected [views][3][4]")
    _call("lsrm_route_camera", ctypes.byref(desc), _ptr(off), _ptr(coords), int(n_vol_blocks), int(V), _ptr(proj),
          int(tx), int(ty), int(tile_px), _ptr(tile_block), int(radius), int(k_vol), _ptr(idx), _ptr(ws),
          _stream(stream))


def lsrm_nsa_mixture(desc, off, n_blocks_x, q, k, v, gates, out, lse=None, ws=None, stream=None):
    """Self/cross gated mixture: blocks [0, n_blocks_x) are one stream, the rest the other;
    gates [N][Hq][2] = (self, cross); lse (optional) fp32 [N][Hq][2]."""
    for t, n, dt in ((off, "off", torch.int32), (q, "q", torch.bfloat16), (k, "k", torch.bfloat16),
                     (v, "v", torch.bfloat16), (gates, "gates", torch.bfloat16), (out, "out", torch.bfloat16),
                     (lse, "lse", torch.float32)):
        _check(t, dt, n)
    _call("lsrm_nsa_mixture", ctypes.byref(desc), _ptr(off), int(n_blocks_x), _ptr(q), _ptr(k), _ptr(v),
          _ptr(gates), _ptr(out), _ptr(lse), _ptr(ws), _stream(stream))


def lsrm_nsa_forward(desc, off, q, k, v, gates, coords, route_mode, out, idx=None, lse=None, ws=None, stream=None,
                     obr=None):
    """obr: optional bf16 [N][Hq][n_gates][d] that receives the per-branch outputs for the backward."""
    for t, n, dt in ((off, "off", torch.int32), (q, "q", torch.bfloat16), (k, "k", torch.bfloat16),
                     (v, "v", torch.bfloat16), (gates, "gates", torch.bfloat16), (coords, "coords", torch.int32),
                     (out, "out", torch.bfloat16), (idx, "idx", torch.int32), (lse, "lse", torch.float32),
                     (obr, "obr", torch.bfloat16)):
        _check(t, dt, n)
    _call("lsrm_nsa_forward", ctypes.byref(desc), _ptr(off), _ptr(q), _ptr(k), _ptr(v), _ptr(gates), _ptr(coords),
          int(route_mode), _ptr(out), _ptr(idx), _ptr(lse), _ptr(obr), _ptr(ws), _stream(stream))


def lsrm_nsa_backward(desc, off, q, k, v, gates, idx, idx_heads, lse, dout, dq, dk, dv, dgates, ws, stream=None,
                      obr=None):
    """obr: the forward's saved per-branch outputs (optional); with them each branch is streamed once."""
    for t, n, dt in ((off, "off", torch.int32), (q, "q", torch.bfloat16), (k, "k", torch.bfloat16),
                     (v, "v", torch.bfloat16), (gates, "gates", torch.bfloat16), (idx, "idx", torch.int32),
                     (lse, "lse", torch.float32), (dout, "dout", torch.bfloat16), (dq, "dq", torch.bfloat16),
                     (dk, "dk", torch.bfloat16), (dv, "dv", torch.bfloat16), (dgates, "dgates", torch.bfloat16),
                     (obr, "obr", torch.bfloat16)):
        _check(t, dt, n)
    _call("lsrm_nsa_backward", ctypes.byref(desc), _ptr(off), _ptr(q), _ptr(k), _ptr(v), _ptr(gates), _ptr(idx),
          int(idx_heads), _ptr(lse), _ptr(obr), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dgates), _ptr(ws),
          _stream(stream))


def lsrm_nsa_last_device_status(ws: torch.Tensor, stream=None) -> int:
    return int(load_library().lsrm_nsa_last_device_status(ws.data_ptr(), _stream(stream)))


def lsrm_status_string(status: int) -> str:
    return load_library().lsrm_status_string(int(status)).decode()


def default_scale(head_dim: int) -> float:
    return 1.0 / math.sqrt(head_dim)


def lsrm_diag_exp2_poly(x, y, stream=None):
    """y = 2^x through the attention kernels' FMA-pipe polynomial (a diagnostic)."""
    _check(x, torch.float32, "x"); _check(y, torch.float32, "y")
    if x.numel() != y.numel():
        raise ValueError("x and y differ in size")
    _call("lsrm_diag_exp2_poly", _ptr(x), _ptr(y), ctypes.c_int64(x.numel()), _stream(stream))
