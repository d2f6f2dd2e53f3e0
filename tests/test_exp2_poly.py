"""The FMA-pipe 2^x of the attention kernels (poly_exp2_pair): its coefficients are the Remez
fit that block_sparse_gqa_nsa_b200/exp2_fit.py computes (checked bit for bit on the CPU), and
on the GPU its values stay within that fit's relative error of CUDA's exp2f over the whole
range the kernels use."""
import os
import re

import numpy as np
import pytest

from block_sparse_gqa_nsa_b200.exp2_fit import remez_exp2, float32_coefficients

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _kernel_coefficients():
    src = open(os.path.join(ROOT, "block_sparse_gqa_nsa_b200", "csrc", "tc_ptx.cuh")).read()
    body = src[src.index("void poly_exp2_pair"):]
    body = body[:body.index("\n}\n")]
    lits = re.findall(r"\"f\"\(([0-9.eE+-]+)f\)", body)
    # the magic constant 1.5 * 2^23 first, then c3, c2, c1, c0 in Horner order
    vals = [np.float32(float(x)) for x in lits]
    assert vals[0] == np.float32(12582912.0)
    return vals[1:][::-1]  # c0..c3


def test_fit_levels_the_relative_error():
    coef, lev, mx = remez_exp2()
    # equioscillation: the max error on a fine grid equals the levelled error
    assert abs(mx - lev) < 1e-9
    assert 7.0e-5 < lev < 7.6e-5
    # 2^f itself at the ends and the middle
    for f in (-0.5, 0.0, 0.5):
        p = sum(c * f ** i for i, c in enumerate(coef))
        assert abs(p / 2.0 ** f - 1) <= lev * (1 + 1e-9)


def test_kernel_literals_are_the_fit_bit_for_bit():
    got = _kernel_coefficients()
    want = float32_coefficients()
    assert len(got) == 4
    for g, w in zip(got, want):
        assert np.float32(g).view(np.uint32) == np.float32(w).view(np.uint32), (g, w)


@pytest.mark.gpu
def test_device_polynomial_against_exp2f():
    import torch
    from block_sparse_gqa_nsa_b200 import nsa
    from block_sparse_gqa_nsa_b200.build import build
    build()
    nsa.load_library()
    _, lev, _ = remez_exp2()
    # a dense grid over the kernels' range, plus the clamp edge and points either side of the
    # half-integers where round(x) switches
    grid = np.linspace(-125.0, 127.0, 2_000_001, dtype=np.float64)
    half = np.arange(-125, 127) + 0.5
    edges = np.concatenate([half, np.nextafter(half, -np.inf), np.nextafter(half, np.inf),
                            [-125.0, -124.999, 126.999, 127.0, 0.0, -0.0]])
    x = torch.tensor(np.concatenate([grid, edges]).astype(np.float32), device="cuda")
    y = torch.empty_like(x)
    nsa.lsrm_diag_exp2_poly(x, y)
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref) / ref).abs()
    assert torch.isfinite(y).all() and (y > 0).all()
    # the fit's error plus a few float32 roundings of the Horner steps
    assert float(rel.max()) <= lev + 4e-7, float(rel.max())
    # below the clamp the result is tiny and positive, never garbage
    lo = torch.tensor([-126.0, -200.0, -1e30, float("-inf")], device="cuda")
    ylo = torch.empty_like(lo)
    nsa.lsrm_diag_exp2_poly(lo, ylo)
    assert (ylo > 0).all() and (ylo < 2.0 ** -124).all()
