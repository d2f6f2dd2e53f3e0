"""Finite-difference pin of the oracle backward on the 1024-token subset of the sparse-stage
layer: the first 16 blocks (1024 tokens) of the sparse-stage generator, 32 query heads on 2 KV
heads, d = 32, every block selected (k = 16 = all), window 64, indices fixed.  For 256 seeded
coordinates of each of q, k, v and the gates, the central difference (L(x + h) - L(x - h)) / 2h
of L = sum(out * dO) must match the oracle's analytic gradient to 1e-7 (relative above 1).

Step sizes: h = 1e-6 where the loss is one output row (q, gates).  A key or value entry moves a
loss of 16384 rows x 32 products whose rounding differs between the two evaluations by ~1e-12
(measured: the central difference of one dK entry is off by 1.2e-6 at h = 1e-6 and 1e-7 alike,
1.4e-8 at h = 1e-5, 5e-9 at h = 1e-4, 5e-10 at h = 1e-3, so the error there is rounding, not
truncation); those take h = 1e-4, where truncation (h^2 / 6 times the third derivative) and
rounding both stay far below the bound.

The loss is evaluated only where the perturbed coordinate can move it, which keeps the test to a
couple of minutes on the host cores: a query or gate entry of (token t, head h) changes that one
output row, so the row is recomputed from its query block alone; a key or value entry of KV head g
changes the outputs of g's query heads only, and the layer splits by KV head, so g's sub-layer
(16 query heads on one KV head) is recomputed whole.  Loss evaluations run in parallel host
threads (the oracle's C calls release the interpreter lock)."""
from concurrent.futures import ThreadPoolExecutor
import os

import numpy as np
import pytest

import oracle as O
from workloads import make_workload
from workloads.nsa_workloads import bf16_bits_to_f32

pytestmark = pytest.mark.slow

NB = 16
H_ROW, H_GROUP = 1e-6, 1e-4
N_COORDS = 256


def _instance():
    w = make_workload("backward")
    off = np.ascontiguousarray(w.off[:NB + 1].astype(np.int32))
    n = int(off[-1])
    assert n == 1024 and np.all(np.diff(off) == 64)
    f = lambda a: np.ascontiguousarray(bf16_bits_to_f32(a[:n]).astype(np.float64))
    q, k, v, g, do = f(w.q), f(w.k), f(w.v), f(w.gates), f(w.dout)
    D = O.desc_for(n, NB, w.n_q_heads, w.n_kv_heads, w.head_dim, NB, w.window)
    idx = np.ascontiguousarray(np.tile(np.arange(NB, dtype=np.int32), (NB, 1)))
    return D, off, q, k, v, g, do, idx


def test_backward_matches_central_differences_on_the_1024_token_subset():
    D, off, q, k, v, g, do, idx = _instance()
    dq, dk, dv, dg = O.backward_f64(D, off, q, k, v, g, idx, do, nthreads=os.cpu_count() or 1)
    Hq, Hkv = D.n_q_heads, D.n_kv_heads
    G = Hq // Hkv
    rng = np.random.default_rng(20260)

    def row_loss(t, hq, qx, gx):
        # the output row (t, hq) from its query block alone, dotted with its upstream gradient
        b = int(np.searchsorted(off, t, side="right") - 1)
        out = O.forward_f64(D, off, qx, k, v, gx, idx, qblocks=np.array([b], np.int32))
        return float(out[t - off[b], hq] @ do[t, hq])

    def group_loss(grp, kx, vx):
        # KV head grp's sub-layer: its G query heads against KV head grp only
        hs = slice(grp * G, (grp + 1) * G)
        Dg = O.desc_for(D.n_tokens, D.n_blocks, G, 1, D.head_dim, D.top_k, D.window)
        return O.loss_f64(Dg, off, q[:, hs], kx[:, grp:grp + 1], vx[:, grp:grp + 1], g[:, hs], idx, do[:, hs])

    def fd(name, i):
        x = {"q": q, "g": g, "k": k, "v": v}[name]
        h = H_ROW if name in ("q", "g") else H_GROUP
        xp, xm = x.copy(), x.copy()
        xp[i] += h
        xm[i] -= h
        if name in ("q", "g"):
            t, hq = int(i[0]), int(i[1])
            lp = row_loss(t, hq, xp if name == "q" else q, xp if name == "g" else g)
            lm = row_loss(t, hq, xm if name == "q" else q, xm if name == "g" else g)
        else:
            grp = int(i[1])
            lp = group_loss(grp, xp if name == "k" else k, xp if name == "v" else v)
            lm = group_loss(grp, xm if name == "k" else k, xm if name == "v" else v)
        return (lp - lm) / (2 * h)

    jobs = []
    for name, x, grad in (("q", q, dq), ("g", g, dg), ("k", k, dk), ("v", v, dv)):
        coords = {tuple(int(rng.integers(0, s)) for s in x.shape) for _ in range(4 * N_COORDS)}
        coords = sorted(coords)[:N_COORDS]
        rng.shuffle(coords)
        assert len(coords) == N_COORDS
        jobs += [(name, c, grad[c]) for c in coords]
    with ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as pool:
        got = list(pool.map(lambda j: fd(j[0], j[1]), jobs))
    worst = {}
    for (name, c, ref), val in zip(jobs, got):
        err = abs(val - ref)
        assert err <= 1e-7 * max(1.0, abs(ref)), (name, c, val, ref)
        worst[name] = max(worst.get(name, 0.0), err)
    # the pin would be vacuous on an all-zero gradient: each tensor's sampled entries carry signal
    for name, grad in (("q", dq), ("g", dg), ("k", dk), ("v", dv)):
        sampled = np.array([ref for (n, _, ref) in jobs if n == name])
        assert np.abs(sampled).max() > 1e-3, name
