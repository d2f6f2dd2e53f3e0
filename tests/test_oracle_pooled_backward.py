"""Pins of the oracle's backward of the Speed3R pooled-query layer (Speed3R page, 2.1: pooled
compression branch, selection over forced + routed blocks, gated aggregation; the model trains
end to end).  Three independent checks:
  * central finite differences of L = sum(out * dO) at every input of a small ragged case;
  * with every non-forced block routed, g_cmp = 0 and g_slc = 1 the layer is dense MHA, so the
    gradients equal torch autograd through a plain fp64 softmax attention;
  * with g_slc = 0 only the pooled branch remains: the query gradient is the pooled query's
    gradient shared equally by the block's tokens, and every token of a block gets the same key
    and value gradient (the block-mean backward)."""
import numpy as np
import pytest
import torch

import oracle as O
from workloads.nsa_workloads import normal_bf16, sigmoid_normal_bf16, bf16_bits_to_f32


def _f64(bits):
    return bf16_bits_to_f32(np.asarray(bits)).astype(np.float64)


def _case(seed=0, h=2, d=4, k=2):
    # blocks of a tiny two-frame sequence: a 1-token camera block first in each frame, then
    # ragged patch blocks; frame 0 and the camera blocks are forced
    sizes = [1, 4, 3, 2, 1, 4, 2, 3, 1]
    off = np.zeros(len(sizes) + 1, dtype=np.int32)
    off[1:] = np.cumsum(sizes)
    n, B = int(off[-1]), len(sizes)
    forced = np.array([0, 1, 2, 3, 4], dtype=np.int32)  # frame 0 (blocks 0-3) + the second camera
    q = _f64(normal_bf16(seed, 0, (n, h, d), 1.0))
    kk = _f64(normal_bf16(seed, 1, (n, h, d), 1.0))
    v = _f64(normal_bf16(seed, 2, (n, h, d), 1.0))
    g = _f64(sigmoid_normal_bf16(seed, 3, (n, h, 2)))
    dout = np.random.default_rng(seed + 11).standard_normal((n, h, d))
    D = O.desc_for(n, B, h, h, d, k, 0, n_gates=2, pooled_q=True)
    rng = np.random.default_rng(seed)
    nonf = np.setdiff1d(np.arange(B), forced)
    idx = np.stack([np.stack([rng.choice(nonf, k, replace=False) for _ in range(h)]) for _ in range(B)])
    return D, off, q, kk, v, g, dout, idx.astype(np.int32), forced


def test_pooled_backward_matches_central_differences():
    D, off, q, k, v, g, dout, idx, forced = _case()
    dq, dk, dv, dg = O.backward_pooled_f64(D, off, q, k, v, g, idx, forced, dout)
    hstep = 1e-6
    args = {"q": q, "k": k, "v": v, "g": g}
    grads = {"q": dq, "k": dk, "v": dv, "g": dg}
    for name, x in args.items():
        for i in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[i] += hstep
            xm[i] -= hstep
            ap, am = dict(args, **{name: xp}), dict(args, **{name: xm})
            lp = O.loss_forced_f64(D, off, ap["q"], ap["k"], ap["v"], ap["g"], idx, dout, forced)
            lm = O.loss_forced_f64(D, off, am["q"], am["k"], am["v"], am["g"], idx, dout, forced)
            fd = (lp - lm) / (2 * hstep)
            assert abs(fd - grads[name][i]) < 1e-7 * max(1.0, abs(fd)), (name, i, fd, grads[name][i])
    for name in grads:
        assert np.abs(grads[name]).max() > 1e-3, name


def test_pooled_backward_with_every_block_selected_is_dense_mha_autograd():
    D, off, q, k, v, g, dout, _, forced = _case(seed=4)
    B, h = D.n_blocks, D.n_q_heads
    nonf = np.setdiff1d(np.arange(B), forced).astype(np.int32)
    D = O.desc_for(D.n_tokens, B, h, h, D.head_dim, len(nonf), 0, n_gates=2, pooled_q=True)
    idx = np.tile(nonf, (B, h, 1)).astype(np.int32)
    g = np.zeros_like(g)
    g[..., 1] = 1.0
    dq, dk, dv, dg = O.backward_pooled_f64(D, off, q, k, v, g, idx, forced, dout)
    qt, kt, vt = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    s = torch.einsum("thc,uhc->htu", qt, kt) / np.sqrt(D.head_dim)
    o = torch.einsum("htu,uhc->thc", torch.softmax(s, dim=-1), vt)
    (o * torch.tensor(dout)).sum().backward()
    for got, ref in ((dq, qt.grad), (dk, kt.grad), (dv, vt.grad)):
        assert np.abs(got - ref.numpy()).max() < 1e-12
    # the gate of the selected branch sees <dO, o>
    assert np.abs(dg[..., 1] - np.einsum("thc,thc->th", dout, o.detach().numpy())).max() < 1e-12


def test_pooled_backward_compressed_only_shares_the_pooled_gradient():
    D, off, q, k, v, g, dout, idx, forced = _case(seed=2)
    g = g.copy()
    g[..., 1] = 0.0
    dq, dk, dv, dg = O.backward_pooled_f64(D, off, q, k, v, g, idx, forced, dout)
    for b in range(D.n_blocks):
        blk = slice(off[b], off[b + 1])
        for x in (dq, dk, dv):
            assert np.abs(x[blk] - x[off[b]][None]).max() < 1e-15
    # the same gradients from torch autograd through block means, the pooled softmax attention and
    # the copy of each block's output to its tokens
    seg = torch.tensor(np.repeat(np.arange(D.n_blocks), np.diff(off)))
    cnt = torch.tensor(np.diff(off), dtype=torch.float64)[:, None, None]

    def pool(x):
        return torch.zeros((D.n_blocks,) + x.shape[1:], dtype=torch.float64).index_add(0, seg, x) / cnt

    qt, kt, vt = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    qb, kb, vb = pool(qt), pool(kt), pool(vt)
    s = torch.einsum("ahc,jhc->haj", qb, kb) / np.sqrt(D.head_dim)
    ob = torch.einsum("haj,jhc->ahc", torch.softmax(s, dim=-1), vb)
    out = torch.tensor(g[..., :1]) * ob[seg]
    (out * torch.tensor(dout)).sum().backward()
    for got, ref in ((dq, qt.grad), (dk, kt.grad), (dv, vt.grad)):
        assert np.abs(got - ref.numpy()).max() < 1e-12
    assert np.abs(dg[..., 0] - np.einsum("thc,thc->th", dout, ob[seg].detach().numpy())).max() < 1e-12


def test_pooled_backward_threads_agree():
    D, off, q, k, v, g, dout, idx, forced = _case(seed=3)
    a = O.backward_pooled_f64(D, off, q, k, v, g, idx, forced, dout, nthreads=1)
    b = O.backward_pooled_f64(D, off, q, k, v, g, idx, forced, dout, nthreads=3)
    for x, y in zip(a, b):
        assert np.abs(x - y).max() < 1e-13 * max(1.0, np.abs(x).max())
