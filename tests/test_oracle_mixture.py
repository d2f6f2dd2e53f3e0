"""Pins of the oracle's decoupled self/cross gated mixture (LSRM page, 方法: the dense blocks'
gated cross-attention equations) against things other than itself:

* each of its two attentions equals torch's scaled-dot-product attention (a library routine, in
  fp64) of the stream's queries over the own / the other stream's keys;
* one-hot gates (1, 0) and (0, 1) give exactly those two attentions, so the gate order is
  (self, cross);
* the two partial softmaxes recombined by their LSEs equal self-attention over the whole
  concatenated sequence, and their log-sum-exp equals the full row's;
* an empty stream contributes a zero output with LSE -inf.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from workloads import make_workload
from workloads.nsa_workloads import bf16_bits_to_f32, f32_to_bf16_bits


def _f64(bits):
    return torch.from_numpy(bf16_bits_to_f32(bits).astype(np.float64))


def _sdpa(q, k, v, G):
    """q [n, Hq, d] over keys k/v [m, Hkv, d] (head h reads group h // G), fp64."""
    kx = k.repeat_interleave(G, dim=1)
    vx = v.repeat_interleave(G, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(q.transpose(0, 1), kx.transpose(0, 1), vx.transpose(0, 1))
    return o.transpose(0, 1)


def _lse(q, k, G, tau):
    kx = k.repeat_interleave(G, dim=1)
    s = torch.einsum("nhd,mhd->hnm", q, kx) * tau
    return torch.logsumexp(s, dim=-1).transpose(0, 1)


def _desc(w):
    return O.desc_for(w.n_tokens, w.n_blocks, w.n_q_heads, w.n_kv_heads, w.head_dim, 1, 0, n_gates=2)


@pytest.mark.parametrize("name", ["mixture_small", "mixture_ragged"])
def test_mixture_branches_equal_library_attention(name):
    w = make_workload(name)
    D = _desc(w)
    bx, nx, N = w.n_blocks_x, int(w.off[w.n_blocks_x]), w.n_tokens
    G = w.n_q_heads // w.n_kv_heads
    out, br, lse = O.mixture(D, w.off, w.q, w.k, w.v, w.gates, bx, want_branches=True)
    q, k, v = _f64(w.q), _f64(w.k), _f64(w.v)
    x, y = slice(0, nx), slice(nx, N)
    ref_self = torch.cat([_sdpa(q[x], k[x], v[x], G), _sdpa(q[y], k[y], v[y], G)])
    ref_cross = torch.cat([_sdpa(q[x], k[y], v[y], G), _sdpa(q[y], k[x], v[x], G)])
    np.testing.assert_allclose(br[:, :, 0], ref_self.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(br[:, :, 1], ref_cross.numpy(), rtol=0, atol=1e-12)
    # recombined by their LSEs, the two partial softmaxes are attention over the whole sequence
    full = _sdpa(q, k, v, G).numpy()
    tot = np.logaddexp(lse[..., 0], lse[..., 1])
    mix = np.exp(lse[..., 0] - tot)[..., None] * br[:, :, 0] + np.exp(lse[..., 1] - tot)[..., None] * br[:, :, 1]
    np.testing.assert_allclose(mix, full, rtol=0, atol=1e-12)
    np.testing.assert_allclose(tot, _lse(q, k, G, 1.0 / np.sqrt(w.head_dim)).numpy(), rtol=0, atol=1e-10)
    # the gated sum with the workload's gates
    g = bf16_bits_to_f32(w.gates).astype(np.float64)
    np.testing.assert_allclose(out, g[..., 0:1] * br[:, :, 0] + g[..., 1:2] * br[:, :, 1], rtol=0, atol=1e-12)


def test_mixture_one_hot_gates_select_self_then_cross():
    w = make_workload("mixture_small")
    D = _desc(w)
    nx, N = int(w.off[w.n_blocks_x]), w.n_tokens
    G = w.n_q_heads // w.n_kv_heads
    q, k, v = _f64(w.q), _f64(w.k), _f64(w.v)
    x, y = slice(0, nx), slice(nx, N)
    for onehot, ref in (((1.0, 0.0), torch.cat([_sdpa(q[x], k[x], v[x], G), _sdpa(q[y], k[y], v[y], G)])),
                        ((0.0, 1.0), torch.cat([_sdpa(q[x], k[y], v[y], G), _sdpa(q[y], k[x], v[x], G)]))):
        gates = np.empty_like(w.gates)
        gates[...] = f32_to_bf16_bits(np.array(onehot, dtype=np.float32))
        out = O.mixture(D, w.off, w.q, w.k, w.v, gates, w.n_blocks_x)
        np.testing.assert_allclose(out, ref.numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("bx_of", [lambda w: w.n_blocks, lambda w: 0])
def test_mixture_with_an_empty_stream(bx_of):
    w = make_workload("mixture_small")
    D = _desc(w)
    G = w.n_q_heads // w.n_kv_heads
    bx = bx_of(w)
    out, br, lse = O.mixture(D, w.off, w.q, w.k, w.v, w.gates, bx, want_branches=True)
    q, k, v = _f64(w.q), _f64(w.k), _f64(w.v)
    np.testing.assert_allclose(br[:, :, 0], _sdpa(q, k, v, G).numpy(), rtol=0, atol=1e-12)
    assert np.all(br[:, :, 1] == 0.0) and np.all(np.isneginf(lse[..., 1]))
    with pytest.raises(ValueError):
        O.mixture(D, w.off, w.q, w.k, w.v, w.gates, w.n_blocks + 1)
