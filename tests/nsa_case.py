"""Helpers shared by the GPU parity tests: move a seeded workload to the device,
build the ABI descriptor, and compare against the oracle with the stated bounds."""
import numpy as np
import torch

import oracle as O
from block_sparse_gqa_nsa_b200 import nsa

# acceptance bounds for attention outputs from bf16 inputs
MAX_ABS = 1e-2
REL_L2 = 5e-3
# score-routing gap rule: where the oracle's k-th and (k+1)-th scores differ by more than GAP the
# chosen sets must agree; otherwise every chosen block lies within GAP of the k-th score
GAP = 1e-3


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def i32(a, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


def oracle_desc(w, **kw):
    args = dict(n_tokens=w.n_tokens, n_blocks=w.n_blocks, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                head_dim=w.head_dim, top_k=w.top_k, window=w.window, n_gates=w.n_gates, pooled_q=w.pooled_q)
    args.update(kw)
    return O.desc_for(**args)


class DeviceCase:
    """A workload's tensors on the GPU plus its ABI descriptor and workspace."""

    def __init__(self, w, device="cuda", top_k=None):
        self.w = w
        self.off = i32(w.off, device)
        self.q = bf16_tensor(w.q, device)
        self.k = bf16_tensor(w.k, device)
        self.v = bf16_tensor(w.v, device)
        self.gates = bf16_tensor(w.gates, device)
        self.coords = i32(w.coords, device) if w.coords is not None else None
        self.forced = i32(w.forced, device) if len(w.forced) else None
        self.top_k = top_k if top_k is not None else w.top_k
        self.desc = nsa.make_desc(w.n_tokens, w.n_blocks, w.max_block_len, w.n_q_heads, w.n_kv_heads, w.head_dim,
                                  self.top_k, w.window, 0.0, w.pooled_q, w.n_gates, self.forced)
        self.ws = nsa.workspace(self.desc)

    def empty(self, *shape, dtype=torch.float32):
        return torch.empty(*shape, dtype=dtype, device=self.q.device)


def rel_l2(a, ref):
    a = np.asarray(a, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(a - ref) / max(np.linalg.norm(ref), 1e-300))


def assert_close(got, ref, what="", max_abs=MAX_ABS, rel=REL_L2):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = float(np.abs(got - ref).max())
    r = rel_l2(got, ref)
    assert err <= max_abs and r <= rel, f"{what}: max_abs {err:.3e} (<= {max_abs}), rel_l2 {r:.3e} (<= {rel})"
    return err, r


def rows_for(off, qblocks):
    return np.concatenate([np.arange(off[b], off[b + 1]) for b in qblocks])


def to_np(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy()
    return t.cpu().numpy()


def assert_grad_close(got, ref, what=""):
    """Gradient bounds: max-abs 1e-2 scaled by max(1, max|ref|), relative L2 5e-3."""
    ref = np.asarray(ref, dtype=np.float64)
    return assert_close(got, ref, what, max_abs=MAX_ABS * max(1.0, float(np.abs(ref).max())), rel=REL_L2)


def check_pooled_routing(gpu_idx, w, qblocks, k, qc=None, kc=None):
    """Validity of Speed3R routing against the oracle's fp64 pooled logits: k distinct, non-forced
    blocks, each with an oracle logit within 1e-3 of the k-th best; where the oracle gap exceeds
    1e-3 the sets must agree.  qc / kc default to the oracle's fp64 block means; a test of the
    bf16-operand mode passes the bf16 operands it gave the kernel."""
    D = oracle_desc(w, top_k=k)
    if qc is None:
        qc = O.compress(D, w.off, w.q, w.n_q_heads)
    if kc is None:
        kc = O.compress(D, w.off, w.k, w.n_kv_heads)
    _, logits = O.route_pooled(D, qc, kc, w.forced, qblocks=qblocks, want_logits=True)
    forced = set(w.forced.tolist())
    for i, a in enumerate(qblocks):
        for h in range(w.n_q_heads):
            chosen = gpu_idx[a, h].tolist()
            assert len(set(chosen)) == k and not (set(chosen) & forced), (a, h)
            lg = logits[i, h].copy()
            lg[list(forced)] = -np.inf
            order = np.lexsort((np.arange(w.n_blocks), -lg))
            sk = lg[order[k - 1]]
            assert np.all(lg[chosen] >= sk - GAP), (a, h)
            if k < len(order) and sk - lg[order[k]] > GAP:
                assert set(chosen) == set(order[:k].tolist()), (a, h)
