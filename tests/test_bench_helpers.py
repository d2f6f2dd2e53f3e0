"""The FLOP counts bench.py divides by (host logic, no GPU): every (query, key) pair the method
attends is counted once, 4 d FLOPs each for a forward."""
import numpy as np

import bench
from workloads import make_workload


def test_mixture_flops_count_every_pair_of_both_streams():
    w = make_workload("mixture_small")
    f = bench.mixture_flops(w)
    nx = int(w.off[w.n_blocks_x])
    ny = w.n_tokens - nx
    per_pair = 4 * w.head_dim * w.n_q_heads
    # brute force over token pairs: own stream (self) and the other stream (cross)
    stream = np.arange(w.n_tokens) >= nx
    same = (stream[:, None] == stream[None, :]).sum()
    assert f["self"] == per_pair * same == per_pair * (nx * nx + ny * ny)
    assert f["cross"] == per_pair * (w.n_tokens * w.n_tokens - same)
    assert f["total"] == f["self"] + f["cross"]


def test_algorithmic_flops_use_the_routed_blocks_actual_lengths():
    w = make_workload("ragged_geo")
    k = 3
    rng = np.random.default_rng(0)
    idx = np.stack([rng.choice(w.n_blocks, size=k, replace=False) for _ in range(w.n_blocks)]).astype(np.int32)
    f = bench.algorithmic_flops(w, idx)
    n = np.diff(w.off.astype(np.int64))
    slc_pairs = sum(int(n[a]) * int(n[idx[a]].sum()) for a in range(w.n_blocks)) * w.n_q_heads
    assert f["slc"] == 4 * w.head_dim * slc_pairs
    assert f["cmp"] == 4 * w.head_dim * w.n_tokens * w.n_q_heads * w.n_blocks
