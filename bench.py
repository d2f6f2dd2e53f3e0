#!/usr/bin/env python3
"""Benchmark of the LSRM native-sparse-attention layer forward on B200.

Workload: the LSRM sparse stage with 3D-aware geometric routing — 1384 volume
bricks on the 0.35-0.45 shell of a 64^3 grid + 16 views of 64x64 image tokens
with 32 of 64 tiles kept (121344 tokens, 1896 blocks of 64), GQA 32/2, d 32,
geometric top-16, window 64, seeded synthetic bf16 inputs.

One step = one pass of the whole hot path through the C ABI: block mean-pool
(lsrm_nsa_compress), geometric routing (lsrm_route_geometric), and the fused
three-branch attention with the gated combine in its epilogue (lsrm_nsa_attend).
`value` is tokens/s over all ranks with inputs already in HBM; `e2e` is the same
metric through lsrm_nsa_forward with pinned host buffers, host<->device copies
inside the timed region.  `--impl reference` times the fp64 CPU oracle instead
(a bounded sample of query blocks per step, on the host cores).

Multi-GPU: the layer does not shard on one GPU's worth of work here (one
instance per GPU), so N ranks run N independent replicas ("scaling": "weak");
the only collectives are the timing barrier and a max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse-attn fwd tokens/s and effective TFLOP/s vs B200 bf16 tensor peak"
WORKLOAD = "lsrm_sparse_stage_geometric_top16"
L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-sample-blocks", type=int, default=None,
                    help="query blocks of the oracle's bounded CPU sample (default 64 forward, 24 backward: "
                         "10-20 s of one core)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--workload", default="sparse", choices=["sparse", "backward", "dense", "tiny", "speed3r", "speed3r_backward", "mixture", "bandwidth"],
                    help="sparse: the layer forward (the default line); backward: its gradients; dense: the "
                         "dense-stage shape with every block selected; speed3r: the pooled-query variant; "
                         "bandwidth: achieved HBM GB/s of the memory-bound kernels (pooling, routing, combine)")
    ap.add_argument("--record-traffic", nargs=4, metavar=("WHICH", "CSV", "KERNEL_REGEX", "LAUNCHES"),
                    help="write profiles/traffic.json[WHICH] from an ncu raw CSV export and exit")
    ap.add_argument("--frames", type=int, default=512,
                    help="speed3r only: frames of the synthetic sequence (512 is the workload; fewer give the "
                         "small cases that profiler captures use)")
    return ap.parse_args()


def algorithmic_flops(w, idx: np.ndarray) -> dict:
    """4 * d * sum over (token, head) of the keys each branch attends (cmp: B block
    means; slc: tokens of the routed blocks; win: in-block band)."""
    off = w.off.astype(np.int64)
    n = np.diff(off)
    B, Hq, d = w.n_blocks, w.n_q_heads, w.head_dim
    N = int(off[-1])
    cmp = N * Hq * B
    sel_tokens = n[idx].sum(axis=1) if idx.ndim == 2 else n[idx].sum(axis=-1).mean(axis=1)
    slc = float((n * sel_tokens).sum()) * Hq
    win = 0
    if w.window > 0 and w.n_gates >= 3:
        for nb in np.unique(n):
            r = np.arange(nb)
            lo = np.maximum(0, r - w.window // 2)
            hi = np.minimum(nb - 1, r + w.window // 2 - 1)
            win += int((hi - lo + 1).sum()) * int((n == nb).sum())
        win *= Hq
    f = 4 * d
    return {"cmp": f * cmp, "slc": f * slc, "win": f * win, "total": f * (cmp + slc + win)}


def backward_flops(fwd: dict) -> dict:
    """Algorithmic backward FLOPs over the same attended (row, key) pairs: the score recompute
    (2d), dV (2d), dP (2d), dQ (2d) and dK (2d), i.e. 2.5x the forward's 4d per pair."""
    return {k: 2.5 * v for k, v in fwd.items()}


KERNEL_SOURCES = {"attn": ["attn_tc.cu", "tc_ptx.cuh", "tma_map.cuh", "lsrm_common.cuh"],
                  "bwd": ["backward.cu", "tc_ptx.cuh", "tma_map.cuh", "lsrm_common.cuh"]}


def kernel_source_hash(which: str) -> str:
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[which]:
        with open(os.path.join(ROOT, "block_sparse_gqa_nsa_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


TRAFFIC_JSON = os.path.join(ROOT, "profiles", "traffic.json")
TRAFFIC_METRICS = ("dram__bytes_read.sum", "dram__bytes_write.sum")


def profiled_traffic(which: str):
    """DRAM bytes per launch from profiles/traffic.json (written by `bench.py --record-traffic`
    from an ncu capture), used only while the kernel sources hash to the value recorded with
    it (else None: the kernel has changed since the counters were taken)."""
    if not os.path.exists(TRAFFIC_JSON):
        return None
    with open(TRAFFIC_JSON) as f:
        rec = json.load(f).get(which)
    if rec is None or rec.get("source_hash") != kernel_source_hash(which):
        return None
    return float(rec["bytes_per_launch"])


def _ncu_bytes(value: str, unit: str) -> float:
    scale = {"byte": 1.0, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "Tbyte": 1e12,
             "KB": 1e3, "MB": 1e6, "GB": 1e9}
    return float(value.replace(",", "")) * scale[unit]


def record_traffic(which: str, csv_path: str, kernel_regex: str, launches_per_unit: int, note: str) -> dict:
    """Write profiles/traffic.json[which] from `ncu -i <rep> --page raw --csv` output: the DRAM
    read + write bytes of the launches whose name matches kernel_regex, summed over each group of
    launches_per_unit consecutive launches (one call) and averaged over the groups."""
    import csv
    import re
    with open(csv_path) as f:
        rows = list(csv.reader(f))
    head, units = rows[0], rows[1]
    col = {n: i for i, n in enumerate(head)}
    name_col = col["Kernel Name"]
    per = []
    for r in rows[2:]:
        if len(r) != len(head) or not re.search(kernel_regex, r[name_col]):
            continue
        per.append(sum(_ncu_bytes(r[col[m]], units[col[m]]) for m in TRAFFIC_METRICS))
    if not per or len(per) % launches_per_unit:
        raise ValueError(f"{len(per)} matching launches, not a multiple of {launches_per_unit}")
    groups = [sum(per[i:i + launches_per_unit]) for i in range(0, len(per), launches_per_unit)]
    rec = {"bytes_per_launch": sum(groups) / len(groups), "source_hash": kernel_source_hash(which),
           "kernel_regex": kernel_regex, "launches_per_unit": launches_per_unit, "captures": len(groups),
           "note": note}
    data = {}
    if os.path.exists(TRAFFIC_JSON):
        with open(TRAFFIC_JSON) as f:
            data = json.load(f)
    data[which] = rec
    with open(TRAFFIC_JSON, "w") as f:
        json.dump(data, f, indent=1, sort_keys=True)
        f.write("\n")
    return rec


def cpu_baseline(value: float, sample: str) -> dict:
    """The oracle's timing as a reported baseline: one thread of the host's cores."""
    return {"value": value, "unit": "tokens/s", "cores": 1, "host_cores": os.cpu_count(), "kind": "oracle",
            "sample": sample}


def max_over_ranks(ms: float, device, world: int) -> float:
    """The slowest rank's time: every rank contributes its device-measured milliseconds and all
    receive the maximum (one all-reduce; a no-op on one rank)."""
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(world: int, units_per_rank: int, steps: int, max_ms: float) -> float:
    """Whole-job units per second: every rank processes units_per_rank per step (replicas)."""
    return world * units_per_rank * steps / (max_ms / 1000.0)


def pipelined_e2e(dev, world: int, steps: int, warmup: int, h_in: dict, outs_like: dict, compute):
    """End-to-end steps through the public API with the host copies inside the timed region:
    step i's inputs go host -> device on one stream, its compute runs on the current stream and
    its result comes back on a third, with two sets of device buffers, so the copies of
    neighbouring steps overlap the compute (and each other: the link is full duplex).
    Returns (max-over-ranks milliseconds for `steps` steps, the last step's host outputs)."""
    import torch
    import torch.distributed as dist
    h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    comp_s = torch.cuda.current_stream(dev)
    d_in = [{n: torch.empty(t.shape, dtype=t.dtype, device=dev) for n, t in h_in.items()} for _ in range(2)]
    d_out = [{n: torch.empty_like(t) for n, t in outs_like.items()} for _ in range(2)]
    p_out = [{n: torch.empty(t.shape, dtype=t.dtype).pin_memory() for n, t in outs_like.items()} for _ in range(2)]
    h2d_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    d2h_done = [torch.cuda.Event() for _ in range(2)]

    def run(n):
        for i in range(n):
            b = i & 1
            if i >= 2:
                h2d_s.wait_event(comp_done[b])  # step i - 2 has consumed buffer b's inputs
            with torch.cuda.stream(h2d_s):
                for name, t in h_in.items():
                    d_in[b][name].copy_(t, non_blocking=True)
            h2d_done[b].record(h2d_s)
            comp_s.wait_event(h2d_done[b])
            if i >= 2:
                comp_s.wait_event(d2h_done[b])  # step i - 2's result has left buffer b
            compute(d_in[b], d_out[b], comp_s)
            comp_done[b].record(comp_s)
            d2h_s.wait_event(comp_done[b])
            with torch.cuda.stream(d2h_s):
                for name, t in d_out[b].items():
                    p_out[b][name].copy_(t, non_blocking=True)
            d2h_done[b].record(d2h_s)

    run(max(3, warmup))
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(h2d_s)
    run(steps)
    end.record(d2h_s)
    torch.cuda.synchronize(dev)
    return max_over_ranks(start.elapsed_time(end), dev, world), p_out[(steps - 1) & 1]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""

    def __init__(self, gpu_index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={q}",
                                       "--format=csv,noheader,nounits", "-lms", "100"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None
        # start timing only once nvidia-smi is producing samples
        t0 = time.time()
        while self.p is not None and time.time() - t0 < 5.0 and os.path.getsize(self.f.name) == 0:
            time.sleep(0.05)

    def stop(self) -> dict:
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.seek(0)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.f.read().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        os.unlink(self.f.name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ------------------------------------------------------------------------------------------------
# the oracle on the host: cpu_baseline of our arm, and the whole reference arm
# ------------------------------------------------------------------------------------------------

def sparse_config(w, world: int, seed: int) -> dict:
    """The workload description both arms print (identical dicts, so the lines compare)."""
    return {"workload": WORKLOAD, "n_tokens": w.n_tokens, "n_blocks": w.n_blocks,
            "heads": f"{w.n_q_heads}q/{w.n_kv_heads}kv", "head_dim": w.head_dim, "top_k": w.top_k,
            "window": w.window, "route": "geometric",
            "parallelism": f"replicas{world}" if world > 1 else "single",
            "l2": "inputs larger than L2 (q 249 MB + out 249 MB per step)", "seed": seed}


def oracle_sample(w, idx, n_blocks: int, seed: int):
    """Time the fp64 oracle on a seeded sample of query blocks of the workload (1 thread)."""
    import oracle as O
    D = O.desc_for(w.n_tokens, w.n_blocks, w.n_q_heads, w.n_kv_heads, w.head_dim, w.top_k, w.window,
                   n_gates=w.n_gates)
    rng = np.random.default_rng(seed)
    qb = np.sort(rng.choice(w.n_blocks, size=n_blocks, replace=False)).astype(np.int32)
    t0 = time.perf_counter()
    O.forward(D, w.off, w.q, w.k, w.v, w.gates, idx, qblocks=qb)
    dt = time.perf_counter() - t0
    tokens = int((w.off[qb + 1] - w.off[qb]).sum())
    return tokens, dt


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from workloads import make_workload
    import oracle as O
    w = make_workload("sparse", seed=args.seed)
    D = O.desc_for(w.n_tokens, w.n_blocks, w.n_q_heads, w.n_kv_heads, w.head_dim, w.top_k, w.window)
    idx, _ = O.route_geometric(D, w.off, w.coords)
    per_step = 2  # query blocks per step: ~1 s of fp64 work each on one core
    for s in range(args.warmup):
        oracle_sample(w, idx, per_step, 1000 + s)
    tok, tsum = 0, 0.0
    for s in range(args.steps):
        t, dt = oracle_sample(w, idx, per_step, s)
        tok += t
        tsum += dt
    value = tok / tsum
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1000.0 * tsum / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": sparse_config(w, args.gpus, args.seed),
            "cpu_baseline": cpu_baseline(value, f"{per_step} seeded query blocks ({per_step * 64} tokens) per "
                                                f"step, fp64, 1 thread"),
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------------

def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    dev = torch.device("cuda", local)

    from block_sparse_gqa_nsa_b200 import nsa
    from block_sparse_gqa_nsa_b200.build import build
    from workloads import make_workload

    if rank == 0:
        build()
    if world > 1:
        dist.barrier()
    nsa.load_library()

    w = make_workload("sparse", seed=args.seed)
    N, B, Hq, Hkv, d, k = w.n_tokens, w.n_blocks, w.n_q_heads, w.n_kv_heads, w.head_dim, w.top_k

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)

    h_q, h_k, h_v, h_g = bf(w.q), bf(w.k), bf(w.v), bf(w.gates)
    h_off = torch.from_numpy(w.off.astype(np.int32))
    h_coords = torch.from_numpy(w.coords.astype(np.int32))
    q, kk, v, gates = h_q.to(dev), h_k.to(dev), h_v.to(dev), h_g.to(dev)
    off, coords = h_off.to(dev), h_coords.to(dev)
    desc = nsa.make_desc(N, B, w.max_block_len, Hq, Hkv, d, k, w.window, 0.0, False, w.n_gates)
    ws = nsa.workspace(desc, dev)
    kc = torch.empty(B, Hkv, d, dtype=torch.bfloat16, device=dev)
    vc = torch.empty_like(kc)
    idx = torch.empty(B, k, dtype=torch.int32, device=dev)
    out = torch.empty(N, Hq, d, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]

    def step(e=None):
        if e is not None:
            e[0].record(stream)
        nsa.lsrm_nsa_compress(desc, off, None, kk, v, None, kc, None, vc, None, None, ws)
        nsa.lsrm_route_geometric(desc, off, coords, idx, ws)
        if e is not None:
            e[1].record(stream)
        nsa.lsrm_nsa_attend(desc, off, q, kk, v, kc, vc, gates, idx, 1, 0, out, None, ws)
        if e is not None:
            e[2].record(stream)

    launches_per_step = 4  # compress, centroids, top-k, fused attention
    for _ in range(max(3, args.warmup)):
        step()
    st = nsa.lsrm_nsa_last_device_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")
    flops = algorithmic_flops(w, idx.cpu().numpy())

    sampler = ClockSampler(local) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step(ev[i])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    total_ms = t_start.elapsed_time(t_end)
    attn_ms = [ev[i][1].elapsed_time(ev[i][2]) for i in range(args.steps)]
    pre_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(args.steps)]
    total_ms = max_over_ranks(total_ms, dev, world)
    ms_per_step = total_ms / args.steps
    value = throughput(world, N, args.steps, total_ms)

    # end to end through lsrm_nsa_forward with pinned host buffers
    e2e = None
    if not args.no_e2e:
        h_in = {"q": h_q.pin_memory(), "k": h_k.pin_memory(), "v": h_v.pin_memory(), "gates": h_g.pin_memory(),
                "off": h_off.pin_memory(), "coords": h_coords.pin_memory()}

        def fwd(di, do, st):
            nsa.lsrm_nsa_forward(desc, di["off"], di["q"], di["k"], di["v"], di["gates"], di["coords"],
                                 nsa.ROUTE_GEOMETRIC, do["out"], None, None, ws, stream=st)

        te, last = pipelined_e2e(dev, world, args.steps, args.warmup, h_in, {"out": out}, fwd)
        h2d = sum(t.numel() * t.element_size() for t in h_in.values())
        d2h = out.numel() * out.element_size()
        e2e = {"value": throughput(world, N, args.steps, te), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "overlap": "H2D, compute and D2H of neighbouring steps on three streams"}
        if not torch.equal(last["out"].view(torch.int16), out.view(torch.int16).cpu()):
            raise RuntimeError("end-to-end output differs from the device-resident run")

    if rank == 0:
        peaks, src = measured_peaks()
        attn_avg = sum(attn_ms) / len(attn_ms)
        achieved = flops["total"] / (attn_avg / 1000.0) / 1e12
        peak = float(peaks["bf16_tflops"])
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": sparse_config(w, world, args.seed),
                "effective_tflops": flops["total"] / (ms_per_step / 1000.0) / 1e12,
                "flops_per_step": flops,
                "kernel_ms": {"fused_attention": attn_avg, "compress_and_route": sum(pre_ms) / len(pre_ms)},
                "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                             "frac": achieved / peak, "traffic": profiled_traffic("attn"),
                             "kernel": "nsa_attn (fused cmp+slc+win attention, gated combine)",
                             "peak_source": f"{src} bf16_tflops (burst)"},
                "gpu_launches": launches_per_step * args.steps,
                "clocks": clocks, "e2e": e2e}
        if not args.no_cpu_baseline and world == 1:
            n_blk = args.cpu_sample_blocks or 64
            tok, dt = oracle_sample(w, idx.cpu().numpy(), n_blk, 7)
            line["cpu_baseline"] = cpu_baseline(tok / dt, f"{n_blk} seeded query blocks ({tok} tokens) "
                                                          f"of the same workload, fp64, 1 thread, {dt:.1f} s")
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ------------------------------------------------------------------------------------------------
# the backward workload: gradients of the same layer, routing indices fixed from its forward
# ------------------------------------------------------------------------------------------------
BWD_METRIC = "sparse-attn bwd tokens/s and effective TFLOP/s vs B200 bf16 tensor peak"
BWD_WORKLOAD = "lsrm_sparse_stage_backward_dO_normal"


def oracle_backward_sample(w, idx, n_blocks: int, seed: int):
    """Time the fp64 oracle backward restricted to a seeded sample of query blocks (1 thread)."""
    import oracle as O
    D = O.desc_for(w.n_tokens, w.n_blocks, w.n_q_heads, w.n_kv_heads, w.head_dim, w.top_k, w.window,
                   n_gates=w.n_gates)
    rng = np.random.default_rng(seed)
    qb = np.sort(rng.choice(w.n_blocks, size=n_blocks, replace=False)).astype(np.int32)
    t0 = time.perf_counter()
    O.backward(D, w.off, w.q, w.k, w.v, w.gates, idx, w.dout, nthreads=1, qblocks=qb)
    dt = time.perf_counter() - t0
    return int((w.off[qb + 1] - w.off[qb]).sum()), dt


def bwd_config(w, world, seed):
    """The backward workload description both arms print (identical dicts)."""
    return {"workload": BWD_WORKLOAD, "n_tokens": w.n_tokens, "n_blocks": w.n_blocks,
            "heads": f"{w.n_q_heads}q/{w.n_kv_heads}kv", "head_dim": w.head_dim, "top_k": w.top_k,
            "window": w.window, "route": "geometric (indices fixed from the forward)",
            "parallelism": f"replicas{world}" if world > 1 else "single", "seed": seed,
            "l2": "inputs larger than L2 (q, dO, dq 249 MB each per step)",
            "saved_branch_outputs": "bf16 o_b from the forward (745 MB), one pass per branch"}


def run_backward_reference(args):
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    from workloads import make_workload
    import oracle as O
    w = make_workload("backward", seed=args.seed)
    D = O.desc_for(w.n_tokens, w.n_blocks, w.n_q_heads, w.n_kv_heads, w.head_dim, w.top_k, w.window)
    idx, _ = O.route_geometric(D, w.off, w.coords)
    for s in range(args.warmup):
        oracle_backward_sample(w, idx, 1, 1000 + s)
    tok, tsum = 0, 0.0
    for s in range(args.steps):
        t, dt = oracle_backward_sample(w, idx, 1, s)
        tok += t
        tsum += dt
    value = tok / tsum
    line = {"metric": BWD_METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1000.0 * tsum / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": bwd_config(w, args.gpus, args.seed),
            "cpu_baseline": cpu_baseline(value, "1 seeded query block (64 tokens) per step, fp64 backward, "
                                                "1 thread"),
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_backward(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    dev = torch.device("cuda", local)

    from block_sparse_gqa_nsa_b200 import nsa
    from block_sparse_gqa_nsa_b200.build import build
    from workloads import make_workload

    if rank == 0:
        build()
    if world > 1:
        dist.barrier()
    nsa.load_library()

    w = make_workload("backward", seed=args.seed)
    N, B, Hq, Hkv, d, k = w.n_tokens, w.n_blocks, w.n_q_heads, w.n_kv_heads, w.head_dim, w.top_k

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)

    h_in = {"q": bf(w.q), "k": bf(w.k), "v": bf(w.v), "gates": bf(w.gates), "dout": bf(w.dout),
            "off": torch.from_numpy(w.off.astype(np.int32)), "coords": torch.from_numpy(w.coords.astype(np.int32))}
    x = {n: t.to(dev) for n, t in h_in.items()}
    desc = nsa.make_desc(N, B, w.max_block_len, Hq, Hkv, d, k, w.window, 0.0, False, w.n_gates)
    ws = nsa.workspace(desc, dev)
    bf16 = torch.bfloat16
    out = torch.empty(N, Hq, d, dtype=bf16, device=dev)
    idx = torch.empty(B, 1, k, dtype=torch.int32, device=dev)
    lse = torch.empty(N, Hq, w.n_gates, dtype=torch.float32, device=dev)
    # the forward keeps its per-branch outputs (bf16), so the backward streams each branch once
    obr = torch.empty(N, Hq, w.n_gates, d, dtype=torch.bfloat16, device=dev)
    nsa.lsrm_nsa_forward(desc, x["off"], x["q"], x["k"], x["v"], x["gates"], x["coords"], nsa.ROUTE_GEOMETRIC,
                         out, idx, lse, ws, obr=obr)
    grads = {"dq": torch.empty(N, Hq, d, dtype=bf16, device=dev), "dk": torch.empty(N, Hkv, d, dtype=bf16, device=dev),
             "dv": torch.empty(N, Hkv, d, dtype=bf16, device=dev),
             "dgates": torch.empty(N, Hq, w.n_gates, dtype=bf16, device=dev)}
    stream = torch.cuda.current_stream(dev)

    def step(t=x, g=grads, ix=idx, ls=lse, ob=obr):
        nsa.lsrm_nsa_backward(desc, t["off"], t["q"], t["k"], t["v"], t["gates"], ix, 1, ls, t["dout"], g["dq"],
                              g["dk"], g["dv"], g["dgates"], ws, obr=ob)

    # compress, then the inverse routing lists (count, scan, fill, sort), then the query, local-key,
    # compressed-key and finishing kernels
    launches_per_step = 9
    for _ in range(max(3, args.warmup)):
        step()
    st = nsa.lsrm_nsa_last_device_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")
    flops = backward_flops(algorithmic_flops(w, idx.view(B, k).cpu().numpy()))

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    sampler = ClockSampler(local) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    total_ms = max_over_ranks(t0.elapsed_time(t1), dev, world)
    call_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
    value = throughput(world, N, args.steps, total_ms)

    e2e = None
    if not args.no_e2e:
        h_in = {n: t.pin_memory() for n, t in h_in.items() if n != "coords"}
        h_in["idx"] = idx.cpu().pin_memory()
        h_in["lse"] = lse.cpu().pin_memory()
        h_in["obr"] = obr.cpu().pin_memory()

        def bwd(di, do, st):
            nsa.lsrm_nsa_backward(desc, di["off"], di["q"], di["k"], di["v"], di["gates"], di["idx"], 1, di["lse"],
                                  di["dout"], do["dq"], do["dk"], do["dv"], do["dgates"], ws, stream=st,
                                  obr=di["obr"])

        te, last = pipelined_e2e(dev, world, args.steps, args.warmup, h_in, grads, bwd)
        h2d = sum(t.numel() * t.element_size() for t in h_in.values())
        d2h = sum(t.numel() * t.element_size() for t in grads.values())
        e2e = {"value": throughput(world, N, args.steps, te), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "overlap": "H2D, compute and D2H of neighbouring steps on three streams"}
        for n in grads:
            if not torch.equal(last[n].view(torch.int16), grads[n].view(torch.int16).cpu()):
                raise RuntimeError(f"end-to-end {n} differs from the device-resident run")

    if rank == 0:
        peaks, src = measured_peaks()
        achieved = flops["total"] / (call_ms / 1000.0) / 1e12
        peak = float(peaks["bf16_tflops"])
        line = {"metric": BWD_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": bwd_config(w, world, args.seed),
                "flops_per_step": flops,
                "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                             "frac": achieved / peak, "traffic": profiled_traffic("bwd"),
                             "kernel": "lsrm_nsa_backward (all launches of one call)",
                             "peak_source": f"{src} bf16_tflops (burst)"},
                "gpu_launches": launches_per_step * args.steps, "clocks": clocks, "e2e": e2e}
        if not args.no_cpu_baseline and world == 1:
            n_blk = args.cpu_sample_blocks or 24
            tok, dt = oracle_backward_sample(w, idx.view(B, k).cpu().numpy(), n_blk, 7)
            line["cpu_baseline"] = cpu_baseline(tok / dt, f"{n_blk} seeded query blocks ({tok} tokens) of the "
                                                          f"same workload, fp64 backward, 1 thread, {dt:.1f} s")
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ------------------------------------------------------------------------------------------------
# the other forward workloads: the dense-stage shape (every block selected) and the Speed3R variant
# ------------------------------------------------------------------------------------------------
EXTRA = {
    "dense": ("sparse-attn fwd tokens/s, dense-stage shape (k = B)", "lsrm_dense_stage_all_blocks"),
    "tiny": ("sparse-attn fwd tokens/s, score-routed small case", "lsrm_tiny_score_top4"),
    "speed3r": ("sparse-attn fwd tokens/s, Speed3R pooled-query variant", "speed3r_512_frames_top32_forced"),
    "mixture": ("self/cross gated mixture fwd tokens/s, dense-stage shape", "lsrm_dense_stage_self_cross_mixture"),
    "speed3r_backward": ("sparse-attn bwd tokens/s, Speed3R pooled-query variant",
                         "speed3r_512_frames_top32_forced_backward"),
}


def extra_config(w, workload: str, world: int, seed: int) -> dict:
    return {"workload": workload, "n_tokens": w.n_tokens, "n_blocks": w.n_blocks,
            "heads": f"{w.n_q_heads}q/{w.n_kv_heads}kv", "head_dim": w.head_dim, "top_k": w.top_k,
            "window": w.window, "n_forced": int(len(w.forced)),
            "parallelism": f"replicas{world}" if world > 1 else "single", "seed": seed,
            "l2": "inputs larger than L2"}


def speed3r_flops(w, idx: np.ndarray) -> dict:
    """4 d per attended (query, key): pooled queries against every block mean (one query per
    block and head), and every token against its block's forced and routed tokens."""
    n = np.diff(w.off.astype(np.int64))
    B, H, d = w.n_blocks, w.n_q_heads, w.head_dim
    cmp = B * B * H
    forced_tok = int(n[w.forced].sum())
    routed_tok = n[np.clip(idx, 0, B - 1)].sum(axis=-1)  # [B][H]
    slc = float((n[:, None] * (forced_tok + routed_tok)).sum())
    f = 4 * d
    return {"cmp": f * cmp, "slc": f * slc, "total": f * (cmp + slc)}


def mixture_flops(w) -> dict:
    """4 d per (query, key) pair: every query attends every key of its own stream (self) and of
    the other stream (cross), for each query head."""
    nx = int(w.off[w.n_blocks_x])
    ny = w.n_tokens - nx
    f = 4 * w.head_dim * w.n_q_heads
    return {"self": float(f * (nx * nx + ny * ny)), "cross": float(f * 2 * nx * ny),
            "total": float(f * w.n_tokens * w.n_tokens)}


def run_extra(args):
    import torch
    metric, workload = EXTRA[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return 0
        if args.workload == "speed3r_backward":
            print(json.dumps({"impl": "reference", "metric": metric,
                              "unavailable": "the oracle's pooled-query backward has no per-block sampling: "
                                             "it runs at the test sizes only"}), flush=True)
            return 0
        return run_extra_reference(args, metric, workload)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    dev = torch.device("cuda", local)
    from block_sparse_gqa_nsa_b200 import nsa
    from block_sparse_gqa_nsa_b200.build import build
    from workloads import make_workload
    if rank == 0:
        build()
    if world > 1:
        dist.barrier()
    nsa.load_library()
    base = "speed3r" if args.workload == "speed3r_backward" else args.workload
    if base == "speed3r" and args.frames != 512:
        w = make_workload("speed3r_small", seed=args.seed, n_frames=args.frames)
        workload = workload.replace("512_frames", f"{args.frames}_frames")
    else:
        w = make_workload(base, seed=args.seed)
    N, B, Hq, Hkv, d, k = w.n_tokens, w.n_blocks, w.n_q_heads, w.n_kv_heads, w.head_dim, w.top_k

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    q, kk, v, gates = bf(w.q), bf(w.k), bf(w.v), bf(w.gates)
    off = torch.from_numpy(w.off.astype(np.int32)).to(dev)
    forced = torch.from_numpy(w.forced.astype(np.int32)).to(dev) if len(w.forced) else None
    desc = nsa.make_desc(N, B, w.max_block_len, Hq, Hkv, d, k, w.window, 0.0, w.pooled_q, w.n_gates, forced)
    ws = nsa.workspace(desc, dev)
    out = torch.empty(N, Hq, d, dtype=torch.bfloat16, device=dev)
    if args.workload == "speed3r_backward":
        from workloads.nsa_workloads import STREAM_DOUT, normal_bf16
        idx = torch.empty(B, Hq, k, dtype=torch.int32, device=dev)
        lse = torch.empty(N, Hq, 2, dtype=torch.float32, device=dev)
        obr = torch.empty(N, Hq, 2, d, dtype=torch.bfloat16, device=dev)
        nsa.lsrm_nsa_forward(desc, off, q, kk, v, gates, None, nsa.ROUTE_SCORE, out, idx, lse, ws, obr=obr)
        dout = bf(normal_bf16(args.seed, STREAM_DOUT, (N, Hq, d), 1.0))
        dq, dk, dv = (torch.empty(N, Hq, d, dtype=torch.bfloat16, device=dev) for _ in range(3))
        dg = torch.empty(N, Hq, 2, dtype=torch.bfloat16, device=dev)

        def step():
            nsa.lsrm_nsa_backward(desc, off, q, kk, v, gates, idx, Hq, lse, dout, dq, dk, dv, dg, ws, obr=obr)
        # forced bitmap / prefix / gather, compress, two preparation passes, the pooled branch's dq and
        # dK/dV, the forced part's dq and dK/dV, four inverse-list passes, the routed dq and dK/dV, the
        # forced-token map and scatter
        launches_per_step = 18
    elif args.workload == "mixture":
        idx = None
        bx = w.n_blocks_x

        def step():
            nsa.lsrm_nsa_mixture(desc, off, bx, q, kk, v, gates, out, None, ws)
        launches_per_step = 1  # both attentions and the gated sum in one kernel
    elif args.workload == "speed3r":
        idx = torch.empty(B, Hq, k, dtype=torch.int32, device=dev)

        def step():
            nsa.lsrm_nsa_forward(desc, off, q, kk, v, gates, None, nsa.ROUTE_SCORE, out, idx, None, ws)
        # forced bitmap / prefix / gather, key row order, compress (Q, K, V), the bound pass, the
        # pooled compressed pass with the streaming top-k, the forced-token pass, the routed part
        # with the merge and gated combine
        launches_per_step = 9
    else:
        idx = None

        def step():
            nsa.lsrm_nsa_forward(desc, off, q, kk, v, gates, None, nsa.ROUTE_ALL, out, None, None, ws)
        launches_per_step = 2  # compress, fused attention over every block
    if args.workload == "tiny":
        idx = torch.empty(B, Hkv, k, dtype=torch.int32, device=dev)

        def step():
            nsa.lsrm_nsa_forward(desc, off, q, kk, v, gates, None, nsa.ROUTE_SCORE, out, idx, None, ws)
        launches_per_step = 4  # compress, score routing (row splits, then the top-k), fused attention
    for _ in range(max(3, args.warmup)):
        step()
    st = nsa.lsrm_nsa_last_device_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")
    if args.workload == "speed3r":
        flops = speed3r_flops(w, idx.cpu().numpy())
    elif args.workload == "speed3r_backward":
        # 10 d per attended (query, key) pair against the forward's 4 d: the score recompute, dV, dP,
        # dq and dK
        flops = {kk_: 2.5 * v_ for kk_, v_ in speed3r_flops(w, idx.cpu().numpy()).items()}
    elif args.workload == "mixture":
        flops = mixture_flops(w)
    elif args.workload == "tiny":
        flops = algorithmic_flops(w, idx.cpu().numpy())
    else:
        flops = algorithmic_flops(w, np.tile(np.arange(B, dtype=np.int32), (B, 1)))
    kernel_ms = None
    if args.workload == "tiny":
        # the score routing against the fused attention it feeds, each timed alone (CUDA events)
        kc32 = torch.empty(B, Hkv, d, dtype=torch.float32, device=dev)
        kc16, vc16 = (torch.empty(B, Hkv, d, dtype=torch.bfloat16, device=dev) for _ in range(2))
        nsa.lsrm_nsa_compress(desc, off, None, kk, v, kc32, kc16, None, vc16, ws=ws)

        def timed_ms(fn, n=100):
            for _ in range(5):
                fn()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(n):
                fn()
            e1.record()
            torch.cuda.synchronize(dev)
            return e0.elapsed_time(e1) / n
        kernel_ms = {"score_route": timed_ms(lambda: nsa.lsrm_route_score_topk(desc, off, q, kc32, idx, None, ws)),
                     "fused_attention": timed_ms(lambda: nsa.lsrm_nsa_attend(desc, off, q, kk, v, kc16, vc16, gates,
                                                                             idx, Hkv, 0, out, None, ws))}
    sampler = ClockSampler(local) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    total_ms = max_over_ranks(t0.elapsed_time(t1), dev, world)
    ms = total_ms / args.steps
    if rank == 0:
        peaks, src = measured_peaks()
        achieved = flops["total"] / (ms / 1000.0) / 1e12
        peak = float(peaks["bf16_tflops"])
        line = {"metric": metric, "value": throughput(world, N, args.steps, total_ms), "unit": "tokens/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic",
                "config": extra_config(w, workload, world, args.seed),
                "flops_per_step": flops,
                "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                             "frac": achieved / peak, "traffic": None,
                             "kernel": ("nsa_attn_tc_kernel (mixture mode, one launch)" if args.workload == "mixture"
                                        else "lsrm_nsa_backward (all launches of one call)"
                                        if args.workload == "speed3r_backward"
                                        else "lsrm_nsa_forward (all launches of one call)"),
                             "peak_source": f"{src} bf16_tflops (burst)"},
                "gpu_launches": launches_per_step * args.steps, "clocks": clocks}
        if kernel_ms is not None:
            line["kernel_ms"] = kernel_ms
        if not args.no_cpu_baseline and world == 1 and args.workload == "speed3r_backward":
            tok, dt = speed3r_backward_oracle_sample(args.seed)
            line["cpu_baseline"] = cpu_baseline(tok / dt, f"the whole backward of the 3-frame case ({tok} tokens, "
                                                          f"the oracle has no per-block sampling), fp64, "
                                                          f"1 thread, {dt:.1f} s")
        elif not args.no_cpu_baseline and world == 1:
            n_blk = args.cpu_sample_blocks or 4
            tok, dt = extra_oracle_sample(w, idx.cpu().numpy() if idx is not None else None, n_blk, 7)
            line["cpu_baseline"] = cpu_baseline(tok / dt, f"{n_blk} seeded query blocks ({tok} tokens) of the "
                                                          f"same workload, fp64, 1 thread, {dt:.1f} s")
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def speed3r_backward_oracle_sample(seed: int):
    """The fp64 oracle's pooled-query backward on the 3-frame case (1 thread), with routing
    indices from the oracle's own pooled routing."""
    import oracle as O
    from workloads import make_workload
    from workloads.nsa_workloads import STREAM_DOUT, normal_bf16
    w = make_workload("speed3r_small", seed=seed, n_frames=3)
    D = O.desc_for(w.n_tokens, w.n_blocks, w.n_q_heads, w.n_kv_heads, w.head_dim, w.top_k, w.window,
                   n_gates=w.n_gates, pooled_q=w.pooled_q)
    qc = O.compress(D, w.off, w.q, w.n_q_heads)
    kc = O.compress(D, w.off, w.k, w.n_kv_heads)
    idx, _ = O.route_pooled(D, qc, kc, w.forced)
    dout = normal_bf16(seed, STREAM_DOUT, (w.n_tokens, w.n_q_heads, w.head_dim), 1.0)
    t0 = time.perf_counter()
    O.backward_pooled(D, w.off, w.q, w.k, w.v, w.gates, idx, w.forced, dout, nthreads=1)
    return w.n_tokens, time.perf_counter() - t0


def extra_oracle_sample(w, idx, n_blocks: int, seed: int):
    """The fp64 oracle forward on a seeded sample of query blocks (1 thread); the Speed3R sample
    uses routing indices given (the GPU's, or the oracle's own in the reference arm)."""
    import oracle as O
    D = O.desc_for(w.n_tokens, w.n_blocks, w.n_q_heads, w.n_kv_heads, w.head_dim, w.top_k, w.window,
                   n_gates=w.n_gates, pooled_q=w.pooled_q)
    rng = np.random.default_rng(seed)
    qb = np.sort(rng.choice(w.n_blocks, size=n_blocks, replace=False)).astype(np.int32)
    if idx is None:
        idx = np.tile(np.arange(w.n_blocks, dtype=np.int32), (w.n_blocks, 1))
    t0 = time.perf_counter()
    if w.route == "mixture":
        O.mixture(D, w.off, w.q, w.k, w.v, w.gates, w.n_blocks_x, qblocks=qb)
    elif w.pooled_q:
        O.forward(D, w.off, w.q, w.k, w.v, w.gates, idx, forced=w.forced, qblocks=qb)
    else:
        O.forward(D, w.off, w.q, w.k, w.v, w.gates, idx, qblocks=qb)
    dt = time.perf_counter() - t0
    return int((w.off[qb + 1] - w.off[qb]).sum()), dt


def run_extra_reference(args, metric, workload):
    from workloads import make_workload
    import oracle as O
    w = make_workload(args.workload, seed=args.seed)
    D = O.desc_for(w.n_tokens, w.n_blocks, w.n_q_heads, w.n_kv_heads, w.head_dim, w.top_k, w.window,
                   n_gates=w.n_gates, pooled_q=w.pooled_q)
    qc = kc = kc_score = None
    if w.route == "score" and not w.pooled_q:
        kc_score = O.compress(D, w.off, w.k, w.n_kv_heads)
    if w.pooled_q:
        qc = O.compress(D, w.off, w.q, w.n_q_heads)
        kc = O.compress(D, w.off, w.k, w.n_kv_heads)
    all_idx = np.tile(np.arange(w.n_blocks, dtype=np.int32), (w.n_blocks, 1))

    def one(seed):
        # one seeded query block: (Speed3R: its routing by the oracle, then) the layer forward
        qb = np.array([np.random.default_rng(seed).integers(w.n_blocks)], dtype=np.int32)
        t0 = time.perf_counter()
        if w.route == "mixture":
            O.mixture(D, w.off, w.q, w.k, w.v, w.gates, w.n_blocks_x, qblocks=qb)
        elif w.route == "score":
            rows, _ = O.route_score(D, w.off, w.q, kc_score, qblocks=qb)
            idx = np.zeros((w.n_blocks, w.n_kv_heads, w.top_k), dtype=np.int32)
            idx[qb] = rows
            O.forward(D, w.off, w.q, w.k, w.v, w.gates, idx, qblocks=qb)
        elif w.pooled_q:
            rows, _ = O.route_pooled(D, qc, kc, w.forced, qblocks=qb)
            idx = np.zeros((w.n_blocks, w.n_q_heads, w.top_k), dtype=np.int32)
            idx[qb] = rows
            O.forward(D, w.off, w.q, w.k, w.v, w.gates, idx, forced=w.forced, qblocks=qb)
        else:
            O.forward(D, w.off, w.q, w.k, w.v, w.gates, all_idx, qblocks=qb)
        return int((w.off[qb + 1] - w.off[qb]).sum()), time.perf_counter() - t0

    for s in range(args.warmup):
        one(1000 + s)
    tok, tsum = 0, 0.0
    for s in range(args.steps):
        t, dt = one(s)
        tok += t
        tsum += dt
    value = tok / tsum
    line = {"metric": metric, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1000.0 * tsum / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": extra_config(w, workload, args.gpus, args.seed),
            "cpu_baseline": cpu_baseline(value, "1 seeded query block per step, fp64, 1 thread"),
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------------------------
# the memory-bound kernels on their own: achieved HBM bandwidth against the measured copy peak
# ------------------------------------------------------------------------------------------------

def run_bandwidth(args):
    """Block mean-pool of Q, K and V (Speed3R shape, --frames frames), the standalone gated combine
    of two fp32 branch outputs (same shape) and the geometric routing of the sparse stage, each
    timed alone with CUDA events (mean of --steps launches after --warmup); algorithmic bytes =
    every input byte read once plus every output byte written once."""
    import torch
    from block_sparse_gqa_nsa_b200 import nsa
    from block_sparse_gqa_nsa_b200.build import build
    from workloads import make_workload
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    if args.impl == "reference":
        print(json.dumps({"impl": "reference", "unavailable": "the bandwidth workload times single kernels; "
                          "the oracle has no counterpart of a kernel's memory traffic"}))
        return 0
    build()
    nsa.load_library()
    dev = torch.device("cuda", 0)
    peaks, src = measured_peaks()
    hbm = float(peaks["hbm_gbs"])

    def timed(fn):
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            fn()
        e1.record()
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / args.steps

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    res = {}
    w = make_workload("speed3r_small", seed=args.seed, n_frames=args.frames)
    N, B, H, d = w.n_tokens, w.n_blocks, w.n_q_heads, w.head_dim
    q, k, v, g = bf(w.q), bf(w.k), bf(w.v), bf(w.gates)
    off = torch.from_numpy(w.off.astype(np.int32)).to(dev)
    desc = nsa.make_desc(N, B, w.max_block_len, H, H, d, w.top_k, 0, 0.0, True, 2)
    ws = nsa.workspace(desc, dev)
    outs = {n: torch.empty(B, H, d, dtype=dt, device=dev) for n, dt in
            (("kc32", torch.float32), ("kc", torch.bfloat16), ("vc32", torch.float32), ("vc", torch.bfloat16),
             ("qc32", torch.float32), ("qc", torch.bfloat16))}
    ms = timed(lambda: nsa.lsrm_nsa_compress(desc, off, q, k, v, outs["kc32"], outs["kc"], outs["vc32"], outs["vc"],
                                             outs["qc32"], outs["qc"], ws))
    byt = 3 * N * H * d * 2 + 3 * B * H * d * 6 + (B + 1) * 4
    res["compress_kernel"] = {"what": f"mean-pool of q, k, v over {B} blocks ({N} tokens, {H}x{d})",
                              "ms": ms, "bytes": byt}
    oc = torch.randn(N, H, d, device=dev)
    osl = torch.randn(N, H, d, device=dev)
    out = torch.empty(N, H, d, dtype=torch.bfloat16, device=dev)
    ms = timed(lambda: nsa.lsrm_nsa_gate_combine(desc, oc, osl, None, g, out))
    byt = 2 * N * H * d * 4 + N * H * 2 * 2 + N * H * d * 2
    res["gate_combine_kernel"] = {"what": f"out = g_cmp o_cmp + g_slc o_slc, {N} tokens x {H}x{d} fp32 in, bf16 out",
                                  "ms": ms, "bytes": byt}
    del q, k, v, oc, osl, out, outs, ws
    ws_ = make_workload("sparse", seed=args.seed)
    offs = torch.from_numpy(ws_.off.astype(np.int32)).to(dev)
    coords = torch.from_numpy(ws_.coords.astype(np.int32)).to(dev)
    dsc = nsa.make_desc(ws_.n_tokens, ws_.n_blocks, ws_.max_block_len, ws_.n_q_heads, ws_.n_kv_heads, ws_.head_dim,
                        ws_.top_k, ws_.window, 0.0, False, ws_.n_gates)
    wsp = nsa.workspace(dsc, dev)
    idx = torch.empty(ws_.n_blocks, ws_.top_k, dtype=torch.int32, device=dev)
    ms = timed(lambda: nsa.lsrm_route_geometric(dsc, offs, coords, idx, wsp))
    byt = ws_.n_tokens * 12 + (ws_.n_blocks + 1) * 4 + ws_.n_blocks * ws_.top_k * 4
    res["centroid_kernel+geo_topk_reg_kernel"] = {
        "what": f"geometric routing of the sparse stage ({ws_.n_blocks} blocks, top-{ws_.top_k}); the centroids "
                f"({ws_.n_blocks * 12} B) stay in L2 for the top-k's {ws_.n_blocks}^2 distances", "ms": ms,
        "bytes": byt}
    for r in res.values():
        r["gbs"] = r["bytes"] / (r["ms"] / 1000.0) / 1e9
        r["frac"] = r["gbs"] / hbm
    print(json.dumps({"metric": "achieved HBM GB/s of the memory-bound kernels", "unit": "GB/s",
                      "peak": hbm, "peak_source": f"{src} hbm_gbs", "steps": args.steps, "warmup": args.warmup,
                      "frames": args.frames, "kernels": res}), flush=True)
    return 0


def main():
    args = parse()
    if args.workload == "bandwidth":
        return run_bandwidth(args)
    if args.record_traffic:
        which, csv_path, regex, launches = args.record_traffic
        print(json.dumps(record_traffic(which, csv_path, regex, int(launches), f"from {os.path.basename(csv_path)}")))
        return 0
    if args.workload == "backward":
        return run_backward_reference(args) if args.impl == "reference" else run_backward(args)
    if args.workload in EXTRA:
        return run_extra(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
