#!/usr/bin/env python
"""Benchmark of the ClusterAttention forward path (cluster -> route -> attend).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one forward of one attention layer on the tabular-shaped
workload (B=1, H=8, N=65,536 tokens, d=64, bf16, cluster size 128, 64 of 512
key clusters kept per query cluster, compensation on), inputs resident in HBM.
Under torchrun each rank runs its own independent layer (weak scaling, no
collective on the data path); the reported value is layer forwards per second
over all ranks, timed with CUDA events as the max over ranks.

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload (one head's clustering and routing, a sample of its query clusters'
attention), extrapolated to the whole layer.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "ClusterAttention fwd latency & speedup vs dense attn at N=64k; tensor-pipe %"
UNIT = "layer-fwd/s"
CONFIG_ID = 2


# DRAM traffic (read + write bytes) of one attention-kernel launch on this
# workload, from the ncu capture summarised in
# profiles/tc_attend_kernel_64_128_layer_B1_H8_N65536.md. It describes the
# kernel source whose SHA-256 starts with `source_sha256`; for any other source
# the bench reports null.
ATTN_TRAFFIC = {"bytes": 205448192 + 52447232, "source_sha256": "1f30034b366e1e6c"}


def attention_traffic():
    import hashlib
    src = os.path.join(ROOT, "free_clustered_block_b200", "csrc", "attend_tc.cu")
    try:
        with open(src, "rb") as f:
            h = hashlib.sha256(f.read()).hexdigest()
    except OSError:
        return None
    return ATTN_TRAFFIC["bytes"] if h.startswith(ATTN_TRAFFIC["source_sha256"]) else None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return dict(hbm=j["hbm_gbs"], bf16=j["bf16_tflops"], bf16_sus=j["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


def workload_config(w):
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N_alloc, "n_valid": w.n_valid, "d": w.d, "c": w.c,
            "k": w.k, "clusters": w.C, "compensate": bool(w.compensate), "input_dtype": w.dtype,
            "l2": "inputs larger than L2: Q, K, V are 3 x 67 MB per layer (L2 126 MB)"}


def attention_flops(w):
    """Algorithmic FLOPs of the attention step: kept blocks (QK^T and PV over
    k*c keys per query) plus the compensation terms of the excluded clusters."""
    kept = 4.0 * w.n_valid * (w.k * w.c) * w.d * w.H * w.B
    smc = 4.0 * w.n_valid * (w.C - w.k) * w.d * w.H * w.B if w.compensate else 0.0
    return kept, smc


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.gpu)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads", 1) for p in threadpool_info() if p.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def oracle_sample(w, n_clusters=48, heads=(0,)):
    """Time the oracle on a bounded sample and extrapolate to one whole layer.
    Per sampled head: full clustering of queries and keys, routing, and the
    attention of `n_clusters` query clusters (work per query cluster is the
    same k kept blocks plus compensation). Returns seconds per layer."""
    import numpy as np
    from oracle import ca_oracle as orc
    t_head = []
    for h in heads:
        Qf, Kf, Vf = (x[0, h, :w.n_valid].astype(np.float64) for x in (w.Q, w.K, w.V))
        t0 = time.perf_counter()
        hc = orc.cluster_head(Qf, Kf, w.c, seed=0, bh=h)
        kept = orc.topk_route(orc.centroid_scores(hc.qbar, hc.kbar), w.k)
        t1 = time.perf_counter()
        sample = list(range(0, w.C, max(1, w.C // n_clusters)))[:n_clusters]
        orc.compensated_attention(Qf, Kf, Vf, hc.perm_q, hc.count_q, hc.perm_k, hc.count_k, kept, w.c,
                                  compensate=w.compensate, clusters=sample)
        t2 = time.perf_counter()
        t_head.append((t1 - t0) + (t2 - t1) * w.C / len(sample))
    return statistics.mean(t_head) * w.H * w.B, {"heads": list(heads), "query_clusters": n_clusters}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import workloads as wl
    w = wl.config_workload(CONFIG_ID)
    times = []
    for i in range(args.warmup + args.steps):
        t, smp = oracle_sample(w)
        if i >= args.warmup:
            times.append(t)
    t = statistics.mean(times)
    value = 1.0 / t
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"per step: head 0 clustered and routed in full, attention of 48 of "
                                   f"{w.C} query clusters; extrapolated to {w.H} heads x {w.C} clusters"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def rank_seed(rank: int) -> int:
    """Seed of the independent layer a rank runs (rank 0: the standard workload)."""
    return 1000 + CONFIG_ID + 7919 * rank


def whole_job_value(world: int, steps: int, total_ms: float) -> float:
    """Layer forwards per second over all ranks, from the max-over-ranks time."""
    return world * steps / (total_ms / 1e3)


def max_over_ranks(x: float, world: int, device) -> float:
    """Max of a per-rank time over the process group (identity on one rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    import free_clustered_block_b200 as ca
    import workloads as wl

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    def ranks_max(x):
        return max_over_ranks(x, world, "cuda")

    # Each rank: an independent layer (its own seeded inputs).
    w = wl.config_workload(CONFIG_ID, seed=rank_seed(rank))

    def dev(x):
        return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).cuda().contiguous()

    Q, K, V = dev(w.Q), dev(w.K), dev(w.V)
    O = torch.empty_like(Q)
    layer = ca.ClusterAttention(w.B, w.H, w.N_alloc, w.n_valid, w.d, w.c, w.k, dtype=w.dtype,
                                compensate=w.compensate)
    stream = torch.cuda.current_stream()

    def step():
        layer.cluster(Q, K)
        layer.route()
        layer.attend(Q, K, V, O)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = ca.ca_get_device_error()
    if st != ca.CA_OK:
        raise RuntimeError(f"device error after warm-up: {ca.status_string(st)}")

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        torch.cuda.synchronize()
        start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            layer.cluster(Q, K)
            ev[i][1].record(stream)
            layer.route()
            ev[i][2].record(stream)
            layer.attend(Q, K, V, O)
            ev[i][3].record(stream)
        end.record(stream)
        torch.cuda.synchronize()
        barrier()
    total_ms = ranks_max(start.elapsed_time(end))
    clocks = clk.summary()
    stage = {name: statistics.mean(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(args.steps))
             for j, name in enumerate(("cluster", "route", "attend"))}
    ms_per_step = total_ms / args.steps
    value = whole_job_value(world, args.steps, total_ms)

    # Dense attention (this build's own kernel) on the same inputs, for the speedup.
    Od = torch.empty_like(Q)
    layer.dense(Q, K, V, Od)
    torch.cuda.synchronize()
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dense_iters = max(1, min(args.steps, 3))
    d0.record(stream)
    for _ in range(dense_iters):
        layer.dense(Q, K, V, Od)
    d1.record(stream)
    torch.cuda.synchronize()
    dense_ms = ranks_max(d0.elapsed_time(d1) / dense_iters)

    # End to end through the C ABI with host buffers (pinned), copies inside the region.
    shape = layer.shape
    hQ, hK, hV = (x.cpu().pin_memory() for x in (Q, K, V))
    hO = torch.empty_like(hQ).pin_memory()
    wsh = torch.empty(ca.forward_host_workspace_bytes(shape, w.k), dtype=torch.uint8, device="cuda")
    for _ in range(max(1, args.warmup)):
        ca.ca_forward_host(hQ, hK, hV, shape, layer.params, w.k, w.compensate, hO, wsh)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.steps):
        ca.ca_forward_host(hQ, hK, hV, shape, layer.params, w.k, w.compensate, hO, wsh)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = ranks_max(e0.elapsed_time(e1))
    e2e_value = whole_job_value(world, args.steps, e2e_ms)
    in_bytes = 3 * Q.numel() * Q.element_size()
    out_bytes = O.numel() * O.element_size()

    pk = peaks()
    kept_f, smc_f = attention_flops(w)
    attn_s = stage["attend"] / 1e3
    achieved = (kept_f + smc_f) / attn_s / 1e12
    launches = args.steps * sum(ca.launch_count(shape, s) for s in (0, 1, 2))
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "dtype_detail": "clustering and routing f64; attention bf16 products with f32 accumulation",
        "data": "synthetic", "config": workload_config(w),
        "latency_ms": ms_per_step, "stage_ms": stage, "dense_ms": dense_ms,
        "speedup_vs_dense": dense_ms / ms_per_step,
        "roofline": {"kernel": "attention (ca_attend span: prep + attention)", "bound": "tensor",
                     "achieved": achieved, "peak": pk["bf16_sus"], "unit": "TFLOP/s",
                     "frac": achieved / pk["bf16_sus"], "traffic": attention_traffic(),
                     "traffic_unit": "bytes per launch (ncu dram__bytes_read + dram__bytes_write)",
                     "peak_source": f"bf16 dense sustained, {pk['source']}",
                     "algorithmic_flops": kept_f + smc_f},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": in_bytes,
                "d2h_bytes_per_step": out_bytes, "ms_per_step": e2e_ms / args.steps},
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        t_cpu, smp = oracle_sample(w)
        line["cpu_baseline"] = {"value": 1.0 / t_cpu, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                                "sample": f"head 0 clustered and routed in full, attention of 48 of {w.C} query "
                                          f"clusters; extrapolated to {w.H} heads x {w.C} clusters "
                                          f"({t_cpu:.1f} s per layer)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
