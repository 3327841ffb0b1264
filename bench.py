#!/usr/bin/env python
"""Benchmark of the ClusterAttention forward path (cluster -> route -> attend).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one forward of one attention layer on the tabular-shaped
workload (B=1, H=8, N=65,536 tokens, d=64, bf16, cluster size 128, 64 of 512
key clusters kept per query cluster, compensation on), inputs resident in HBM.
Under torchrun the layer's heads are split over the ranks (each head is
clustered and attended on its own, so no collective runs on the data path;
strong scaling); --shard layers gives each rank an independent layer
instead (weak scaling). The reported value is layer forwards per second over
all ranks, timed with CUDA events as the max over ranks.

--config 5 runs the sweep over cluster size, keep fraction and compensation
at N = 32,768 (d = 64 and 128), one JSON line per point.

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


# Figures taken from single-kernel ncu captures of the attention kernel
# (`ncu --set full --clock-control none -k regex:tc_attend -s 1 -c 1` around
# `python bench.py --steps 1 --warmup 3 --no-cpu-baseline [--config N]`):
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) and tensor-pipe
# activity of one launch. Each entry holds for the attention source whose
# SHA-256 starts with `sha` and the workload it names; for any other source
# or workload the bench reports null.
ATTN_CAPTURES = [
    {"sha": "ff025bea226f0ade", "workload": "cfg2-lowrank-N65536-d64-bf16",
     "traffic": 205868288 + 52257536, "tensor_pipe_pct": 31.01},
    {"sha": "ff025bea226f0ade", "workload": "cfg3-grid-21x45x80-d128-bf16",
     "traffic": 2505658880 + 781805568, "tensor_pipe_pct": 46.43},
]


def _attn_source_sha():
    import hashlib
    src = os.path.join(ROOT, "free_clustered_block_b200", "csrc", "attend_tc.cu")
    try:
        with open(src, "rb") as f:
            return hashlib.sha256(f.read()).hexdigest()
    except OSError:
        return ""


def attention_capture(workload_name):
    h = _attn_source_sha()
    for c in ATTN_CAPTURES:
        if h.startswith(c["sha"]) and c["workload"] == workload_name:
            return c
    return None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return dict(hbm=j["hbm_gbs"], bf16=j["bf16_tflops"], bf16_sus=j["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


L2_BYTES = 126 * 2 ** 20


def input_bytes(w):
    return 3 * w.B * w.H * w.N_alloc * w.d * (2 if w.dtype == "bf16" else 4)


def needs_flush(w):
    """Inputs that fit in L2 get an L2 flush before every timed step."""
    return input_bytes(w) < 2 * L2_BYTES


def key_size(w):
    """Key cluster size of a workload (the query cluster size c unless set)."""
    return getattr(w, "c_k", 0) or w.c


def key_clusters(w):
    return -(-w.n_valid // key_size(w))


def workload_config(w):
    mb = input_bytes(w) / 3 / 1e6
    l2 = (f"L2 flushed (512 MB write) before every timed step: Q, K, V are 3 x {mb:.1f} MB" if needs_flush(w)
          else f"inputs larger than L2: Q, K, V are 3 x {mb:.0f} MB per layer (L2 126 MB)")
    out = {"workload": w.name, "B": w.B, "H": w.H, "N": w.N_alloc, "n_valid": w.n_valid, "d": w.d, "c": w.c,
           "k": w.k, "clusters": w.C, "compensate": bool(w.compensate), "input_dtype": w.dtype, "l2": l2}
    if key_size(w) != w.c:
        out.update(c_k=key_size(w), key_clusters=key_clusters(w))
    return out


def dense_flops(w):
    """FLOPs of dense attention over the valid tokens (QK^T and PV)."""
    return 4.0 * w.n_valid * w.n_valid * w.d * w.H * w.B


def attention_flops(w, kept_counts=None, count_q=None):
    """Algorithmic FLOPs of the attention step: kept blocks (QK^T and PV over
    the kept clusters' c keys per query) plus the compensation terms of the
    excluded clusters. With adaptive selection the per-query-cluster kept
    counts (and the query-cluster sizes) give the sums."""
    ck, Ck = key_size(w), key_clusters(w)
    if kept_counts is None:
        kept = 4.0 * w.n_valid * (w.k * ck) * w.d * w.H * w.B
        smc = 4.0 * w.n_valid * (Ck - w.k) * w.d * w.H * w.B if w.compensate else 0.0
        return kept, smc
    import numpy as np
    kc = np.asarray(kept_counts, np.float64)
    nq = np.asarray(count_q, np.float64)
    kept = float(4.0 * (nq * kc * ck).sum() * w.d)
    smc = float(4.0 * (nq * (Ck - kc)).sum() * w.d) if w.compensate else 0.0
    return kept, smc


class ClockSampler:
    """SM clocks and throttle reasons sampled while the timed region runs: a
    thread reads them through NVML every 10 ms (read-only queries); without
    NVML, nvidia-smi every 200 ms."""
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.thread = None
        self.samples = []

    def _nvml_loop(self, nvml, handle):
        while not self.stop:
            try:
                sm = nvml.nvmlDeviceGetClockInfo(handle, nvml.NVML_CLOCK_SM)
                mx = nvml.nvmlDeviceGetMaxClockInfo(handle, nvml.NVML_CLOCK_SM)
                rs = nvml.nvmlDeviceGetCurrentClocksEventReasons(handle)
                self.samples.append((float(sm), float(mx), int(rs)))
            except Exception:
                pass
            time.sleep(0.01)

    def __enter__(self):
        import threading
        self.stop = False
        try:
            import pynvml as nvml
            nvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(vis.split(",")[self.gpu]) if vis and vis.split(",")[0].isdigit() else self.gpu
            handle = nvml.nvmlDeviceGetHandleByIndex(idx)
            self.thread = threading.Thread(target=self._nvml_loop, args=(nvml, handle), daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.thread = None
        fields = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                  "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={fields}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.gpu)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.stop = True
        if self.thread is not None:
            self.thread.join(timeout=2)
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for l in out.splitlines():
                parts = [p.strip() for p in l.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm, mx = float(parts[1]), float(parts[2])
                except ValueError:
                    continue
                rs = 0
                for nm, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        rs |= self.REASONS[nm]
                self.samples.append((sm, mx, rs))

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = sorted(nm for nm, bit in self.REASONS.items() if any(r & bit for _, _, r in self.samples))
        return {"sm_mhz": statistics.median(s for s, _, _ in self.samples), "sm_max_mhz": self.samples[-1][1],
                "reasons": reasons, "samples": len(self.samples),
                "source": "nvml every 10 ms" if self.thread is not None else "nvidia-smi every 200 ms"}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads", 1) for p in threadpool_info() if p.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def oracle_sample(w, n_clusters=48, heads=(0,), keep=None, selection="topk", recall=0.9, clustering="split"):
    """Time the oracle on a bounded sample and extrapolate to one whole layer.
    Per sampled head: full clustering of queries and keys, routing, and the
    attention of `n_clusters` query clusters (work per query cluster is the
    same k kept blocks plus compensation). Returns seconds per layer and, when
    `keep` is a dict, stores head 0's oracle output and sampled clusters there."""
    import numpy as np
    from oracle import ca_oracle as orc
    t_head = []
    for h in heads:
        Qf, Kf, Vf = (x[0, h, :w.n_valid].astype(np.float64) for x in (w.Q, w.K, w.V))
        t0 = time.perf_counter()
        if clustering == "random":
            hc = orc.cluster_head_random(Qf, Kf, w.c, seed=0, bh=h, c_k=key_size(w))
            kept = orc.topk_route(orc.centroid_scores(hc.qbar, hc.kbar), w.k)
        elif selection == "adaptive":
            hc = orc.cluster_head(Qf, Kf, w.c, seed=0, bh=h, query_form="adaptive", c_k=key_size(w),
                                  splitting="diagonal" if clustering == "diagonal" else "basic")
            kept = orc.adaptive_route(orc.centroid_scores(hc.qbar, hc.kbar), hc.count_k, w.d, recall, 16)
        else:
            hc = orc.cluster_head(Qf, Kf, w.c, seed=0, bh=h, c_k=key_size(w),
                                  splitting="diagonal" if clustering == "diagonal" else "basic")
            kept = orc.topk_route(orc.centroid_scores(hc.qbar, hc.kbar), w.k)
        t1 = time.perf_counter()
        sample = list(range(0, w.C, max(1, w.C // n_clusters)))[:n_clusters]
        out = orc.compensated_attention(Qf, Kf, Vf, hc.perm_q, hc.count_q, hc.perm_k, hc.count_k, kept, w.c,
                                        compensate=w.compensate, clusters=sample, c_k=key_size(w))
        t2 = time.perf_counter()
        t_head.append((t1 - t0) + (t2 - t1) * w.C / len(sample))
        if keep is not None and h == heads[0]:
            keep.update(head=h, out=out, perm_q=hc.perm_q, sample=sample)
    return statistics.mean(t_head) * w.H * w.B, {"heads": list(heads), "query_clusters": n_clusters}


def error_vs_dense(w, O_gpu_head, kept, n_clusters=8):
    """Max-abs and relative-L2 error against fp64 dense attention on the rows
    of `n_clusters` of the oracle's sampled query clusters of one head, for
    the GPU output and for the oracle's output."""
    import numpy as np
    from oracle import ca_oracle as orc
    h = kept["head"]
    Qf, Kf, Vf = (x[0, h, :w.n_valid].astype(np.float64) for x in (w.Q, w.K, w.V))
    rows = []
    for a in kept["sample"][:n_clusters]:
        r = kept["perm_q"][a * w.c:(a + 1) * w.c]
        rows.extend(int(x) for x in r if x >= 0)
    rows = np.array(rows)
    ref = orc.dense_attention(Qf, Kf, Vf, rows=rows)
    res = {"rows": int(rows.size), "reference": "fp64 dense softmax attention over all valid keys"}
    for name, got in (("gpu", O_gpu_head[rows].astype(np.float64)), ("oracle", kept["out"][rows])):
        d = got - ref
        res[name] = {"max_abs": float(np.abs(d).max()),
                     "rel_l2": float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300))}
    return res


def build_workload(args, rank: int):
    """The layer a rank runs: a configuration's workload, or (--tokens) the
    latency-scaling workload: configuration 2's generator (H = 8, d = 64,
    c = 128) at another token count, keeping 1/8 of the clusters or a fixed 64."""
    import workloads as wl
    if args.tokens:
        C = -(-args.tokens // 128)
        kk = 64 if args.fixed_k else max(1, C // 8)
        return wl.make_workload("lowrank", B=1, H=8, N=args.tokens, d=64, c=128, k=min(kk, C), dtype="bf16",
                                seed=rank_seed(rank, 2), compensate=args.smc == "on",
                                name=f"cfg2gen-lowrank-N{args.tokens}-d64-bf16-k{min(kk, C)}", rank=16,
                                noise=0.1)
    w = wl.config_workload(args.config, seed=rank_seed(rank, args.config),
                           **({"compensate": False} if args.smc == "off" else {}))
    return with_cluster_sizes(w, args)


def with_cluster_sizes(w, args):
    """--cq / --ck: other query / key cluster sizes on the same inputs, keeping
    the configuration's fraction of key clusters."""
    if not (getattr(args, "cq", 0) or getattr(args, "ck", 0)):
        return w
    import dataclasses
    cq = args.cq or w.c
    ck = args.ck or w.c
    keep = w.k / w.C
    Ck = -(-w.n_valid // ck)
    k = max(1, min(Ck, math.ceil(keep * Ck - 1e-9)))
    w2 = dataclasses.replace(w, c=cq, k=k, name=f"{w.name}-cq{cq}-ck{ck}")
    object.__setattr__(w2, "c_k", ck)
    return w2


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = build_workload(args, 0)
    times = []
    for i in range(args.warmup + args.steps):
        t, smp = oracle_sample(w, selection=args.selection, recall=args.recall, clustering=args.clustering)
        if i >= args.warmup:
            times.append(t)
    t = statistics.mean(times)
    value = 1.0 / t
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(workload_config(w), selection=args.selection, clustering=args.clustering,
                       **({"recall": args.recall, "min_count": 16} if args.selection == "adaptive" else {})),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": affinity_cores(), "blas_threads": blas_threads(),
                         "kind": "oracle",
                         "sample": f"per step: head 0 clustered and routed in full, attention of 48 of "
                                   f"{w.C} query clusters; extrapolated to {w.H} heads x {w.C} clusters"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def rank_seed(rank: int, config: int = CONFIG_ID) -> int:
    """Seed of the independent layer a rank runs (rank 0: the standard workload)."""
    return 1000 + config + 7919 * rank


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


def cluster_levels(ca, shape):
    """Levels of the split tree (the clustering launches 6 + 5 per level)."""
    n = ca.launch_count(shape, 0)
    return max(0, (n - 6) // 5)


def cluster_row_bytes(w, levels):
    """Algorithmic HBM bytes of the clustering stage: at every level of the
    split tree both tensors' rows are read once for the projections
    (2 x B x H x n x d x element size per level)."""
    esz = 2 if w.dtype == "bf16" else 4
    return float(levels) * 2 * w.B * w.H * w.n_valid * w.d * esz


def affinity_cores():
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def make_layer(ca, w, args, head_base=0, layout=None):
    adaptive = args.selection == "adaptive"
    return ca.ClusterAttention(w.B, w.H, w.N_alloc, w.n_valid, w.d, w.c, key_clusters(w) if adaptive else w.k,
                               dtype=w.dtype, compensate=w.compensate, selection=args.selection,
                               recall=args.recall, min_count=16, clustering=args.clustering,
                               head_base=head_base, c_k=getattr(w, "c_k", 0),
                               layout=layout or args.layout)


def head_share(w, world, rank):
    """This rank's slice of one layer's heads: the workload restricted to the
    flattened heads [b0, b1) (B = 1, H = b1 - b0) and b0, the global index of
    its first head."""
    import dataclasses
    from free_clustered_block_b200 import heads
    b0, b1 = heads.rank_slice(w.B * w.H, world, rank)
    cut = lambda x: x.reshape(w.B * w.H, w.N_alloc, w.d)[b0:b1][None]
    ws = dataclasses.replace(w, B=1, H=b1 - b0, Q=cut(w.Q), K=cut(w.K), V=cut(w.V),
                             name=f"{w.name}-heads{b0}-{b1}")
    return ws, b0


def time_layer(ca, torch, w, layer, Q, K, V, O, steps, warmup, barrier, local, sample_clocks=True):
    """Warm up, then time `steps` layer forwards with CUDA events on the
    launching stream: per step the clustering, the routing, the attention's
    preparation and the attention kernel (ca_attend_prepared) separately.
    Returns (total ms, per-stage mean ms, clock summary)."""
    stream = torch.cuda.current_stream()

    def step():
        layer.cluster(Q, K)
        layer.route()
        layer.attend_prepare(Q, K, V)
        layer.attend_prepared(Q, K, V, O)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    st = ca.ca_get_device_error()
    if st != ca.CA_OK:
        raise RuntimeError(f"device error after warm-up: {ca.status_string(st)}")
    flush = needs_flush(w)
    scrub = torch.empty(512 * 2 ** 20, dtype=torch.uint8, device="cuda") if flush else None
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(local) if sample_clocks else None
    if clk:
        clk.__enter__()
    try:
        barrier()
        torch.cuda.synchronize()
        start.record(stream)
        for i in range(steps):
            if flush:
                scrub.zero_()
            ev[i][0].record(stream)
            layer.cluster(Q, K)
            ev[i][1].record(stream)
            layer.route()
            ev[i][2].record(stream)
            layer.attend_prepare(Q, K, V)
            ev[i][3].record(stream)
            layer.attend_prepared(Q, K, V, O)
            ev[i][4].record(stream)
        end.record(stream)
        torch.cuda.synchronize()
        barrier()
    finally:
        if clk:
            clk.__exit__(None, None, None)
    st = ca.ca_get_device_error()
    if st != ca.CA_OK:
        raise RuntimeError(f"device error in the timed region: {ca.status_string(st)}")
    # with flushes, the steps are timed one by one (the flushes are not timed)
    total_ms = (sum(ev[i][0].elapsed_time(ev[i][4]) for i in range(steps)) if flush
                else start.elapsed_time(end))
    names = ("cluster", "route", "attend_prep", "attend_kernel")
    stage = {nm: statistics.mean(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(steps))
             for j, nm in enumerate(names)}
    stage["attend"] = stage["attend_prep"] + stage["attend_kernel"]
    return total_ms, stage, (clk.summary() if clk else None)


def time_dense(torch, layer, Q, K, V, iters):
    stream = torch.cuda.current_stream()
    Od = torch.empty_like(Q)
    layer.dense(Q, K, V, Od)
    torch.cuda.synchronize()
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0.record(stream)
    for _ in range(iters):
        layer.dense(Q, K, V, Od)
    d1.record(stream)
    torch.cuda.synchronize()
    return d0.elapsed_time(d1) / iters


def rooflines(ca, w, layer, stage, dense_ms, adaptive):
    """Attention kernel (tensor pipe, its own event time, burst peak: the
    timed region is short), dense kernel (same), clustering stage (HBM)."""
    pk = peaks()
    if adaptive:
        kc = layer.buf.kept_count.cpu().numpy()
        kept_f, smc_f = attention_flops(w, kc, layer.buf.count_q.cpu().numpy())
    else:
        kept_f, smc_f = attention_flops(w)
    attn_s = stage["attend_kernel"] / 1e3
    achieved = (kept_f + smc_f) / attn_s / 1e12
    cap = attention_capture(w.name)
    if w.dtype == "bf16":
        roof = {"kernel": f"tc_attend_kernel<{w.d}> (ca_attend_prepared: the attention kernel"
                          f"{' + padding-row zeroing' if w.N_alloc > w.n_valid else ''})",
                "bound": "tensor", "achieved": achieved, "peak": pk["bf16"], "unit": "TFLOP/s",
                "frac": achieved / pk["bf16"],
                "peak_source": f"bf16 dense burst (cuBLAS), {pk['source']}",
                "traffic": cap["traffic"] if cap else None,
                "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
                "tensor_pipe_pct": cap["tensor_pipe_pct"] if cap else None,
                "algorithmic_flops": kept_f + smc_f, "kernel_ms": stage["attend_kernel"]}
        dflops = dense_flops(w)
        dense_roof = {"kernel": f"tc_attend_kernel<{w.d}> dense mode", "bound": "tensor",
                      "achieved": dflops / (dense_ms / 1e3) / 1e12, "peak": pk["bf16"], "unit": "TFLOP/s",
                      "frac": dflops / (dense_ms / 1e3) / 1e12 / pk["bf16"],
                      "peak_source": f"bf16 dense burst (cuBLAS), {pk['source']}"}
    else:
        # fp32 inputs run the SIMT attention kernel on the FMA pipe: peak from
        # 148 SMs x 128 fp32 lanes x 2 FLOP x 1.965 GHz
        fp32_peak = 148 * 128 * 2 * 1.965e9 / 1e12
        roof = {"kernel": "simt_attend_kernel (ca_attend_prepared)", "bound": "alu", "achieved": achieved,
                "peak": fp32_peak, "unit": "TFLOP/s", "frac": achieved / fp32_peak, "traffic": None,
                "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 x 1.965 GHz",
                "algorithmic_flops": kept_f + smc_f, "kernel_ms": stage["attend_kernel"]}
        dense_roof = None
    levels = cluster_levels(ca, layer.shape)
    cbytes = cluster_row_bytes(w, levels)
    gbs = cbytes / (stage["cluster"] / 1e3) / 1e9
    cluster_roof = {"stage": "clustering (ca_cluster)", "bound": "hbm", "levels": levels,
                    "algorithmic_bytes": cbytes, "achieved": gbs, "peak": pk["hbm"], "unit": "GB/s",
                    "frac": gbs / pk["hbm"],
                    "definition": "per level, both tensors' rows read once: levels x 2 x B x H x n x d x bytes"}
    return roof, dense_roof, cluster_roof, (kept_f, smc_f)


def run_sweep(args):
    """Configuration 5: latency and error against dense attention over cluster
    size, keep fraction and compensation (one JSON line per point)."""
    import numpy as np
    import torch
    import free_clustered_block_b200 as ca
    import workloads as wl
    torch.cuda.set_device(0)
    no_barrier = (lambda: None)
    for d in (64, 128):
        for c in (64, 128, 256):
            for keep in (1 / 32, 1 / 8, 1 / 4, 1.0):
                for smc in (True, False):
                    w = wl.config_workload(5, d=d, c=c, keep=keep, compensate=smc)
                    Q, K, V = (torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
                               .cuda().contiguous() for x in (w.Q, w.K, w.V))
                    O = torch.empty_like(Q)
                    layer = make_layer(ca, w, args, layout="bhnd")
                    total_ms, stage, _ = time_layer(ca, torch, w, layer, Q, K, V, O, args.steps, args.warmup,
                                                    no_barrier, 0, sample_clocks=False)
                    ms = total_ms / args.steps
                    dense_ms = time_dense(torch, layer, Q, K, V, 3)
                    roof, dense_roof, cluster_roof, _ = rooflines(ca, w, layer, stage, dense_ms, False)
                    line = {"sweep": "config 5", "config": workload_config(w), "keep": keep,
                            "latency_ms": ms, "stage_ms": stage, "dense_ms": dense_ms,
                            "speedup_vs_dense": dense_ms / ms,
                            "attention_frac": roof["frac"], "dense_frac": dense_roof["frac"],
                            "cluster_hbm_frac": cluster_roof["frac"]}
                    if not args.no_cpu_baseline:
                        kept = {}
                        oracle_sample(w, n_clusters=8, keep=kept)
                        line["error_vs_dense_fp64"] = error_vs_dense(w, O[0, kept["head"]].float().cpu().numpy(),
                                                                     kept)
                    print(json.dumps(line), flush=True)
                    del layer, Q, K, V, O
                    torch.cuda.empty_cache()
    return 0


def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    import free_clustered_block_b200 as ca

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

    # One layer split by heads across the ranks (the default for N > 1: no
    # collective on the data path), or (--shard layers) an independent layer
    # per rank.
    shard_heads = world > 1 and args.shard == "heads"
    head_base = 0
    if shard_heads:
        w_layer = build_workload(args, 0)
        w, head_base = head_share(w_layer, world, rank)
    else:
        w = w_layer = build_workload(args, rank)
    if w.H == 0:
        raise RuntimeError("more ranks than heads: every rank needs at least one head")
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def dev(x):
        # [B, H, N, d], or token-major [B, N, H, d] with --layout bnhd
        a = x if args.layout == "bhnd" else x.transpose(0, 2, 1, 3)
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(tdt).cuda().contiguous()

    def head_rows(O, h):
        """Rows [N, d] of head h of batch 0 of a layer output."""
        return O[0, h] if args.layout == "bhnd" else O[0, :, h]

    Q, K, V = dev(w.Q), dev(w.K), dev(w.V)
    O = torch.empty_like(Q)
    adaptive = args.selection == "adaptive"
    layer = make_layer(ca, w, args, head_base)
    stream = torch.cuda.current_stream()
    # layer forwards completed by all ranks together per step
    layers_per_step = 1 if shard_heads else world

    local_ms, stage, clocks = time_layer(ca, torch, w, layer, Q, K, V, O, args.steps, args.warmup, barrier, local)
    total_ms = ranks_max(local_ms)
    ms_per_step = total_ms / args.steps
    value = whole_job_value(layers_per_step, args.steps, total_ms)

    # Dense attention (this library's own kernel) on the same inputs, for the speedup.
    dense_ms = ranks_max(time_dense(torch, layer, Q, K, V, max(1, min(args.steps, 3))))

    # End to end with host buffers (pinned), copies inside the region: the
    # single ca_forward_host call for top-k; the layer API (copy in, cluster,
    # route, attend, copy out) for adaptive selection.
    shape = layer.shape
    hQ, hK, hV = (x.cpu().pin_memory() for x in (Q, K, V))
    hO = torch.empty_like(hQ).pin_memory()
    if adaptive:
        dQ, dK, dV, dO = (torch.empty_like(x) for x in (Q, K, V, O))

        def e2e_step():
            dQ.copy_(hQ, non_blocking=True); dK.copy_(hK, non_blocking=True); dV.copy_(hV, non_blocking=True)
            layer(dQ, dK, dV, dO)
            hO.copy_(dO, non_blocking=True)
    else:
        wsh = torch.empty(ca.forward_host_workspace_bytes(shape, w.k), dtype=torch.uint8, device="cuda")

        def e2e_step():
            ca.ca_forward_host(hQ, hK, hV, shape, layer.params, w.k, w.compensate, hO, wsh)
    for _ in range(max(1, args.warmup)):
        e2e_step()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = ranks_max(e0.elapsed_time(e1))
    e2e_value = whole_job_value(layers_per_step, args.steps, e2e_ms)
    in_bytes = 3 * Q.numel() * Q.element_size()
    out_bytes = O.numel() * O.element_size()

    # The same layer captured once in a CUDA graph and replayed.
    graph_ms = None
    try:
        gstream = torch.cuda.Stream()
        gstream.wait_stream(stream)
        with torch.cuda.stream(gstream):
            layer(Q, K, V, O)
        gstream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=gstream):
            layer(Q, K, V, O)
        graph.replay()
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        g1.record(stream)
        torch.cuda.synchronize()
        graph_ms = ranks_max(g0.elapsed_time(g1)) / args.steps
        del graph
    except Exception as e:  # capture is an extra figure; the timed line above stands
        graph_ms = f"capture failed: {type(e).__name__}"

    roof, dense_roof, cluster_roof, (kept_f, smc_f) = rooflines(ca, w, layer, stage, dense_ms, adaptive)
    kc = layer.buf.kept_count.cpu().numpy() if adaptive else None
    per_step = [ca.launch_count(shape, s) for s in (0, 1, 2)]
    if args.clustering == "random" and per_step[0] > 1:
        # no metric, norm or direction kernels: plan, per level hash / select /
        # count / scatter, centroids
        levels = (per_step[0] - 6) // 5
        per_step[0] = 2 + 4 * levels
    if args.clustering == "diagonal" and per_step[0] > 1:
        # weighted query column sums and Gram, covariance reduce, basis
        per_step[0] += 4
    launches = args.steps * sum(per_step)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "strong" if shard_heads else "weak",
        "vs_baseline": None, "dtype": w.dtype,
        "dtype_detail": ("clustering and routing f64; attention bf16 products with f32 accumulation"
                         if w.dtype == "bf16" else "clustering and routing f64; attention f32"),
        "data": "synthetic",
        "config": dict(workload_config(w_layer), selection=args.selection, clustering=args.clustering,
                       layout="[B, H, N, d]" if args.layout == "bhnd" else "[B, N, H, d] (token-major)",
                       parallelism=(f"heads split over {world} GPUs ({w.H} per GPU, head_base {head_base} on "
                                    f"rank {rank})" if shard_heads else
                                    (f"an independent layer per GPU ({world} GPUs)" if world > 1 else "one GPU")),
                       **({"recall": args.recall, "min_count": 16,
                           "mean_kept": float(kc.mean())} if adaptive else {})),
        "latency_ms": ms_per_step, "stage_ms": stage, "dense_ms": dense_ms,
        "speedup_vs_dense": dense_ms / ms_per_step,
        "graph_ms_per_step": graph_ms,
        "tflops": {"dense_equivalent": layers_per_step * dense_flops(w_layer) / (ms_per_step / 1e3) / 1e12,
                   "algorithmic_attention": roof["achieved"]},
        "roofline": roof,
        "dense_roofline": dense_roof,
        "cluster_roofline": cluster_roof,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": in_bytes,
                "d2h_bytes_per_step": out_bytes, "ms_per_step": e2e_ms / args.steps},
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        kept = {}
        t_cpu, smp = oracle_sample(w, keep=kept, selection=args.selection, recall=args.recall,
                                   clustering=args.clustering)
        line["error_vs_dense_fp64"] = error_vs_dense(w, head_rows(O, kept["head"]).float().cpu().numpy(), kept)
        line["cpu_baseline"] = {"value": 1.0 / t_cpu, "unit": UNIT, "cores": affinity_cores(),
                                "blas_threads": blas_threads(), "kind": "oracle",
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
    ap.add_argument("--selection", choices=["topk", "adaptive"], default="topk",
                    help="key-cluster selection (adaptive: mass recall, capacity C per query cluster)")
    ap.add_argument("--recall", type=float, default=0.9)
    ap.add_argument("--clustering", choices=["split", "diagonal", "random"], default="split",
                    help="diagonal: diagonalized recursive splitting; random: the random-cluster "
                         "baseline of the paper's error analysis")
    ap.add_argument("--smc", choices=["on", "off"], default="on", help="striped mean-compensation")
    ap.add_argument("--tokens", type=int, default=0,
                    help="latency scaling: configuration 2's generator at this token count")
    ap.add_argument("--fixed-k", action="store_true", help="with --tokens: keep 64 clusters instead of 1/8")
    ap.add_argument("--cq", type=int, default=0, choices=[0, 64, 128, 256],
                    help="query cluster size (default: the configuration's)")
    ap.add_argument("--ck", type=int, default=0, choices=[0, 64, 128, 256],
                    help="key cluster size (default: the query cluster size); --cq 64 --ck 128 is the paper's "
                         "evaluated block shape")
    ap.add_argument("--shard", choices=["heads", "layers"], default="heads",
                    help="with N > 1 GPUs: split one layer's heads over the GPUs (default) or run an independent "
                         "layer per GPU")
    ap.add_argument("--layout", choices=["bhnd", "bnhd"], default="bhnd",
                    help="memory layout of Q, K, V and O: head-major [B, H, N, d] or token-major [B, N, H, d]")
    ap.add_argument("--config", type=int, choices=[1, 2, 3, 4, 5], default=CONFIG_ID,
                    help="workload (default 2: the metric's N = 64k configuration); 5: the sweep over cluster "
                         "size, keep fraction and compensation at N = 32,768, one JSON line per point")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.config == 5:
        return run_sweep(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
