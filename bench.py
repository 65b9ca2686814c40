#!/usr/bin/env python
"""Decode throughput of the 78-layer IndexCache F/S stack at 128K context.

Workload (one replica per GPU): 78 layers, schedule F F F S S S ... with 21 F
layers, 32 decode queries, 131072 cached tokens per layer, indexer 64 heads x
128 dims (bf16 keys), top-k 2048, sparse MLA with 128 heads of 576 dims,
per-head sink and sigmoid gate. Synthetic seeded inputs drawn on the device.

A step is one pass of the whole hot path over the stack: on each F layer the
lightning indexer and top-k, on every layer the sparse MLA attention over the
shared index buffer. The metric is decode tokens/s = queries x steps / time.

Prints ONE JSON line (rank 0). ``--impl reference`` times the float64 CPU
oracle on a bounded sample of the same workload instead.
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
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode tokens/s per 78-layer F/S stack at 128K ctx; indexer GB/s vs HBM peak"
UNIT = "tokens/s"

L, N_FULL, B, N, H_I, D_I, TOPK, H = 78, 21, 32, 131072, 64, 128, 2048, 128
D_QK, D_V = 576, 512
WORKLOAD = "stack78_B32_N131072_topk2048"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained", d["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock/throttle samples at 100 ms, for the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.rows = []
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [x.strip() for x in line.split(",")]))

    def mark(self, begin: bool):
        if begin:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = self.rows
        if self.t0 is not None and self.t1 is not None:
            inside = [r for t, r in rows if self.t0 - 0.15 <= t <= self.t1 + 0.15]
            rows = inside if inside else [r for _, r in rows]
        else:
            rows = [r for _, r in rows]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if len(r) > 8 and num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if len(r) > 8 and num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = []
        for i, n in enumerate(names):
            if any(len(r) > 8 and r[5 + i].lower().startswith("active") for r in rows):
                reasons.append(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- CPU oracle sample
def cpu_sample_step(seed: int = 7):
    """One bounded oracle sample of the workload: one query through one F
    layer (indexer over all 131072 tokens + top-k) and one attention layer.
    Returns (seconds_F, seconds_attention, threads)."""
    import numpy as np
    import torch
    import oracle
    from lightning_indexer_cross_b200 import workloads as W

    g = torch.Generator().manual_seed(seed)
    q_i = (torch.randn((1, H_I, D_I), generator=g) / math.sqrt(D_I)).to(torch.bfloat16)
    w = torch.rand((1, H_I), generator=g) / H_I
    k = (torch.randn((1, N, D_I), generator=g) / math.sqrt(D_I)).to(torch.bfloat16)
    q = torch.randn((1, H, D_QK), generator=g).to(torch.bfloat16)
    kv = torch.randn((1, N, D_QK), generator=g).to(torch.bfloat16)
    sink = torch.randn((H,), generator=g) * 0.5
    gate = torch.randn((1, H, D_V), generator=g).to(torch.bfloat16)
    t0 = time.perf_counter()
    sc = oracle.indexer_scores(q_i, w, k)
    idx = oracle.topk_indices(sc, TOPK)
    t1 = time.perf_counter()
    oracle.sparse_mla(q, kv, idx, sink, gate, 1.0 / math.sqrt(D_QK))
    t2 = time.perf_counter()
    return t1 - t0, t2 - t1


def cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_tokens_per_s(tf, ta):
    # per decoded token (one query): 21 F layers (indexer + top-k + attention)
    # and 57 S layers (attention)
    return 1.0 / (N_FULL * tf + L * ta)


# ----------------------------------------------------------------------------- dist
def dist_setup(n_gpus, backend=None):
    """One process per GPU (torchrun): NCCL between the ranks' GPUs; the CPU
    tests pass backend="gloo"."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = backend or "nccl"
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """The maximum of a per-rank device time over all ranks."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_seed(rank):
    """Each rank runs an independent replica of the decode batch."""
    return 2 + rank


def replica_value(world, queries, steps, ms_max):
    """Whole-job decode tokens/s: every rank's queries over the slowest rank's time."""
    return world * queries * steps / (ms_max / 1000.0)


# ----------------------------------------------------------------------------- reference arm
def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    for _ in range(args.warmup_ref):
        cpu_sample_step()
    tf_all, ta_all = [], []
    t0 = time.perf_counter()
    for s in range(args.steps):
        tf, ta = cpu_sample_step(seed=100 + s)
        tf_all.append(tf)
        ta_all.append(ta)
    wall = time.perf_counter() - t0
    tf, ta = sum(tf_all) / len(tf_all), sum(ta_all) / len(ta_all)
    v = cpu_tokens_per_s(tf, ta)
    sample = (f"1 query: indexer+top-k over N={N} on 1 F layer and sparse MLA on 1 layer per step, "
              f"extrapolated to the 78-layer schedule (21 F + 78 attention)")
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * wall / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "layers": L, "full_layers": N_FULL, "queries": B, "ctx": N,
                   "topk": TOPK, "sample": "1 query per step"},
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- native arm
def distinct_rows(trace, sched):
    import torch
    tot = 0
    for l in range(len(sched)):
        u = torch.unique(trace[l][trace[l] >= 0])
        tot += u.numel()
    return tot


def run_native(args):
    import torch
    from lightning_indexer_cross_b200 import _abi, ops
    from lightning_indexer_cross_b200 import workloads as W

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    hbm_gbs, tf_burst, tf_sust, peak_kind = peaks()

    wl = W.stack(dev, seed=replica_seed(rank), L=L, n_full=N_FULL, B=B, N=N, H_I=H_I, d_I=D_I, topk=TOPK, H=H)
    st = ops.stack_from_workload(wl, trace=False)
    torch.cuda.synchronize()

    # one traced step to count distinct gathered rows (algorithmic attention bytes)
    st_tr = ops.stack_from_workload(wl, trace=True)
    st_tr.step()
    torch.cuda.synchronize()
    rows_distinct = distinct_rows(st_tr.trace, wl.schedule)
    launches_per_step = st_tr.step()
    torch.cuda.synchronize()
    if st_tr.device_status() != 0:
        raise RuntimeError("device status not OK after a traced step")
    del st_tr

    stream = torch.cuda.Stream(device=dev)
    graph = None
    if not args.no_graph:
        st.step()  # first call sets kernel attributes before capture
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            st.step()
        torch.cuda.synchronize()

    def one_step():
        if graph is not None:
            graph.replay()
        else:
            st.step()

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()

    clk = ClockSampler(local)
    clk.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    cur = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    clk.mark(True)
    e0.record(cur)
    for _ in range(args.steps):
        one_step()
    e1.record(cur)
    torch.cuda.synchronize()
    clk.mark(False)
    barrier(world)
    ms = e0.elapsed_time(e1)
    ms_max = max_over_ranks(ms, world)
    if st.device_status() != 0:
        raise RuntimeError("device status not OK after the timed steps")
    value = replica_value(world, B, args.steps, ms_max)

    # ------------------------------------------------------------------ per-kernel timing
    kern = time_kernels(wl, st, args, dev, rows_distinct, hbm_gbs, tf_burst)
    step_roof_us = kern.pop("step_roofline_us")
    try:  # reported beside the step, never part of it; a failure here is recorded, not fatal
        kern["cache_append"] = time_cache_append(dev, hbm_gbs)
    except Exception as e:  # noqa: BLE001
        kern["cache_append"] = {"error": f"{type(e).__name__}: {e}"}
    try:
        kern["decompress_gate"] = time_gate(dev, hbm_gbs, tf_burst)
    except Exception as e:  # noqa: BLE001
        kern["decompress_gate"] = {"error": f"{type(e).__name__}: {e}"}
    configs = None
    if not args.no_configs:
        configs = time_configs(dev, hbm_gbs, tf_burst)
    clk.stop()
    clocks = clk.summary()

    # ------------------------------------------------------------------ e2e (host buffers)
    e2e = None if args.no_e2e else time_e2e(wl, st, args, dev, world)

    # dominant kernel: largest total time per step
    per_step = {
        "indexer": kern["indexer"]["us"] * N_FULL,
        "topk": kern["topk"]["us"] * N_FULL,
        "sparse_mla": kern["sparse_mla"]["us"] * L,
    }
    dom = max(per_step, key=per_step.get)
    roof = dict(kern[dom]["roofline"])
    roof["kernel"] = dom
    roof["traffic"] = load_traffic(dom)

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "layers": L, "full_layers": N_FULL, "schedule": wl.schedule,
                   "queries": B, "global_batch": B * world, "ctx": N, "indexer_heads": H_I, "d_I": D_I,
                   "topk": TOPK, "heads": H, "head_dim": D_QK, "parallelism": f"replicas{world}",
                   "graph": graph is not None,
                   "l2": "working set per step ~12.5 GB of KV/key caches > 126 MB L2; no flush needed"},
        "roofline": roof,
        "kernels": {k: {kk: vv for kk, vv in v.items()} for k, v in kern.items()},
        "kernel_share_of_step": {k: v / sum(per_step.values()) for k, v in per_step.items()},
        "step_roofline": {"us": step_roof_us, "ms_per_step": ms_max / args.steps,
                          "frac": step_roof_us / 1000.0 / (ms_max / args.steps),
                          "sum_of": "21 x (indexer + top-k) + 78 x sparse MLA, each max(bytes/HBM, FLOP/tensor) "
                                    "of measured peaks"},
        "peaks": {"hbm_gbs": hbm_gbs, "bf16_tflops": tf_burst, "kind": peak_kind},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if configs is not None:
        line["configs"] = configs
        ref = configs.get("single_F_B8_N131072_per_query_caches", {}).get("indexer")
        if ref and "roofline" in ref:
            line["indexer_hbm_128k"] = {"workload": "single_F_B8_N131072_per_query_caches", "gbs": ref["gbs"],
                                        "frac_of_hbm": ref["gbs"] / hbm_gbs, "us": ref["us"]}
    if rank == 0 and world == 1 and not args.no_configs:
        del st, graph, wl
        torch.cuda.empty_cache()
        line["reuse_overlap"] = reuse_diagnostic(dev)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tf, ta = cpu_sample_step()
        tf, ta = cpu_sample_step(seed=8)
        line["cpu_baseline"] = {
            "value": cpu_tokens_per_s(tf, ta), "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
            "sample": "1 query: indexer+top-k over N=131072 on 1 F layer + sparse MLA on 1 layer, "
                      "extrapolated to 21 F + 78 attention layers"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


# ----------------------------------------------------------------------------- ncu summaries
# Helpers for the committed profile notes (profiles/*.md): a per-kernel
# summary of an ncu launch list, and the DRAM traffic per launch of a kernel
# family recorded with the SHA-256 of its sources, which load_traffic reads
# back only while the sources are unchanged.
_NCU_UNIT = {"nsecond": 1e-3, "ns": 1e-3, "usecond": 1.0, "us": 1.0, "msecond": 1e3, "ms": 1e3, "second": 1e6}


def _ncu_rows(path):
    import csv
    rows = list(csv.reader(open(path)))
    hi = next(i for i, r in enumerate(rows) if "Kernel Name" in r)
    return rows[hi], rows[hi + 1:]


def _ncu_name(k):
    return k.split("(")[0].replace("void ", "").replace("(anonymous namespace)::", "")


def ncu_launches(path):
    """Per kernel of a gpu__time_duration.sum launch list: launches, total
    time, mean and share."""
    import collections
    h, body = _ncu_rows(path)
    ki, mi, vi, ui = (h.index(x) for x in ("Kernel Name", "Metric Name", "Metric Value", "Metric Unit"))
    agg = collections.defaultdict(lambda: [0, 0.0])
    for r in body:
        if len(r) <= vi or r[mi] != "gpu__time_duration.sum":
            continue
        name = _ncu_name(r[ki])
        agg[name][0] += 1
        agg[name][1] += float(r[vi].replace(",", "")) * _NCU_UNIT.get(r[ui], 1e-3)
    tot = sum(t for _, t in agg.values())
    print(f"{'kernel':58s} {'launches':>8s} {'total_us':>11s} {'mean_us':>9s} {'share':>6s}")
    for k, (n, t) in sorted(agg.items(), key=lambda x: -x[1][1]):
        print(f"{k[:58]:58s} {n:8d} {t:11.1f} {t / n:9.2f} {t / tot:6.3f}")


def sources_sha256(paths):
    import hashlib
    h = hashlib.sha256()
    for p in paths:
        h.update(open(os.path.join(ROOT, p), "rb").read())
    return h.hexdigest()


def ncu_traffic(path, name, regex, sources):
    """DRAM bytes (read + write) of one launch of each kernel matching regex,
    summed, as the traffic block load_traffic reads."""
    import collections
    import re
    h, body = _ncu_rows(path)
    ki, ii, mi, vi = (h.index(x) for x in ("Kernel Name", "ID", "Metric Name", "Metric Value"))
    per = collections.defaultdict(dict)
    kern = {}
    for r in body:
        if len(r) <= vi or not re.search(regex, r[ki]):
            continue
        per[r[ii]][r[mi]] = float(r[vi].replace(",", ""))
        kern[r[ii]] = _ncu_name(r[ki])
    first = {}
    for lid in sorted(per, key=int):
        first.setdefault(kern[lid], per[lid])
    total = sum(m.get("dram__bytes_read.sum", 0.0) + m.get("dram__bytes_write.sum", 0.0) for m in first.values())
    print(f"traffic-kernel: {name}")
    print(f"traffic-sources: {' '.join(sources)}")
    print(f"traffic-sha256: {sources_sha256(sources)}")
    print(f"traffic-dram-bytes-per-launch: {int(total)}")
    for k, m in first.items():
        print(f"traffic-part: {k} read {int(m.get('dram__bytes_read.sum', 0))} write "
              f"{int(m.get('dram__bytes_write.sum', 0))}")


def load_traffic(kernel):
    """DRAM bytes per launch from the committed ncu summary under profiles/,
    if one was taken on the current kernel sources; else None."""
    import re
    pdir = os.path.join(ROOT, "profiles")
    if not os.path.isdir(pdir):
        return None
    for fn in sorted(os.listdir(pdir)):
        if not fn.endswith(".md"):
            continue
        kv = dict(re.findall(r"^traffic-([a-z0-9-]+):\s*(.+)$", open(os.path.join(pdir, fn)).read(), flags=re.M))
        if kv.get("kernel") != kernel or "dram-bytes-per-launch" not in kv:
            continue
        try:
            if sources_sha256(kv["sources"].split()) != kv["sha256"].strip():
                continue
        except OSError:
            continue
        return int(kv["dram-bytes-per-launch"])
    return None


# ----------------------------------------------------------------------------- one kernel family, for profiling
DRIVER_SHAPES = {
    "stack": dict(B=32, N=131072, shared=True),     # one layer of the 78-layer stack
    "single": dict(B=8, N=131072, shared=False),    # the single F layer, per-query caches
    "long": dict(B=4, N=262144, shared=False),      # the long-context shape at a quarter of its length
    "prefill": dict(B=256, N=264192, shared=True),  # 256 rows of the prefill chunk
}


def kernel_driver(kernel, shape, fp8, warmup, iters):
    """Run one kernel family on a fixed shape: `warmup` untimed launches,
    then `iters` timed ones (for ncu -k <kernel> -s <warm-up launches>)."""
    import torch
    from lightning_indexer_cross_b200 import _abi, ops
    from lightning_indexer_cross_b200 import workloads as W
    sh = DRIVER_SHAPES[shape]
    dev = torch.device("cuda:0")
    Bq, Nk, shared = sh["B"], sh["N"], sh["shared"]
    K = TOPK
    if kernel == "gate":
        o, wv, gl = W.gate_case(Bq, H, seed=90, device=dev)
        ws = ops.new_workspace(_abi.ic_decompress_gate_workspace_size(), dev)
        fn = lambda: ops.decompress_gate(o, wv, gl, workspace=ws)
    elif kernel == "append":
        # Bq new tokens into an Nk-row shared cache, Bq queries' rotary dims
        c = W.append_case(Bq, Nk, D_I, per_token=False, fp8=fp8, B=Bq, H=H, seed=70, device=dev)
        ws = ops.new_workspace(_abi.ic_cache_append_workspace_size(), dev)
        fn = lambda: ops.cache_append(c["k_raw"], c["gamma"], c["beta"], c["kv_raw"], c["pos"], c["key_cache"],
                                      c["kv_cache"], key_scale=c.get("key_scale"), q=c["q"], q_pos=c["q_pos"],
                                      workspace=ws)
    else:
        q, w, k, ks, _ = W.indexer_case(Bq, Nk, H_I, D_I, shared=shared, fp8=fp8, seed=5, device=dev)
        scores = ops.indexer_score(q, w, k, ks)
        idx = ops.topk(scores, K)
        torch.cuda.synchronize()
        if kernel == "indexer":
            ws = ops.new_workspace(256, dev)
            fn = lambda: ops.indexer_score(q, w, k, ks, scores=scores, workspace=ws)
        elif kernel == "topk":
            ws = ops.new_workspace(_abi.ic_topk_workspace_size(Bq, Nk, K), dev)
            fn = lambda: ops.topk(scores, K, idx=idx, workspace=ws)
        else:
            g = torch.Generator(device=dev).manual_seed(6)
            qa = torch.randn((Bq, H, W.D_QK), generator=g, device=dev).to(torch.bfloat16)
            kv = torch.randn((1 if shared else Bq, Nk, W.D_QK), generator=g, device=dev).to(torch.bfloat16)
            sink = torch.randn((H,), generator=g, device=dev) * 0.5
            gate = torch.randn((Bq, H, W.D_LATENT), generator=g, device=dev).to(torch.bfloat16)
            out = torch.empty((Bq, H, W.D_LATENT), dtype=torch.bfloat16, device=dev)
            ws = ops.new_workspace(_abi.ic_sparse_mla_workspace_size(Bq, H, K), dev)
            fn = lambda: ops.sparse_mla_decode(qa, kv, idx, sink, gate, out=out, want_lse=False, workspace=ws)
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        fn()
    e1.record()
    torch.cuda.synchronize()
    print(f"{kernel} {shape}{' fp8' if fp8 else ''}: {e0.elapsed_time(e1) * 1000 / max(iters, 1):.2f} us/call")
    return 0


def _time_loop(fn, n, stream, replays=3):
    """Capture n calls of fn in a CUDA graph (so host launch cost cannot hide
    in the number), replay it, and return the mean device time per call (us)
    measured with events on the stream the kernels run on."""
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(n):
            fn(i)
    g.replay()
    torch.cuda.synchronize()
    cur = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(cur)
    for _ in range(replays):
        g.replay()
    e1.record(cur)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1000.0 / (n * replays)  # us


def roofline_time_us(bytes_, flops, hbm_gbs, tf_peak):
    """The kernel's roofline time: the slower of moving its algorithmic bytes
    at the HBM peak and doing its FLOPs at the tensor peak."""
    return max(bytes_ / (hbm_gbs * 1e9), flops / (tf_peak * 1e12)) * 1e6


def roofline_of(bytes_, flops, us, hbm_gbs, tf_peak):
    """Achieved rate against the bound that sets the kernel's roofline."""
    t_hbm = bytes_ / (hbm_gbs * 1e9)
    t_tc = flops / (tf_peak * 1e12)
    if t_tc > t_hbm:
        ach = flops / (us * 1e-6) / 1e12
        return {"bound": "tensor", "achieved": ach, "peak": tf_peak, "unit": "TFLOP/s",
                "frac": ach / tf_peak, "algorithmic_flops": flops, "algorithmic_bytes": bytes_}
    ach = bytes_ / (us * 1e-6) / 1e9
    return {"bound": "hbm", "achieved": ach, "peak": hbm_gbs, "unit": "GB/s", "frac": ach / hbm_gbs,
            "algorithmic_bytes": bytes_, "algorithmic_flops": flops}


def indexer_work(B, N, H_I, d_I, key_bytes_per_token, shared):
    """Algorithmic bytes and FLOPs of one indexer call: every key read once
    (once per query with per-query caches), queries and weights, the score
    row written."""
    keys = N * key_bytes_per_token * (1 if shared else B)
    return keys + B * H_I * d_I * 2 + B * H_I * 4 + B * N * 4, 2.0 * B * H_I * d_I * N


def topk_work(B, N, k):
    return B * N * 4 + B * k * 4


def mla_work(rows, B, H, k, gate):
    """Gathered rows once each, q, the output (and gate) once, the indices."""
    return (rows * D_QK * 2 + B * H * D_QK * 2 + B * H * D_V * 2 * (2 if gate else 1) + B * k * 4,
            2.0 * B * H * k * (D_QK + D_V))


def reuse_diagnostic(dev):
    """Recall of the reused index on every S layer of the stack (outside the
    timed region): the overlap of the last F layer's top-k with the top-k the
    S layer would compute from indexer inputs of its own, over k. Two key
    recipes: independent keys per layer (the stack's; recall ~ k/N by
    construction) and one key cache for all layers (the queries' layer-to-
    layer correlation rho = 0.8 is then what the reuse keeps)."""
    import torch
    from lightning_indexer_cross_b200 import ops
    from lightning_indexer_cross_b200 import workloads as W
    out = {"what": "overlap of the reused index with the S layer's own top-k, / k (mean over queries)"}
    for keys in ("per_layer", "shared"):
        wl = W.stack(dev, seed=replica_seed(0), L=L, n_full=N_FULL, B=B, N=N, H_I=H_I, d_I=D_I, topk=TOPK, H=H,
                     gate=False, s_indexers=True, layer_keys=keys)
        for lay in wl.layers:  # only the indexer inputs are used
            lay.kv = lay.q = None
        torch.cuda.empty_cache()
        got = ops.reuse_overlap(wl.layers, wl.schedule, wl.topk)
        torch.cuda.synchronize()
        gov, last = [], -1
        for l, c in enumerate(wl.schedule):
            last = l if c == "F" else last
            gov.append(last)
        rec = {l: float(v.double().mean().item()) / wl.topk for l, v in got.items()}
        by_d = {}
        for l, r in rec.items():
            by_d.setdefault(l - gov[l], []).append(r)
        vals = list(rec.values())
        out[keys + "_keys"] = {"s_layers": len(vals), "recall_mean": sum(vals) / len(vals), "recall_min": min(vals),
                               "recall_max": max(vals),
                               "recall_by_distance": {str(d): sum(v) / len(v) for d, v in sorted(by_d.items())}}
        del wl, got
        torch.cuda.empty_cache()
    return out


def time_configs(dev, hbm_gbs, tf_burst):
    """The other workloads' kernels, each timed alone (graph of n launches,
    CUDA events on its stream): the single F layer at model shape (8 queries,
    per-query caches of 131072 tokens), the 1M-token context (4 queries,
    bf16 and e4m3 keys) and the prefill chunk (2048 causal queries over
    264192 tokens). Inputs are larger than L2 except where noted."""
    import gc
    import torch
    from lightning_indexer_cross_b200 import _abi, ops
    from lightning_indexer_cross_b200 import workloads as W
    stream = torch.cuda.Stream(device=dev)
    res = {}

    def leg(wl, n_ind, n_mla, rows_per_pass=None):
        lay = wl.layers[0]
        B, N = wl.B, wl.N
        scores = torch.empty((B, N), dtype=torch.float32, device=dev)
        idx = torch.empty((B, wl.topk), dtype=torch.int32, device=dev)
        out = torch.empty((B, wl.H, D_V), dtype=torch.bfloat16, device=dev)
        ws_i = ops.new_workspace(_abi.ic_indexer_workspace_size(), dev)
        ws_t = ops.new_workspace(_abi.ic_topk_workspace_size(B, N, wl.topk), dev)
        ws_m = ops.new_workspace(_abi.ic_sparse_mla_workspace_size(B, wl.H, wl.topk), dev)

        def ind(i):
            ops.indexer_score(lay.q_idx, lay.w, lay.k_idx, lay.k_scale, wl.n_valid, scores=scores, workspace=ws_i)

        def tk(i):
            ops.topk(scores, wl.topk, wl.n_valid, idx=idx, workspace=ws_t)

        def mla(i):
            ops.sparse_mla_decode(lay.q, lay.kv, idx, lay.sink, lay.gate, sm_scale=wl.sm_scale, out=out,
                                  want_lse=False, workspace=ws_m)

        ind(0)
        tk(0)
        mla(0)
        torch.cuda.synchronize()
        rows = 0
        kvb = lay.kv.shape[0]
        for b in range(B):
            sel = idx[b][idx[b] >= 0]
            rows += int(sel.numel()) if kvb > 1 else 0
        if kvb == 1:
            rows = int(torch.unique(idx[idx >= 0]).numel())
        t_i = _time_loop(ind, n_ind, stream)
        t_t = _time_loop(tk, n_ind, stream)
        t_m = _time_loop(mla, n_mla, stream)
        fused = {}
        if rows_per_pass is not None:
            ws_f = ops.new_workspace(_abi.ic_indexer_topk_workspace_size(B, N, wl.topk, rows_per_pass), dev)

            def fz(i):
                ops.indexer_topk(lay.q_idx, lay.w, lay.k_idx, wl.topk, lay.k_scale, wl.n_valid,
                                 rows_per_pass=rows_per_pass, idx=idx, workspace=ws_f)

            fz(0)
            torch.cuda.synchronize()
            t_f = _time_loop(fz, n_ind, stream)
            fused = {"indexer_topk": {"us": t_f, "rows_per_pass": rows_per_pass,
                                      "score_scratch_bytes": int(ws_f.numel())}}
            del ws_f
        if _abi.ic_last_device_status(ops._ptr(ws_i), ops._stream_ptr()) != _abi.IC_OK:
            raise RuntimeError("device status not OK")
        kb = (wl.d_I + 4) if wl.k_fp8 else wl.d_I * 2
        ib, iflops = indexer_work(B, N, wl.H_I, wl.d_I, kb, wl.shared_keys)
        if wl.n_valid is not None:  # causal: only the visible keys are scored
            nv = wl.n_valid.double()
            iflops = 2.0 * wl.H_I * wl.d_I * float(nv.sum())
        mb, mflops = mla_work(rows, B, wl.H, wl.topk, lay.gate is not None)
        return {
            "indexer": {"us": t_i, "gbs": ib / (t_i * 1e-6) / 1e9,
                        "roofline": roofline_of(ib, iflops, t_i, hbm_gbs, tf_burst)},
            "topk": {"us": t_t, "elems_per_s": B * N / (t_t * 1e-6),
                     "roofline": roofline_of(topk_work(B, N, wl.topk), 0.0, t_t, hbm_gbs, tf_burst)},
            "sparse_mla": {"us": t_m, "gathered_rows": rows,
                           "roofline": roofline_of(mb, mflops, t_m, hbm_gbs, tf_burst)},
            **fused,
        }

    cases = [
        ("single_F_B8_N131072_per_query_caches", lambda: W.single_f(dev), 6, 6, None),
        ("long_ctx_B4_N1048576_bf16", lambda: W.long_context(dev, fp8=False), 3, 6, None),
        ("long_ctx_B4_N1048576_e4m3", lambda: W.long_context(dev, fp8=True), 3, 6, None),
        ("prefill_C2048_P262144_causal", lambda: W.prefill(dev), 2, 2, 128),
    ]
    for name, make, n_ind, n_mla, rpp in cases:
        try:
            wl = make()
            torch.cuda.synchronize()
            res[name] = leg(wl, n_ind, n_mla, rpp)
        except Exception as e:  # noqa: BLE001  (recorded, not fatal: the headline step is measured above)
            res[name] = {"error": f"{type(e).__name__}: {e}"}
        wl = None
        gc.collect()
        torch.cuda.empty_cache()
    return res


def time_gate(dev, hbm_gbs, tf_burst):
    """The decompressed-space gate after each layer's attention at the
    stack's decode shape (32 queries, 128 heads, d_v 128): 16 weight sets
    rotated (269 MB, more than L2), one launch per layer in a graph."""
    import torch
    from lightning_indexer_cross_b200 import _abi, ops
    from lightning_indexer_cross_b200 import workloads as Wl
    stream = torch.cuda.Stream(device=dev)
    sets = [Wl.gate_case(B, H, seed=90 + i, device=dev) for i in range(16)]
    ws = ops.new_workspace(_abi.ic_decompress_gate_workspace_size(), dev)
    out = torch.empty((B, H, 128), dtype=torch.bfloat16, device=dev)

    def g(i):
        o, w, gl = sets[i % len(sets)]
        ops.decompress_gate(o, w, gl, out=out, workspace=ws)

    for i in range(3):
        g(i)
    torch.cuda.synchronize()
    us = _time_loop(g, L, stream)
    if _abi.ic_last_device_status(ops._ptr(ws), ops._stream_ptr()) != _abi.IC_OK:
        raise RuntimeError("device status not OK after the gate launches")
    bytes_ = H * 128 * D_V * 2 + B * H * D_V * 2 + B * H * 128 * 2 * 2
    flops = 2.0 * B * H * 128 * D_V
    return {"us": us, "launches": L, "roofline": roofline_of(bytes_, flops, us, hbm_gbs, tf_burst)}


def time_kernels(wl, st, args, dev, rows_distinct, hbm_gbs, tf_burst):
    """Each kernel family alone, on the stream it is launched on, rotating over
    the layers' own inputs (so each launch streams fresh data from HBM)."""
    import torch
    from lightning_indexer_cross_b200 import _abi, ops
    stream = torch.cuda.Stream(device=dev)
    f_layers = [l for l in range(wl.L) if wl.schedule[l] == "F"]
    scores = torch.empty((B, N), dtype=torch.float32, device=dev)
    ws_i = ops.new_workspace(_abi.ic_indexer_workspace_size(), dev)
    ws_t = ops.new_workspace(_abi.ic_topk_workspace_size(B, N, TOPK), dev)
    ws_m = ops.new_workspace(_abi.ic_sparse_mla_workspace_size(B, H, TOPK), dev)
    idx = torch.empty((B, TOPK), dtype=torch.int32, device=dev)
    out = torch.empty((B, H, D_V), dtype=torch.bfloat16, device=dev)
    reps = 2 * len(f_layers)

    def ind(i):
        lay = wl.layers[f_layers[i % len(f_layers)]]
        ops.indexer_score(lay.q_idx, lay.w, lay.k_idx, None, None, scores=scores, workspace=ws_i)

    def tk(i):
        ops.topk(scores, TOPK, None, idx=idx, workspace=ws_t)

    idx_by_layer = []
    for l in f_layers:
        ind_l = f_layers.index(l)
        ind(ind_l)
        tk(0)
        idx_by_layer.append(idx.clone())

    def mla(i):
        l = i % wl.L
        lay = wl.layers[l]
        gi = [j for j in range(len(f_layers)) if f_layers[j] <= l][-1]
        ops.sparse_mla_decode(lay.q, lay.kv, idx_by_layer[gi], lay.sink, lay.gate, out=out, want_lse=False,
                              workspace=ws_m)

    ws_f = ops.new_workspace(_abi.ic_indexer_topk_workspace_size(B, N, TOPK, 0), dev)
    idx_f = torch.empty((B, TOPK), dtype=torch.int32, device=dev)

    def fused(i):
        lay = wl.layers[f_layers[i % len(f_layers)]]
        ops.indexer_topk(lay.q_idx, lay.w, lay.k_idx, TOPK, idx=idx_f, workspace=ws_f)

    for fn in (ind, tk, mla, fused):
        for i in range(3):
            fn(i)
    torch.cuda.synchronize()
    t_fused = _time_loop(fused, reps, stream)
    t_ind = _time_loop(ind, reps, stream)
    # top-k reads scores written just before (as in the stack); time it alone
    t_tk = _time_loop(tk, reps, stream)
    t_mla = _time_loop(mla, wl.L, stream)

    # algorithmic work per launch
    ind_bytes, ind_flops = indexer_work(B, N, H_I, D_I, D_I * 2, True)
    tk_bytes = topk_work(B, N, TOPK)
    mla_rows = rows_distinct / wl.L
    mla_bytes, mla_flops = mla_work(mla_rows, B, H, TOPK, True)

    def roofline(bytes_, flops, us):
        return roofline_of(bytes_, flops, us, hbm_gbs, tf_burst)

    step_roof_us = (N_FULL * (roofline_time_us(ind_bytes, ind_flops, hbm_gbs, tf_burst) +
                              roofline_time_us(tk_bytes, 0.0, hbm_gbs, tf_burst)) +
                    L * roofline_time_us(mla_bytes, mla_flops, hbm_gbs, tf_burst))
    return {
        "step_roofline_us": step_roof_us,
        "indexer_topk": {"us": t_fused, "launches": reps,
                         "what": "ic_indexer_topk per F layer (indexer and top-k in one call)",
                         "roofline": roofline(ind_bytes + tk_bytes, ind_flops, t_fused)},
        "indexer": {"us": t_ind, "launches": reps, "gbs": ind_bytes / (t_ind * 1e-6) / 1e9,
                    "roofline": roofline(ind_bytes, ind_flops, t_ind)},
        "topk": {"us": t_tk, "launches": reps, "elems_per_s": B * N / (t_tk * 1e-6),
                 "roofline": roofline(tk_bytes, 0.0, t_tk)},
        "sparse_mla": {"us": t_mla, "launches": wl.L, "gbs": mla_bytes / (t_mla * 1e-6) / 1e9,
                       "distinct_rows_per_layer": mla_rows,
                       "roofline": roofline(mla_bytes, mla_flops, t_mla)},
    }


def time_cache_append(dev, hbm_gbs):
    """The cache-append step that precedes each decode step (not inside the
    step's timed region): one launch per layer writes the 32 queries' new
    tokens into a 131072-row shared cache (bf16 LayerNorm'd keys, latent rows
    with rotated rotary dims) and rotates the 32 queries' rotary dims, timed
    like the other kernels (graph of L launches, events on their stream)."""
    import torch
    from lightning_indexer_cross_b200 import _abi, ops, workloads as Wl
    stream = torch.cuda.Stream(device=dev)
    c = Wl.append_case(B, N, D_I, per_token=False, fp8=False, B=B, H=H, seed=70, device=dev)
    ws = ops.new_workspace(_abi.ic_cache_append_workspace_size(), dev)

    def app(i):
        ops.cache_append(c["k_raw"], c["gamma"], c["beta"], c["kv_raw"], c["pos"], c["key_cache"], c["kv_cache"],
                         q=c["q"], q_pos=c["q_pos"], workspace=ws)

    for i in range(3):
        app(i)
    torch.cuda.synchronize()
    us = _time_loop(app, L, stream)
    if _abi.ic_last_device_status(ops._ptr(ws), ops._stream_ptr()) != _abi.IC_OK:
        raise RuntimeError("device status not OK after the cache-append launches")
    # algorithmic bytes per launch: key rows in and out, latent rows in and
    # out, the queries' rotary dims in and out, LayerNorm parameters, rows
    bytes_ = (B * (D_I * 2 * 2 + D_QK * 2 * 2) + B * H * (D_QK - D_V) * 2 * 2 + 2 * D_I * 4 + 2 * B * 8)
    ach = bytes_ / (us * 1e-6) / 1e9
    return {"us": us, "launches": L, "tokens_per_launch": B,
            "roofline": {"bound": "hbm", "achieved": ach, "peak": hbm_gbs, "unit": "GB/s", "frac": ach / hbm_gbs,
                         "algorithmic_bytes": bytes_, "algorithmic_flops": 0.0}}


def time_e2e(wl, st, args, dev, world):
    """Same metric through the public call with host buffers: per step, the
    per-layer queries (indexer q and weights on F layers, attention q and gate
    on every layer) are copied from pinned host memory on a copy stream, one
    event per layer; the stack waits on layer l's event before layer l (so
    layer l runs while later layers' inputs are still being copied), and the
    last layer's attention output is read back to the host. Two sets of
    device input buffers (two stacks over the same caches) alternate between
    steps, so one step's copies overlap the previous step's compute; a set is
    refilled only after the step that last read it has finished."""
    import dataclasses
    import torch
    from lightning_indexer_cross_b200 import ops
    names = ("q_idx", "w", "q", "gate")
    layers2 = [dataclasses.replace(lay, **{n: (torch.empty_like(getattr(lay, n)) if getattr(lay, n) is not None
                                               else None) for n in names})
               for lay in wl.layers]
    st2 = ops.stack_from_workload(dataclasses.replace(wl, layers=layers2), trace=False)
    stacks = [(st, wl.layers), (st2, layers2)]
    hosts = []
    h2d = 0
    for lay in wl.layers:
        hs = []
        for n in names:
            t = getattr(lay, n)
            hs.append(None if t is None else t.detach().cpu().pin_memory())
            if t is not None:
                h2d += t.numel() * t.element_size()
        hosts.append(hs)
    out_host = torch.empty(st.outs[-1].shape, dtype=st.outs[-1].dtype).pin_memory()
    d2h = out_host.numel() * out_host.element_size()
    compute = torch.cuda.current_stream()
    copies = [torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)]  # layers alternate
    ready = [[torch.cuda.Event() for _ in wl.layers] for _ in stacks]
    done = [torch.cuda.Event() for _ in stacks]
    for i, (s_i, _) in enumerate(stacks):
        s_i.set_wait_events(ready[i])
        done[i].record(compute)
    counter = [0]

    def step():
        i = counter[0] & 1
        counter[0] += 1
        s_i, lays = stacks[i]
        for c in copies:
            c.wait_event(done[i])  # the step that last read this input set has finished
        for l, lay in enumerate(lays):
            c = copies[l & 1]
            with torch.cuda.stream(c):
                for n, h in zip(names, hosts[l]):
                    if h is not None:
                        getattr(lay, n).copy_(h, non_blocking=True)
                ready[i][l].record(c)
        s_i.step(stream=compute)
        out_host.copy_(s_i.outs[-1], non_blocking=True)
        done[i].record(compute)

    n = max(3, min(args.steps, 20))
    for _ in range(2):
        step()
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(compute)
    for _ in range(n):
        step()
    e1.record(compute)
    torch.cuda.synchronize()
    for s_i, _ in stacks:
        s_i.set_wait_events(None)
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    return {"value": world * B * n / (ms / 1000.0), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": n,
            "overlap": "per-layer input copies on two copy streams, two input buffer sets alternating",
            "note": "the per-layer queries, weights and gates are uploaded every step because the path starts at "
                    "them; a model computes them on the device from one hidden state per token (which the pages "
                    "do not size), so its step would move far fewer host bytes and run at about the device-"
                    "resident value"}


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip timing the other workloads' kernels")
    ap.add_argument("--warmup-ref", type=int, default=1)
    ap.add_argument("--kernel-driver", choices=["indexer", "topk", "mla", "gate", "append"],
                    help="run one kernel family on --shape instead (for ncu): --warmup untimed, --steps timed")
    ap.add_argument("--shape", choices=list(DRIVER_SHAPES), default="stack")
    ap.add_argument("--fp8", action="store_true", help="e4m3 keys for --kernel-driver")
    ap.add_argument("--ncu-launches", metavar="CSV", help="summarise an ncu launch list and exit")
    ap.add_argument("--ncu-traffic", nargs="+", metavar="ARG",
                    help="CSV NAME REGEX SOURCE...: the DRAM traffic block of a kernel family, then exit")
    args = ap.parse_args()
    if args.ncu_launches:
        ncu_launches(args.ncu_launches)
        return 0
    if args.ncu_traffic:
        ncu_traffic(args.ncu_traffic[0], args.ncu_traffic[1], args.ncu_traffic[2], args.ncu_traffic[3:])
        return 0
    if args.kernel_driver:
        return kernel_driver(args.kernel_driver, args.shape, args.fp8, args.warmup, args.steps)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_native(args)


if __name__ == "__main__":
    sys.exit(main())
