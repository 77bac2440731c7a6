#!/usr/bin/env python
"""Benchmark of the DSA decode/verify step (indexer scan -> causal top-k ->
sparse GQA attention) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

A step is one full pass of the path over one batch of synthetic inputs that are
resident in HBM.  Each timed step starts with a cold L2 (a write of twice the L2
size runs before it, outside the timed region) and is replayed from a CUDA graph
of dsa_decode_ws; its time is taken with CUDA events on the launching stream.
`value` is algorithmic HBM bytes per step (indexer keys, unique selected K/V
rows, queries, outputs, indices) over the step time, summed over ranks.  With
N > 1 every rank runs an independent replica (the step has no data-path
exchange on one GPU) and the time is the max over ranks.

--impl reference times the CPU oracle (test infrastructure, fp64) on the host
cores on the same workload and prints the same line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from sparse_attention_decode_relu_b200 import synth  # noqa: E402

METRIC = "µs per DSA decode/verify step and achieved HBM GB/s (% of B200 peak) vs context L"
KEY_BYTES = {"bf16": 128, "fp8": 68}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def algorithmic_bytes(w, sel):
    """Bytes the method must move per step: the indexer key cache up to the
    furthest visible position, each unique selected K/V row once, per-query
    inputs and outputs."""
    n_max = int(w.pos.max()) + 1
    uniq = np.unique(sel[sel >= 0]).size
    per_query = 64 * 128 * 2 + 16 * 64 * 2 + 16 * 4 + 64 * 128 * 2 + 4 * w.topk
    return {
        "indexer": n_max * KEY_BYTES[w.key_dtype],
        "attention": uniq * 2048 + w.T * (64 * 128 * 2 + 4 * w.topk),
        "step": n_max * KEY_BYTES[w.key_dtype] + uniq * 2048 + w.T * per_query,
        "unique_rows": uniq,
        "gathered_rows": int((sel >= 0).sum()),
    }


class Clocks:
    """nvidia-smi sampler running during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.p = None
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(index), "--query-gpu=" + self.FIELDS,
                                       "--format=csv,noheader,nounits", "-lms", "100"],
                                      stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.p = None

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        out, _ = self.p.communicate(timeout=10)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 7:
                continue
            try:
                sm.append(float(f[0]))
                mx = float(f[1])
            except ValueError:
                continue
            for n, v in zip(names, f[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(n):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n:
        raise SystemExit(f"--gpus {n} but WORLD_SIZE={world}")
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def reduce_max(x, world):
    if world == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
    torch.cuda.synchronize()


def cpu_baseline(w, budget_s=15.0):
    """The oracle as it stands, on this host's cores, over whole steps of the same
    workload until about budget_s seconds have passed."""
    import oracle

    kv = w.kv
    times = []
    t_end = time.perf_counter() + budget_s
    while True:
        t0 = time.perf_counter()
        _, sel = oracle.decode(w.q, w.q_idx, w.w_idx, w.k_idx, w.k_scale, kv, w.pos, w.topk)
        times.append(time.perf_counter() - t0)
        if time.perf_counter() > t_end or len(times) >= 50:
            break
    return statistics.median(times), len(times), sel, oracle.threads()


def run_reference(args, w, rank, world):
    if rank != 0:
        return
    import oracle

    kv = w.kv
    for _ in range(args.warmup):
        oracle.decode(w.q, w.q_idx, w.w_idx, w.k_idx, w.k_scale, kv, w.pos, w.topk)
    times = []
    sel = None
    for _ in range(args.steps):
        t0 = time.perf_counter()
        _, sel = oracle.decode(w.q, w.q_idx, w.w_idx, w.k_idx, w.k_scale, kv, w.pos, w.topk)
        times.append(time.perf_counter() - t0)
    ab = algorithmic_bytes(w, sel)
    t = statistics.mean(times)
    value = ab["step"] / t / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t * 1e3, 3), "us_per_step": round(t * 1e6, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "L": w.L, "T": w.T, "topk": w.topk, "key_dtype": w.key_dtype,
                   "recipe": w.recipe, "seed": w.seed},
        "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": oracle.threads(), "kind": "oracle",
                         "sample": f"whole steps of {w.name} (fp64 C oracle, OpenMP), {args.steps} timed"},
        "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="verify_block")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    w = synth.config(args.config)

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, w, rank, int(os.environ.get("WORLD_SIZE", "1")))
        return

    from sparse_attention_decode_relu_b200 import dsa

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    d = dsa.to_device(w, device=dev)
    T, L, topk = w.T, w.L, w.topk
    ws = dsa.workspace(T, L, topk, device=dev)
    out = torch.empty((T, 64, 128), dtype=torch.bfloat16, device=dev)
    sel = torch.empty((T, topk), dtype=torch.int32, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]

    def step():
        dsa.dsa_decode_ws(d["q"], d["q_idx"], d["w_idx"], d["k_idx"], d["kv"], d["pos"], topk, out, sel, ws,
                          k_scale=d["k_scale"])

    # One eager call counts the kernels of a step; then capture the step (with its
    # stage events) into a graph.
    with torch.cuda.stream(stream):
        n0 = dsa.dsa_launch_count()
        step()
        kernels_per_step = dsa.dsa_launch_count() - n0
    stream.synchronize()
    dsa.dsa_device_status(stream)
    # torch only reports elapsed time for events it has recorded itself once.
    for e in ev:
        e.record(stream)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()

    def timed_step():
        """Cold L2, then one graph replay of the whole step, timed by events."""
        flush.zero_()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            stream.wait_stream(torch.cuda.current_stream())
            s0.record(stream)
            graph.replay()
            s1.record(stream)
        stream.synchronize()
        return s0.elapsed_time(s1)

    def staged_step():
        """Cold L2, then the step launched eagerly with an event after every kernel.
        A spin on the stream first lets the host enqueue all launches, so the
        gaps between events are device time only."""
        flush.zero_()
        with torch.cuda.stream(stream):
            stream.wait_stream(torch.cuda.current_stream())
            torch.cuda._sleep(200000)
            dsa.dsa_set_stage_events(ev)
            step()
            dsa.dsa_set_stage_events(None)
        stream.synchronize()
        return [ev[i].elapsed_time(ev[i + 1]) for i in range(4)] + [ev[0].elapsed_time(ev[4])]

    for _ in range(args.warmup):
        timed_step()
        staged_step()
    barrier(world)
    clocks = Clocks(local)
    totals, stage_sum = [], [0.0] * 5
    for _ in range(args.steps):
        totals.append(timed_step())
    for _ in range(args.steps):
        stage_sum = [a + b for a, b in zip(stage_sum, staged_step())]
    barrier(world)
    clk = clocks.stop()
    dsa.dsa_device_status(stream)
    ms = reduce_max(statistics.mean(totals), world)
    stage_ms = [s / args.steps for s in stage_sum[:4]]
    eager_ms = stage_sum[4] / args.steps

    sel_np = sel.cpu().numpy()
    ab = algorithmic_bytes(w, sel_np)
    value = world * ab["step"] / (ms * 1e-3) / 1e9

    # End to end through the public API: per step the query-side inputs come from
    # pinned host memory and the outputs go back to it; the caches stay resident.
    h_in = {k: d[k].cpu().pin_memory() for k in ("q", "q_idx", "w_idx")}
    dev_in = {k: torch.empty_like(d[k]) for k in h_in}
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h_sel = torch.empty(sel.shape, dtype=sel.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in h_in.values())
    d2h = h_out.numel() * h_out.element_size() + h_sel.numel() * h_sel.element_size()

    def e2e_step():
        with torch.cuda.stream(stream):
            for k in h_in:
                dev_in[k].copy_(h_in[k], non_blocking=True)
            dsa.dsa_decode_ws(dev_in["q"], dev_in["q_idx"], dev_in["w_idx"], d["k_idx"], d["kv"], d["pos"], topk,
                              out, sel, ws, k_scale=d["k_scale"])
            h_out.copy_(out, non_blocking=True)
            h_sel.copy_(sel, non_blocking=True)

    for _ in range(args.warmup):
        e2e_step()
    stream.synchronize()
    e_times = []
    for _ in range(args.steps):
        flush.zero_()
        torch.cuda.current_stream().synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        e2e_step()
        b.record(stream)
        stream.synchronize()
        e_times.append(a.elapsed_time(b))
    e_ms = reduce_max(statistics.mean(e_times), world)
    e2e = {"value": round(world * ab["step"] / (e_ms * 1e-3) / 1e9, 3), "unit": "GB/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e_ms, 4)}

    # Roofline of the dominant kernel (largest share of the step).
    names = ["indexer", "topk", "attention", "tail"]
    dom = int(np.argmax(stage_ms))
    peak, which = peaks()
    alg = {"indexer": ab["indexer"], "attention": ab["attention"]}
    roof = None
    if names[dom] in alg:
        achieved = alg[names[dom]] / (stage_ms[dom] * 1e-3) / 1e9
        roof = {"kernel": names[dom], "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "peak_source": which, "traffic": None,
                "algorithmic_bytes": alg[names[dom]]}
    else:
        roof = {"kernel": names[dom], "bound": "hbm", "achieved": None, "peak": peak, "unit": "GB/s", "frac": None,
                "peak_source": which, "traffic": None}

    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 5), "us_per_step": round(ms * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "L": L, "T": T, "topk": topk, "key_dtype": w.key_dtype, "recipe": w.recipe,
                   "seed": w.seed, "parallelism": f"replicas{world}", "l2": "flushed before every step",
                   "timing": "CUDA-graph replay of dsa_decode_ws, CUDA events per step",
                   "algorithmic_bytes_per_step": ab["step"], "unique_kv_rows": ab["unique_rows"],
                   "gathered_kv_rows": ab["gathered_rows"]},
        "frac_of_peak_hbm": round(ab["step"] / (ms * 1e-3) / 1e9 / peak, 4),
        "stage_us": {n: round(s * 1e3, 2) for n, s in zip(names, stage_ms)},
        "eager_us_per_step": round(eager_ms * 1e3, 2),
        "roofline": roof,
        "e2e": e2e,
        "gpu_launches": int(kernels_per_step * args.steps),
        "clocks": clk,
    }
    if rank == 0 and not args.no_cpu_baseline:
        t_cpu, n_cpu, _, cores = cpu_baseline(w, args.cpu_budget)
        line["cpu_baseline"] = {"value": round(ab["step"] / t_cpu / 1e9, 4), "unit": "GB/s", "cores": cores,
                                "kind": "oracle", "us_per_step": round(t_cpu * 1e6, 1),
                                "sample": f"{n_cpu} whole steps of {w.name}, median"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()
