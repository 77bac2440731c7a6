#!/usr/bin/env python
"""Benchmark of the DSA decode/verify step (indexer scan -> causal top-k ->
sparse GQA attention) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

A step is one full pass of the path over one batch of synthetic inputs that are
resident in HBM.  Each timed step starts with a cold L2 (outside the timed
region a buffer of twice the L2 size is written, then another one is read, so no
dirty lines of the flush are left to write back) and is replayed from a CUDA graph
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
SPIN_CYCLES = 200_000   # ~0.1 ms of GPU-side spin before each timed region
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from sparse_attention_decode_relu_b200 import synth  # noqa: E402

METRIC = "µs per DSA decode/verify step and achieved HBM GB/s (% of B200 peak) vs context L"
KEY_BYTES = {"bf16": 128, "fp8": 68}


def source_code_only(src: str) -> str:
    """C/C++ source without its comments, blank space collapsed; string and
    character literals are kept as written."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_sources_sha256():
    """sha256 over the sorted file names and the code of the CUDA sources
    (comments and blank space removed: a comment edit leaves a capture's record
    valid, any change to the code does not)."""
    import hashlib
    d = os.path.join(ROOT, "sparse_attention_decode_relu_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(os.listdir(d)):
        h.update(f.encode())
        with open(os.path.join(d, f), encoding="utf-8") as fh:
            h.update(source_code_only(fh.read()).encode())
    return h.hexdigest()


def profiled_traffic(kernel, workload):
    """DRAM bytes per launch of `kernel` from the committed ncu capture of this
    workload, or None when there is none or the kernel sources changed since."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)[kernel]
    except (OSError, KeyError, ValueError):
        return None
    if rec.get("source_sha256") != kernel_sources_sha256():
        return None
    wl = rec.get("per_workload", {}).get(workload)
    return None if wl is None else wl["dram_bytes_read"] + wl["dram_bytes_write"]


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def bf16_peak():
    """Measured dense bf16 tensor-core throughput (TFLOP/s, burst), or the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def indexer_flops(w):
    """Algorithmic multiply-adds x 2 of the indexer: every visible key against the
    T x 16 query heads over 64 dims."""
    return 2 * 16 * 64 * w.T * (int(w.pos.max()) + 1)


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
    """NVML sampler (a background thread, ~1 ms period) running during the timed
    region: SM clock and the clock-event (throttle) reasons."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, index):
        import threading

        self.samples, self.reasons, self.max_mhz, self.err = [], set(), None, None
        self.stop_flag = False
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report it
            self.nv, self.err = None, str(e)
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def _run(self):
        if self.nv is None:
            return
        while not self.stop_flag:
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for n, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(n)
            except Exception as e:
                self.err = str(e)
                return
            time.sleep(0.001)

    def stop(self):
        self.stop_flag = True
        self.thread.join(timeout=5)
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml",
                **({"error": self.err} if self.err else {})}


def dist_setup(n, backend="nccl"):
    """One process per GPU (torchrun sets RANK / WORLD_SIZE / LOCAL_RANK); every
    rank runs an independent replica of the step.  backend "gloo" (CPU, no
    device) serves the host-side tests."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n:
        raise SystemExit(f"--gpus {n} but WORLD_SIZE={world}")
    if world > 1:
        import datetime

        import torch.distributed as dist

        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif backend == "nccl":
        torch.cuda.set_device(0)
    return rank, world, local


def reduce_max(x, world, device="cuda"):
    """The maximum of x over all ranks (the slowest replica sets the step time)."""
    if world == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world, cuda=True):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
    if cuda:
        torch.cuda.synchronize()


def whole_job_gbs(bytes_per_step, ms_max, world):
    """Weak scaling: every rank moves bytes_per_step per step; the job's rate is
    the bytes of all ranks over the slowest rank's step time."""
    return world * bytes_per_step / (ms_max * 1e-3) / 1e9


def swa_bytes(w, window):
    """Sliding-window decode: each unique K/V row of the windows once, plus the
    queries and outputs.  Query t reads positions [pos_t + 1 - n_t, pos_t] with
    n_t = min(pos_t + 1, window)."""
    rows = [np.arange(int(p) + 1 - min(int(p) + 1, window), int(p) + 1) for p in w.pos]
    uniq = np.unique(np.concatenate(rows)).size
    gathered = sum(r.size for r in rows)
    return {"step": uniq * 2048 + w.T * 2 * 64 * 128 * 2, "unique_rows": uniq, "gathered_rows": gathered}


def index_bytes(w):
    """The indexer stage alone: the key cache up to the furthest visible
    position, the per-query indexer inputs, and the fp32 scores it writes."""
    n_max = int(w.pos.max()) + 1
    step = n_max * KEY_BYTES[w.key_dtype] + w.T * (16 * 64 * 2 + 16 * 4) + w.T * w.L * 4
    return {"step": step, "unique_rows": 0, "gathered_rows": 0}


def oracle_step(w, op, window):
    """One step of the oracle (test infrastructure) for this workload and op."""
    import oracle

    if op == "swa":
        return oracle.swa_decode(w.q, w.kv, w.pos, window), oracle.window_select(w.pos, window)
    if op == "index":
        return oracle.index_scores(w.q_idx, w.w_idx, w.k_idx, w.k_scale, w.pos), None
    return oracle.decode(w.q, w.q_idx, w.w_idx, w.k_idx, w.k_scale, w.kv, w.pos, w.topk)


def cpu_model():
    """The host CPU's model name and logical core count."""
    name = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    name = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return name, os.cpu_count()


def one_query(w):
    """The workload restricted to its last query (the same caches): the bounded
    sample of the one-thread oracle timing."""
    import copy

    s = copy.copy(w)
    t = w.T - 1
    s.T, s.q, s.q_idx, s.w_idx, s.pos = 1, w.q[t:t + 1], w.q_idx[t:t + 1], w.w_idx[t:t + 1], w.pos[t:t + 1]
    return s


def cpu_baseline(w, budget_s=15.0, op="step", window=128):
    """The oracle as it stands, on this host's cores, over whole steps of the same
    workload until about budget_s seconds have passed (mean step time); then one
    thread on a bounded sample: the step of the workload's last query alone."""
    import oracle

    times = []
    t_end = time.perf_counter() + budget_s
    while True:
        t0 = time.perf_counter()
        _, sel = oracle_step(w, op, window)
        times.append(time.perf_counter() - t0)
        if time.perf_counter() > t_end or len(times) >= 50:
            break
    cores = oracle.threads()
    w1 = one_query(w)
    oracle.set_threads(1)
    try:
        t1 = []
        t_end = time.perf_counter() + budget_s / 3
        while True:
            t0 = time.perf_counter()
            _, sel1 = oracle_step(w1, op, window)
            t1.append(time.perf_counter() - t0)
            if time.perf_counter() > t_end or len(t1) >= 20:
                break
    finally:
        oracle.set_threads(cores)
    return {"mean_s": statistics.mean(times), "steps": len(times), "sel": sel, "cores": cores,
            "one_thread_mean_s": statistics.mean(t1), "one_thread_steps": len(t1), "one_thread_sel": sel1,
            "one_thread_workload": w1}


def workload_config(w, args):
    """The workload's identity (the same in both arms)."""
    c = {"workload": w.name, "op": args.op, "L": w.L, "T": w.T, "topk": w.topk, "key_dtype": w.key_dtype,
         "recipe": w.recipe, "seed": w.seed}
    if args.op == "swa":
        c["window"] = args.window
    return c


def run_reference(args, w, rank, world):
    if rank != 0:
        return
    import oracle

    for _ in range(args.warmup):
        oracle_step(w, args.op, args.window)
    times = []
    sel = None
    for _ in range(args.steps):
        t0 = time.perf_counter()
        _, sel = oracle_step(w, args.op, args.window)
        times.append(time.perf_counter() - t0)
    ab = (swa_bytes(w, args.window) if args.op == "swa" else index_bytes(w) if args.op == "index"
          else algorithmic_bytes(w, sel))
    t = statistics.mean(times)
    value = ab["step"] / t / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t * 1e3, 3), "us_per_step": round(t * 1e6, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, args),
        "run": {"timing": "wall clock per whole oracle step, mean", "cpu": cpu_model()[0], "nproc": cpu_model()[1]},
        "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": oracle.threads(), "kind": "oracle",
                         "sample": f"whole steps of {w.name} (fp64 C oracle, OpenMP), {args.steps} timed, mean"},
        "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="verify_1m",
                    help="workload name (default: the 1M-context 8-token verify block, the largest single-GPU case)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg (profiling runs)")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--op", choices=["step", "swa", "index"], default="step",
                    help="step: the DSA decode/verify step; swa: sliding-window decode on the same q / K/V; "
                         "index: the indexer stage alone (dsa_index_scores)")
    ap.add_argument("--window", type=int, default=128, help="window of --op swa")
    ap.add_argument("--no-bypass", action="store_true", help="score and select even when every query sees <= topk")
    ap.add_argument("--pos", choices=["host", "device"], default="host",
                    help="device: query positions in device memory (dsa_decode_devpos_ws), one graph for every position")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    w = synth.config(args.config)

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, w, rank, int(os.environ.get("WORLD_SIZE", "1")))
        return

    from sparse_attention_decode_relu_b200 import dsa

    dsa.dsa_set_short_context_bypass(not args.no_bypass)
    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    d = dsa.to_device(w, device=dev, with_kv=args.op != "index")
    T, L, topk = w.T, w.L, w.topk
    scores = torch.empty((T, (L + 3) // 4 * 4), dtype=torch.float32, device=dev) if args.op == "index" else None
    ws = dsa.workspace(T, L, topk, device=dev)
    out = torch.empty((T, 64, 128), dtype=torch.bfloat16, device=dev)
    sel = torch.empty((T, topk), dtype=torch.int32, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
    sweep = torch.ones(2 * l2 // 4, dtype=torch.float32, device=dev)

    def flush_l2():
        # Write a buffer twice the L2 size (evicts everything, writing back our
        # outputs), then read another one (the L2 ends up full of clean lines, so
        # the timed step does not pay for write-backs of the flush itself).
        flush.zero_()
        sweep.amax()
    stream = torch.cuda.Stream(device=dev)
    grid = dsa.dsa_step_grid(w.key_dtype == "fp8")
    trace = torch.zeros(grid * 32, dtype=torch.int64, device=dev)

    pos_dev = torch.tensor(w.pos, dtype=torch.int32, device=dev)

    def step():
        if args.op == "index":
            dsa.dsa_index_scores(d["q_idx"], d["w_idx"], d["k_idx"], w.pos, scores, k_scale=d["k_scale"])
        elif args.op == "swa":
            dsa.dsa_swa_decode(d["q"], d["kv"], w.pos, args.window, out, ws)
        elif args.pos == "device":
            dsa.dsa_decode_devpos_ws(d["q"], d["q_idx"], d["w_idx"], d["k_idx"], d["kv"], pos_dev, topk, out, sel, ws,
                                     k_scale=d["k_scale"])
        else:
            dsa.dsa_decode_ws(d["q"], d["q_idx"], d["w_idx"], d["k_idx"], d["kv"], d["pos"], topk, out, sel, ws,
                              k_scale=d["k_scale"])

    # One eager call counts the kernels of a step; then capture the step in a graph.
    with torch.cuda.stream(stream):
        n0 = dsa.dsa_launch_count()
        step()
        kernels_per_step = dsa.dsa_launch_count() - n0
    stream.synchronize()
    dsa.dsa_device_status(stream)
    # The graph carries the in-kernel phase stamps (a few stores per block).
    graph = torch.cuda.CUDAGraph()
    dsa.dsa_set_step_trace(trace)
    with torch.cuda.graph(graph, stream=stream):
        step()
    dsa.dsa_set_step_trace(None)

    def timed_step():
        """Cold L2, then one graph replay of the whole step, timed by events.  A
        short GPU-side spin ahead of the first event keeps the host's graph
        submission out of the timed region (the GPU never waits for the host)."""
        flush_l2()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        stream.wait_stream(torch.cuda.current_stream())   # the flush (and trace reset) come first
        with torch.cuda.stream(stream):
            torch.cuda._sleep(SPIN_CYCLES)
            s0.record(stream)
            graph.replay()
            s1.record(stream)
        stream.synchronize()
        return s0.elapsed_time(s1)

    def phases():
        """Phase spans of the last replay, from the in-kernel stamps (a phase runs
        from its earliest start stamp to its latest end stamp over the blocks that
        stamped it)."""
        t = trace.view(grid, 32).cpu().numpy().astype(np.int64)

        def span(a, b):
            sa, sb = t[:, a][t[:, a] > 0], t[:, b][t[:, b] > 0]
            return (sb.max() - sa.min()) / 1e3 if sa.size and sb.size else 0.0

        spans = {"indexer": span(0, 1), "barrier": span(1, 2), "topk_extract": span(2, 3),
                 "topk_select": span(4, 5), "attention": span(6, 7), "merge": span(8, 9)}
        spans["kernel"] = span(0, 30)
        # SM clock over the last kernel of the step (its own start: clock 27, time 31)
        spans["sm_mhz_in_kernel"] = float((t[0, 29] - t[0, 27]) / max(1, t[0, 30] - t[0, 31]) * 1e3)
        spans["start_skew"] = (t[:, 0].max() - t[:, 0].min()) / 1e3
        return spans

    for _ in range(args.warmup):
        timed_step()
    barrier(world)
    clocks = Clocks(local)
    totals = []
    phase_sum = {}
    for _ in range(args.steps):
        trace.zero_()
        totals.append(timed_step())
        for k, v in phases().items():
            phase_sum[k] = phase_sum.get(k, 0.0) + v
    barrier(world)
    clk = clocks.stop()
    dsa.dsa_device_status(stream)
    ms = reduce_max(statistics.mean(totals), world)
    phase_us = {k: round(v / args.steps, 2) for k, v in phase_sum.items()}

    ab = (swa_bytes(w, args.window) if args.op == "swa" else index_bytes(w) if args.op == "index"
          else algorithmic_bytes(w, sel.cpu().numpy()))
    value = whole_job_gbs(ab["step"], ms, world)

    # End to end through the public API, as a serving loop would run it: one CUDA
    # graph holds, per step, the host->device copies of the step's query-side
    # inputs and positions from pinned host memory, the step with positions in
    # device memory (dsa_decode_devpos_ws; dsa_swa_decode for --op swa), and the
    # device->host copies of the outputs.  The caches stay resident.
    e2e = None
    if not args.no_e2e and args.op != "index":
        # The step's query-side inputs (and positions) are views of one device
        # buffer filled by one copy from one pinned host buffer; the outputs are
        # views of one device buffer read back by one copy.
        names = ("q",) if args.op == "swa" else ("q", "q_idx", "w_idx")

        def carve(buf, parts):
            views, off = {}, 0
            for k, (shape, dt) in parts.items():
                n = int(np.prod(shape)) * torch.empty((), dtype=dt).element_size()
                views[k] = buf[off:off + n].view(dt).view(shape)
                off = (off + n + 255) // 256 * 256
            return views

        in_parts = {k: (tuple(d[k].shape), d[k].dtype) for k in names}
        if args.op != "swa":
            in_parts["pos"] = ((w.T,), torch.int32)
        out_parts = {"out": (tuple(out.shape), out.dtype)}
        if args.op != "swa":
            out_parts["sel"] = (tuple(sel.shape), sel.dtype)
        n_in = sum((int(np.prod(s_)) * torch.empty((), dtype=t_).element_size() + 255) // 256 * 256 for s_, t_ in in_parts.values())
        n_out = sum((int(np.prod(s_)) * torch.empty((), dtype=t_).element_size() + 255) // 256 * 256 for s_, t_ in out_parts.values())
        h_inbuf = torch.empty(n_in, dtype=torch.uint8).pin_memory()
        d_inbuf = torch.empty(n_in, dtype=torch.uint8, device=dev)
        h_outbuf = torch.empty(n_out, dtype=torch.uint8).pin_memory()
        d_outbuf = torch.empty(n_out, dtype=torch.uint8, device=dev)
        h_in, dev_in = carve(h_inbuf, in_parts), carve(d_inbuf, in_parts)
        h_o, dev_o = carve(h_outbuf, out_parts), carve(d_outbuf, out_parts)
        for k in names:
            h_in[k].copy_(d[k].cpu())
        if args.op != "swa":
            h_in["pos"].copy_(torch.tensor(w.pos, dtype=torch.int32))
        h2d, d2h = n_in, n_out

        def e2e_step():
            d_inbuf.copy_(h_inbuf, non_blocking=True)
            if args.op == "swa":
                dsa.dsa_swa_decode(dev_in["q"], d["kv"], w.pos, args.window, dev_o["out"], ws)
            else:
                dsa.dsa_decode_devpos_ws(dev_in["q"], dev_in["q_idx"], dev_in["w_idx"], d["k_idx"], d["kv"],
                                         dev_in["pos"], topk, dev_o["out"], dev_o["sel"], ws, k_scale=d["k_scale"])
            h_outbuf.copy_(d_outbuf, non_blocking=True)

        with torch.cuda.stream(stream):
            e2e_step()   # eager once (first-call set-up outside the capture)
        stream.synchronize()
        e_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(e_graph, stream=stream):
            e2e_step()
        for _ in range(args.warmup):
            with torch.cuda.stream(stream):
                e_graph.replay()
        stream.synchronize()
        e_times = []
        for _ in range(args.steps):
            flush_l2()
            torch.cuda.current_stream().synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                a.record(stream)
                e_graph.replay()
                b.record(stream)
            stream.synchronize()
            e_times.append(a.elapsed_time(b))
        dsa.dsa_device_status(stream)
        if args.op != "swa":   # the host copies hold the step's results
            assert torch.equal(h_o["sel"], sel.cpu()), "end-to-end selection differs from the device-timed step"
        e_ms = reduce_max(statistics.mean(e_times), world)
        e2e = {"value": round(whole_job_gbs(ab["step"], e_ms, world), 3), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e_ms, 4),
               "timing": "CUDA-graph replay of one H2D copy (inputs and positions) + " +
                         ("dsa_swa_decode" if args.op == "swa" else "dsa_decode_devpos_ws") +
                         " + one D2H copy (outputs), CUDA events per step, mean"}
        del e_graph

    # Roofline of the dominant kernel.  A step with the indexer launches two
    # kernels: the indexer kernel, then the cooperative top-k/attention kernel.
    # Their durations come from the library's stage events (one between the two
    # launches) on eager calls of the same step, under the same cold-L2 protocol
    # (the GPU spins while the host submits, so it never waits for the host);
    # each kernel's algorithmic bytes are its share of the step's.
    peak, which = peaks()
    bypassed = (args.op == "step" and not args.no_bypass and args.pos == "host"
                and int(w.pos.max()) + 1 <= topk)   # no indexer phase then
    kernels = {}
    if args.op == "step" and not bypassed:
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        with torch.cuda.stream(stream):
            for e in evs:   # torch times only events it has seen recorded; the graph re-records them
                e.record(stream)
        stream.synchronize()
        t_idx, t_coop = [], []
        dsa.dsa_set_stage_events(evs)
        for i in range(args.warmup + args.steps):
            flush_l2()
            stream.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(stream):
                torch.cuda._sleep(SPIN_CYCLES)
                step()
            stream.synchronize()
            if i >= args.warmup:
                t_idx.append(evs[0].elapsed_time(evs[1]))
                t_coop.append(evs[1].elapsed_time(evs[4]))
        dsa.dsa_set_stage_events(None)
        dsa.dsa_device_status(stream)
        idx_in = w.T * (16 * 64 * 2 + 16 * 4)
        kernels["index_kernel"] = {"us": reduce_max(statistics.mean(t_idx), world) * 1e3,
                                   "bytes": ab["indexer"] + idx_in}
        kernels["step_kernel"] = {"us": reduce_max(statistics.mean(t_coop), world) * 1e3,
                                  "bytes": ab["step"] - ab["indexer"] - idx_in}
    elif args.op == "index":
        kernels["index_kernel"] = {"us": ms * 1e3, "bytes": ab["step"]}
    else:
        kernels["step_kernel"] = {"us": ms * 1e3, "bytes": ab["step"]}
    dom = max(kernels, key=lambda k: kernels[k]["us"])
    achieved = kernels[dom]["bytes"] / (kernels[dom]["us"] * 1e-6) / 1e9
    key = w.name if args.op == "step" else f"{w.name}:{args.op}"
    roof = {"kernel": dom, "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "peak_source": which,
            "traffic": profiled_traffic(dom, key) if args.pos == "host" else None,
            "algorithmic_bytes": kernels[dom]["bytes"], "duration_us": round(kernels[dom]["us"], 2),
            "kernels": {k: {"us": round(v["us"], 2), "algorithmic_bytes": v["bytes"],
                            "achieved_gbs": round(v["bytes"] / (v["us"] * 1e-6) / 1e9, 1)} for k, v in kernels.items()},
            "timing": "stage events around each kernel of eager calls of the step, cold L2, mean"
                      if args.op == "step" and not bypassed else "the step's own events"}

    # The indexer's tensor-core rate (tcgen05.mma), over its in-kernel phase time.
    tensor = None
    if args.op in ("step", "index") and not bypassed and phase_us.get("indexer", 0) > 0:
        tpk, tsrc = bf16_peak()
        tf = indexer_flops(w) / (phase_us["indexer"] * 1e-6) / 1e12
        tensor = {"phase": "indexer", "flops_per_step": indexer_flops(w), "phase_us": phase_us["indexer"],
                  "tflops": round(tf, 2), "peak": tpk, "unit": "TFLOP/s", "frac": round(tf / tpk, 4),
                  "peak_source": tsrc}

    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 5), "us_per_step": round(ms * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(w, args),
        "run": {"short_context_bypass": not args.no_bypass, "positions": args.pos,
                "parallelism": f"replicas{world}",
                "l2": "flushed before every step (write 2x L2, then read another 2x L2: cold and clean)",
                "timing": "CUDA-graph replay of " + ("dsa_swa_decode" if args.op == "swa" else
                                                       "dsa_index_scores" if args.op == "index" else
                                                       "dsa_decode_devpos_ws" if args.pos == "device" else
                                                       "dsa_decode_ws") + ", CUDA events per step, mean",
                "algorithmic_bytes_per_step": ab["step"], "unique_kv_rows": ab["unique_rows"],
                "gathered_kv_rows": ab["gathered_rows"], "cpu": cpu_model()[0], "nproc": cpu_model()[1]},
        "frac_of_peak_hbm": round(ab["step"] / (ms * 1e-3) / 1e9 / peak, 4),
        "phase_us": phase_us,
        "roofline": roof,
        "tensor": tensor,
        "e2e": e2e,
        "gpu_launches": int(kernels_per_step * args.steps),
        "clocks": clk,
    }
    if rank == 0 and not args.no_cpu_baseline and args.op != "index":
        cb = cpu_baseline(w, args.cpu_budget, args.op, args.window)
        w1 = cb["one_thread_workload"]
        ab1 = swa_bytes(w1, args.window) if args.op == "swa" else algorithmic_bytes(w1, cb["one_thread_sel"])
        cpu, nproc = cpu_model()
        line["cpu_baseline"] = {
            "value": round(ab["step"] / cb["mean_s"] / 1e9, 4), "unit": "GB/s", "cores": cb["cores"],
            "kind": "oracle", "us_per_step": round(cb["mean_s"] * 1e6, 1),
            "sample": f"{cb['steps']} whole steps of {w.name} on {cb['cores']} OpenMP threads, mean",
            "cpu": cpu, "nproc": nproc,
            "one_thread": {"value": round(ab1["step"] / cb["one_thread_mean_s"] / 1e9, 4), "unit": "GB/s",
                           "cores": 1, "us_per_step": round(cb["one_thread_mean_s"] * 1e6, 1),
                           "sample": f"{cb['one_thread_steps']} steps of the last query of {w.name} alone "
                                     f"(T = 1, pos = {int(w1.pos[0])}), mean"}}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()
