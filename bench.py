"""Benchmark of the KLD statistic on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

A step is one pass of the whole statistic over one batch: the fused row pass
(log-softmax of both rows, KL, argmaxes, NLL) over every row, then the
fixed-order reduction and exact percentile selection, then the result copied
to the host. The batch is one 8192-token context at a vocabulary of 151936
(fp32 logits, 2 x 4.98 GB per GPU), generated on the device by the seeded
generator; it is far larger than L2, so no L2 flush is needed between steps.

With N GPUs, one process per GPU (launched with torchrun, or by this script
itself when --gpus N > 1 is given without it), every rank scores its own
context (weak scaling); the per-row records are all-gathered over NCCL and
every rank reduces the full set, since exact percentiles need all rows.

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import shutil
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "logit rows/s and HBM GB/s (fraction of B200 peak) for KLD+top-1 at V=151936"
WORKLOAD = "ctx8192_v151936_f32"
VARIANT = "ctx8192_v151936_bf16"
FALLBACK_HBM_GBS = 6650.0
RESULT_BYTES = 160  # sizeof(kld_result_t)
ROW_RECORD_BYTES = 40  # sizeof(kld_row_t)


def _env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _code_only(text: str) -> str:
    """C/CUDA source without its comments and blank lines, so that an edit
    of the comments alone does not change the hash of the code."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines())
    return "\n".join(ln for ln in lines if ln)


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for name in ("kld_rows_kernel.cuh", "kld_rows.cu", "kld_internal.h", "kld_finish.cuh"):  # the row kernel and its launch
        with open(os.path.join(ROOT, "logit_kl_divergence_b200", "csrc", name), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current row-kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d.get(workload)
        if e and e.get("kernel_source_hash") == kernel_source_hash():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """SM clock and throttle reasons during the timed region.

    NVML is polled from a thread every ~2 ms with a host timestamp per sample
    (nvidia-smi at 100 ms as the fallback). The sampler starts before the
    warm-up steps, so that polling is already running when the timed region
    opens; `mark_start` / `mark_end` bracket that region on the host clock and
    `stop` reports the samples inside it. A region too short to hold three
    samples also reports the warm-up samples (they run the same kernels) and
    says so in "window"."""

    REASONS = {  # NVML clocks-event reason bits
        "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "sw_power_cap": 0x4,
    }

    def __init__(self, gpu_index: int):
        import threading

        self.samples = []  # (host time, sm MHz, max sm MHz, reason names)
        self.t_start = self.t_end = None
        self.t_open = time.perf_counter()
        self._stop = threading.Event()
        self._thread = None
        self._proc = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(gpu_index)
            # queried once: this call takes milliseconds, the per-sample
            # clock and reason queries about a microsecond
            self._max = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._poll, daemon=True)
            self._thread.start()
        except Exception:
            self._nv = None
            exe = shutil.which("nvidia-smi")
            if exe:
                self._proc = subprocess.Popen(
                    [exe, "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active",
                     "--format=csv,noheader,nounits", "-lms", "100", "-i", str(gpu_index)],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)

    def _poll(self):
        nv, h = self._nv, self._h
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                mx = self._max
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                names = {name for name, bit in self.REASONS.items() if bits & bit}
                self.samples.append((time.perf_counter(), sm, mx, names))
            except Exception:
                pass
            self._stop.wait(0.002)

    def mark_start(self):
        self.t_start = time.perf_counter()

    def mark_end(self):
        self.t_end = time.perf_counter()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
            samples = self.samples
        elif self._proc is not None:
            self._proc.terminate()
            try:
                out, _ = self._proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
                out, _ = self._proc.communicate()
            # nvidia-smi lines carry no host time: spread them evenly over
            # the sampler's lifetime.
            lines = out.strip().splitlines()
            t1 = time.perf_counter()
            samples = []
            for i, line in enumerate(lines):
                parts = [x.strip() for x in line.split(",")]
                try:
                    t = self.t_open + (t1 - self.t_open) * (i + 0.5) / max(1, len(lines))
                    samples.append((t, float(parts[0]), float(parts[1]), set()))
                except (ValueError, IndexError):
                    continue
        else:
            return None
        t0 = self.t_start if self.t_start is not None else self.t_open
        t1 = self.t_end if self.t_end is not None else time.perf_counter()
        inside = [s for s in samples if t0 <= s[0] <= t1]
        window = "timed region"
        if len(inside) < 3:
            inside = [s for s in samples if s[0] <= t1]
            window = "warm-up and timed region (the timed region alone held fewer than 3 samples)"
        if not inside:
            return None
        reasons = set()
        for s in inside:
            reasons |= s[3]
        return {"sm_mhz": statistics.median(s[1] for s in inside),
                "sm_max_mhz": max(s[2] for s in inside),
                "sm_min_mhz": min(s[1] for s in inside),
                "reasons": sorted(reasons), "samples": len(inside), "window": window,
                "timed_region_ms": round(1000.0 * (t1 - t0), 3),
                "source": "nvml" if self._thread is not None else "nvidia-smi"}


def cpu_baseline(name: str, budget_s: float = 12.0, max_rows: int = 4096):
    """The oracle, as it stands, single-threaded, on a bounded sample of rows
    of the same workload recipe (generated on the host)."""
    import oracle
    from logit_kl_divergence_b200 import synth

    odt = {synth.F32: oracle.F32, synth.BF16: oracle.BF16, synth.F16: oracle.F16}
    probe = synth.make(name, n=8)
    t0 = time.perf_counter()
    oracle.rows(probe.base, probe.quant, probe.token_ids, odt[probe.dtype], 1)
    per_row = (time.perf_counter() - t0) / 8
    rows = int(max(8, min(max_rows, budget_s / max(per_row, 1e-6))))
    w = synth.make(name, n=rows, seed=synth.WORKLOADS[name][4] + 1000)
    t0 = time.perf_counter()
    r = oracle.rows(w.base, w.quant, w.token_ids, odt[w.dtype], 1)
    oracle.reduce(r, True)
    dt = time.perf_counter() - t0
    single = {"value": rows / dt, "unit": "rows/s", "cores": 1, "kind": "oracle",
              "sample": f"{rows} rows of {name} (same recipe, host-generated), "
                        f"fp64 two-pass oracle, single thread, {dt:.1f} s",
              "cpu_model": _cpu_model()}
    # The same per-row code on every host core (whole rows per thread, so the
    # records are bit-identical to the single-threaded run).
    cores = os.cpu_count() or 1
    rows_mt = int(max(cores, min(64 * cores, 8.0 * cores / max(per_row, 1e-6))))
    w = synth.make(name, n=rows_mt, seed=synth.WORKLOADS[name][4] + 2000)
    t0 = time.perf_counter()
    r = oracle.rows(w.base, w.quant, w.token_ids, odt[w.dtype], cores)
    oracle.reduce(r, True)
    dt = time.perf_counter() - t0
    multi = {"value": rows_mt / dt, "unit": "rows/s", "cores": cores, "kind": "oracle",
             "sample": f"{rows_mt} rows of {name}, the same oracle row-parallel on {cores} "
                       f"threads, {dt:.1f} s"}
    return single, multi


def _cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_reference(args, rank: int):
    if rank != 0:
        return
    from logit_kl_divergence_b200 import synth

    import oracle

    odt = {synth.F32: oracle.F32, synth.BF16: oracle.BF16, synth.F16: oracle.F16}
    rows = 64
    samples = [synth.make(WORKLOAD, n=rows, seed=100 + i) for i in range(min(args.steps, 4))]
    for i in range(args.warmup):
        w = samples[i % len(samples)]
        oracle.reduce(oracle.rows(w.base, w.quant, w.token_ids, odt[w.dtype], 1), True)
    t0 = time.perf_counter()
    for i in range(args.steps):
        w = samples[i % len(samples)]
        oracle.reduce(oracle.rows(w.base, w.quant, w.token_ids, odt[w.dtype], 1), True)
    dt = time.perf_counter() - t0
    value = rows * args.steps / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "rows/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "rows_per_step": rows, "vocab": 151936,
                   "logit_dtype": "f32", "sample": "64-row sample of the workload per step"},
        "cpu_baseline": {"value": value, "unit": "rows/s", "cores": 1, "kind": "oracle",
                         "sample": f"{rows} rows per step of {WORKLOAD}, single-threaded fp64 oracle"},
        "e2e": {"value": value, "unit": "rows/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


SPLIT_ROWS = (1, 4, 16, 32)
SPLIT_CALLS = 1000
SPLIT_COLD_BYTES = 256 << 20  # inputs rotated per call cycle: twice the 126 MB L2


def split_row_latency(dev, stream, min_calls: int = SPLIT_CALLS):
    """Few-row, large-vocabulary launches (N in SPLIT_ROWS, V = 262144 fp32):
    SPLIT_CALLS back-to-back calls of the whole statistic on one stream,
    plainly and as CUDA-graph replays, with the whole-row launch shape
    (kld_stats_run_static) beside them. Each call reads its own copy of the
    inputs from a ring larger than L2, so every call streams from HBM."""
    import torch

    from logit_kl_divergence_b200 import KLDStats, run_static, synth

    out = {"workload": "splitrow{1,4,16,32}_v262144_f32", "min_calls": min_calls,
           "l2": f"inputs rotated over copies totalling >= {SPLIT_COLD_BYTES >> 20} MB per cycle",
           "per_rows": {}}
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    for n in SPLIT_ROWS:
        w = synth.make(f"splitrow{n}_v262144_f32", device=dev)
        V = w.base.shape[1]
        call_bytes = 2 * n * V * w.bytes_per_elem
        k = max(1, -(-SPLIT_COLD_BYTES // call_bytes))
        bs = w.base.unsqueeze(0).repeat(k, 1, 1)
        qs = w.quant.unsqueeze(0).repeat(k, 1, 1)
        tok = w.token_ids
        st = KLDStats(max_rows=n, device=dev)
        res_buf = torch.zeros(256, dtype=torch.uint8, device=dev)
        calls = -(-min_calls // k) * k

        def timed(fn, reps):
            for i in range(min(k, 8)):
                fn(i)
            torch.cuda.synchronize(dev)
            a, b = ev(), ev()
            a.record(stream)
            for i in range(reps):
                fn(i % k)
            b.record(stream)
            torch.cuda.synchronize(dev)
            return a.elapsed_time(b) * 1000.0 / reps

        us_stream = timed(lambda i: st.run(bs[i], qs[i], tok), calls)
        us_whole = timed(lambda i: run_static(bs[i], qs[i], tok, res_buf), calls)
        # one graph holding one call per copy, replayed
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            for i in range(k):
                st.run(bs[i], qs[i], tok)
        stream.wait_stream(side)
        torch.cuda.synchronize(dev)
        with torch.cuda.graph(g):
            for i in range(k):
                st.run(bs[i], qs[i], tok)
        reps = calls // k
        g.replay()
        torch.cuda.synchronize(dev)
        a, b = ev(), ev()
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize(dev)
        us_graph = a.elapsed_time(b) * 1000.0 / (reps * k)
        # kernel-only time of the row pass (events around it, cold inputs)
        st.set_timing(True)
        rp = []
        for i in range(min(k, 50)):
            st.run(bs[i], qs[i], tok)
            st.result()
            rp.append(st.timing()[0] * 1000.0)
        st.set_timing(False)
        res = st.result()
        out["per_rows"][str(n)] = {
            "plan": st.plan(n, V, 0),
            "us_per_call_stream": us_stream, "us_per_call_graph": us_graph,
            "us_per_call_whole_row_launch": us_whole,
            "row_pass_us_median": statistics.median(rp),
            "gbs_stream": call_bytes / (us_stream * 1e3), "gbs_graph": call_bytes / (us_graph * 1e3),
            "gbs_row_pass": call_bytes / (statistics.median(rp) * 1e3),
            "calls": calls, "input_copies": k, "mean_kld": res["mean_kld"]}
        del g, bs, qs, w, st
        torch.cuda.synchronize(dev)
        torch.cuda.empty_cache()
    return out


def free_port() -> int:
    import socket

    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def torchrun_argv(n: int, port: int, script: str, argv: list[str]) -> list[str]:
    """One process per GPU on this node, rendezvous on the loopback address."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
            "--master-addr", "127.0.0.1", "--master-port", str(port), script, *argv]


def relaunch(n: int, argv: list[str]) -> int:
    """`python bench.py --gpus N` without torchrun: start the N ranks here.
    Returns the launcher's exit code (2 when fewer than N GPUs are visible)."""
    import torch

    visible = torch.cuda.device_count()
    if visible < n:
        print(f"bench.py: {n} GPUs requested (--gpus {n}) but {visible} visible; "
              f"nothing was run", file=sys.stderr)
        return 2
    return subprocess.run(torchrun_argv(n, free_port(), os.path.abspath(__file__), argv)).returncode


class DeviceClock:
    """Device time: CUDA events recorded on the launching stream."""

    def __init__(self, dev):
        import torch

        self.torch = torch
        self.dev = dev
        self.stream = torch.cuda.current_stream(dev)

    def mark(self):
        e = self.torch.cuda.Event(enable_timing=True)
        e.record(self.stream)
        return e

    def sync(self):
        self.torch.cuda.synchronize(self.dev)

    def ms(self, a, b) -> float:
        return a.elapsed_time(b)


class HostClock:
    """Host wall time, for ranks that run on CPU cores (the multi-rank logic
    checked with gloo and a stand-in handle); never a GPU measurement."""

    def mark(self):
        return time.perf_counter()

    def sync(self):
        pass

    def ms(self, a, b) -> float:
        return 1000.0 * (b - a)


def _over_ranks(x: float, device, op) -> float:
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=op)
    return float(t.item())


def sharded_line(args, rank: int, world: int, dev, sk, shard, clock, peak: float, peak_kind: str,
                 sampler=None, cpu_fn=None, workload: str = WORKLOAD):
    """The multi-GPU step, timed: every rank runs the row pass on its own
    shard, the records are all-gathered and every rank reduces all of them
    (``sk``: a ShardedKLDStats, the public multi-GPU API), then reads the
    result. Returns rank 0's JSON line (None on the other ranks).

    value: rows of all ranks / the max over ranks of the device time of the
    timed steps. e2e: the same step through ShardedKLDStats.run_host from
    (pinned) host copies of each shard, max over ranks. roofline: the row
    pass of each rank timed by the library's events; achieved = sum over
    ranks of that rank's algorithmic bytes / its mean row-pass time, against
    world x the per-GPU peak."""
    import torch
    import torch.distributed as dist

    base, quant, tok = shard
    N, V = base.shape
    eb = base.element_size()
    in_bytes = 2 * N * V * eb
    sk.stats.set_timing(True)
    res = None
    counts = [N] * world  # equal shards: one host wait per step (the result)
    for _ in range(args.warmup):
        res = sk.run(base, quant, tok, counts=counts)
    dist.barrier()
    clock.sync()
    if sampler is not None:
        sampler.mark_start()
    start = clock.mark()
    row_ms = []
    for _ in range(args.steps):
        res = sk.run(base, quant, tok, counts=counts)
        row_ms.append(sk.stats.timing()[0])
    end = clock.mark()
    clock.sync()
    if sampler is not None:
        sampler.mark_end()
    dist.barrier()
    clocks = sampler.stop() if sampler is not None else None
    ms = _over_ranks(clock.ms(start, end), dev, dist.ReduceOp.MAX)
    ms_per_step = ms / args.steps
    total_rows = N * world
    value = total_rows / (ms_per_step / 1000.0)
    avg_row_ms = sum(row_ms) / len(row_ms)
    achieved_rank = in_bytes / (avg_row_ms / 1000.0) / 1e9
    achieved = _over_ranks(achieved_rank, dev, dist.ReduceOp.SUM)
    slowest_row_ms = _over_ranks(avg_row_ms, dev, dist.ReduceOp.MAX)
    traffic = recorded_traffic(workload)
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak * world, "unit": "GB/s",
                "frac": achieved / (peak * world), "traffic": traffic,
                "peak_source": f"{world} x {peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
                "frac_of_8TBs_nominal": achieved / (8000.0 * world),
                "kernel": f"kld_rows_kernel<{'f32' if eb == 4 else 'bf16'}>",
                "row_pass_ms": avg_row_ms, "row_pass_ms_max_over_ranks": slowest_row_ms,
                "algorithmic_bytes_per_launch": in_bytes,
                "note": "achieved summed over ranks; traffic and bytes per launch are per rank"}

    # End to end: each rank's shard in host memory (pinned where a GPU is
    # present), copied by the library in chunks overlapped with its row pass.
    pin = torch.cuda.is_available() and base.is_cuda
    hb, hq = base.cpu(), quant.cpu()
    ht = None if tok is None else tok.cpu()
    if pin:
        hb, hq = hb.pin_memory(), hq.pin_memory()
        ht = None if ht is None else ht.pin_memory()
    e2e = None
    if args.e2e_steps > 0:
        sk.run_host(hb, hq, ht, device=dev, counts=counts)
        dist.barrier()
        clock.sync()
        a = clock.mark()
        for _ in range(args.e2e_steps):
            sk.run_host(hb, hq, ht, device=dev, counts=counts)
        b = clock.mark()
        clock.sync()
        ems = _over_ranks(clock.ms(a, b), dev, dist.ReduceOp.MAX) / args.e2e_steps
        e2e = {"value": total_rows / (ems / 1000.0), "unit": "rows/s",
               "h2d_bytes_per_step": (in_bytes + (4 * N if tok is not None else 0)) * world,
               "d2h_bytes_per_step": RESULT_BYTES * world, "ms_per_step": ems,
               "path": "ShardedKLDStats.run_host (kld_stats_run_rows_host per rank, record "
                       "all-gather, kld_stats_reduce; host buffers pinned); bytes summed over ranks"}
    del hb, hq, ht

    cpu = cpu_mt = None
    if rank == 0 and cpu_fn is not None and not args.no_cpu_baseline:
        cpu, cpu_mt = cpu_fn(workload)
    dist.barrier()  # the other ranks wait for rank 0's host-core baseline
    if rank != 0:
        return None
    return {
        "metric": METRIC, "value": value, "unit": "rows/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32" if eb == 4 else "bf16",
        "data": "synthetic",
        "config": {"workload": workload, "rows_per_gpu": N, "vocab": V,
                   "logit_dtype": "f32" if eb == 4 else "bf16", "global_rows": total_rows,
                   "parallelism": f"rows sharded over {world} GPU(s): one 8192-token context per "
                                  f"rank, records all-gathered (NCCL), every rank reduces all rows",
                   "l2": f"inputs ({in_bytes / 1e9:.2f} GB per step per GPU) exceed the 126 MB L2; "
                         f"no flush"},
        "roofline": roofline, "cpu_baseline": cpu, "cpu_baseline_all_cores": cpu_mt, "e2e": e2e,
        "gpu_launches": 2 * args.steps * world, "gpu_launches_note": "row pass + reduction per step per rank",
        "clocks": clocks, "gbs": in_bytes * world / (ms_per_step / 1000.0) / 1e9,
        "mean_kld": res["mean_kld"], "top1_agree_pct": res["top1_agree_pct"], "ppl": res["ppl"],
        "ppl_base": res["ppl_base"], "rms_dp": res["rms_dp"], "mean_dp": res["mean_dp"],
        "median_kld": res["median_kld"], "p99_kld": res["p99_kld"], "max_kld": res["max_kld"],
    }


def run_sharded_main(args, rank: int, world: int, local: int):
    """The multi-GPU benchmark (NCCL group, one rank per GPU; --sharded runs
    it on a group of one rank)."""
    import datetime

    import torch
    import torch.distributed as dist

    from logit_kl_divergence_b200 import synth
    from logit_kl_divergence_b200.sharded import ShardedKLDStats

    dev = torch.device("cuda", local)
    if "MASTER_ADDR" not in os.environ:  # one rank, launched without torchrun
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(free_port()), RANK="0",
                          WORLD_SIZE="1", LOCAL_RANK=str(local))
    dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))
    dt = synth.F32 if args.dtype == "f32" else synth.BF16
    w = synth.make(WORKLOAD, device=dev, seed=synth.WORKLOADS[WORKLOAD][4] + 7919 * rank, n=args.rows,
                   dtype=dt)
    sk = ShardedKLDStats(max_rows_per_rank=w.base.shape[0], device=dev)
    peak, peak_kind = measured_peak()
    sampler = ClockSampler(local)
    try:
        line = sharded_line(args, rank, world, dev, sk, (w.base, w.quant, w.token_ids), DeviceClock(dev),
                            peak, peak_kind, sampler=sampler, cpu_fn=cpu_baseline)
        if line is not None:
            if args.rows is not None or args.dtype != "f32":
                line["config"]["override"] = {"rows": w.base.shape[0], "dtype": args.dtype,
                                              "note": "profiling run, not the benchmark workload"}
            print(json.dumps(line), flush=True)
    finally:
        sk.close()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-variants", action="store_true")
    ap.add_argument("--no-split-row", action="store_true")
    ap.add_argument("--no-grad", action="store_true")
    ap.add_argument("--no-topk", action="store_true")
    ap.add_argument("--split-calls", type=int, default=SPLIT_CALLS,
                    help="profiling only: fewer calls per size in the split-row section")
    ap.add_argument("--rows", type=int, default=None,
                    help="profiling only: fewer rows of the same recipe (not a bench line)")
    ap.add_argument("--dtype", choices=["f32", "bf16"], default="f32",
                    help="profiling only: logit dtype of the workload")
    ap.add_argument("--sharded", action="store_true",
                    help="take the row-sharded path (NCCL group, record all-gather) even on "
                         "one GPU: the multi-GPU step with a group of one rank")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    rank = _env_int("RANK", 0)
    world = _env_int("WORLD_SIZE", 1)
    local = _env_int("LOCAL_RANK", 0)

    if args.impl == "reference":
        run_reference(args, rank)
        return
    if world == 1 and args.gpus > 1 and "LOCAL_RANK" not in os.environ:
        sys.exit(relaunch(args.gpus, sys.argv[1:]))

    import torch

    from logit_kl_divergence_b200 import KLDStats, synth

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1 or args.sharded:
        run_sharded_main(args, rank, world, local)
        return

    name = WORKLOAD
    dt = synth.F32 if args.dtype == "f32" else synth.BF16
    w = synth.make(name, device=dev, seed=synth.WORKLOADS[name][4], n=args.rows, dtype=dt)
    N, V = w.base.shape
    eb = w.bytes_per_elem
    in_bytes = 2 * N * V * eb
    stream = torch.cuda.current_stream(dev)

    st = KLDStats(max_rows=N, device=dev)
    st.set_timing(True)
    row_ms, red_ms = [], []

    def step(timed: bool):
        st.run(w.base, w.quant, w.token_ids)
        res = st.result()
        if timed:
            rp_ms, rd_ms = st.timing()
            row_ms.append(rp_ms)
            red_ms.append(rd_ms)
        return res

    sampler = ClockSampler(local)
    for _ in range(args.warmup):
        res = step(False)

    torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler.mark_start()
    start.record(stream)
    for _ in range(args.steps):
        res = step(True)
    end.record(stream)
    torch.cuda.synchronize(dev)
    sampler.mark_end()
    clocks = sampler.stop()
    ms = start.elapsed_time(end)
    ms_per_step = ms / args.steps
    total_rows = N
    value = total_rows / (ms_per_step / 1000.0)

    # Read-only roofline of the row pass on this device, for context beside the
    # copy-bandwidth peak: the library's probe streams the same two inputs
    # into shared memory with the row pass's bulk copies and computes nothing.
    read_probe_gbs = None
    for _ in range(3):
        st.read_probe(w.base, w.quant)
    torch.cuda.synchronize(dev)
    pa, pb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    preps = 10
    pa.record(stream)
    for _ in range(preps):
        st.read_probe(w.base, w.quant)
    pb.record(stream)
    torch.cuda.synchronize(dev)
    read_probe_gbs = in_bytes / (pa.elapsed_time(pb) / preps / 1000.0) / 1e9

    peak, peak_kind = measured_peak()
    avg_row_ms = sum(row_ms) / len(row_ms)
    achieved = in_bytes / (avg_row_ms / 1000.0) / 1e9
    traffic = recorded_traffic(name)
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": traffic,
                "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
                "frac_of_8TBs_nominal": achieved / 8000.0,
                "read_probe_gbs": read_probe_gbs,
                "frac_of_read_probe": (achieved / read_probe_gbs) if read_probe_gbs else None,
                "kernel": f"kld_rows_kernel<{args.dtype}>", "row_pass_ms": avg_row_ms,
                "reduce_ms": (sum(red_ms) / len(red_ms)) if red_ms else None,
                "algorithmic_bytes_per_launch": in_bytes}

    # Other workloads of the same statistic, each through its own handle: the
    # bf16 variant of the same context (the target names both dtypes), four
    # 8192-token contexts in bf16, and the edge-case rows (near-one-hot, exact
    # ties, -inf padding, constant shifts). Row pass timed by the library's
    # events, step = kld_stats_run + kld_stats_result.
    def time_variant(wname):
        wv = synth.make(wname, device=dev)
        sv = KLDStats(max_rows=wv.n, device=dev)
        sv.set_timing(True)
        for _ in range(3):
            sv.run(wv.base, wv.quant, wv.token_ids)
            sv.result()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        rms = []
        a.record(stream)
        for _ in range(args.steps):
            sv.run(wv.base, wv.quant, wv.token_ids)
            rv = sv.result()
            rms.append(sv.timing()[0])
        b.record(stream)
        torch.cuda.synchronize(dev)
        vbytes = 2 * wv.base.numel() * wv.bytes_per_elem
        vms = a.elapsed_time(b) / args.steps
        rrow = sum(rms) / len(rms)
        out = {"rows": wv.n, "vocab": wv.base.shape[1], "logit_dtype": "f32" if wv.bytes_per_elem == 4 else "bf16",
               "value": wv.n / (vms / 1000.0), "unit": "rows/s", "ms_per_step": vms,
               "row_pass_ms": rrow, "achieved_gbs": vbytes / (rrow / 1000.0) / 1e9,
               "frac": vbytes / (rrow / 1000.0) / 1e9 / peak,
               "traffic": recorded_traffic(wname), "algorithmic_bytes_per_launch": vbytes,
               "stats": {k: rv[k] for k in ("mean_kld", "median_kld", "p90_kld", "p99_kld", "max_kld",
                                            "top1_agree_pct", "ppl", "n_flagged")}}
        sv.close()
        del wv
        torch.cuda.empty_cache()
        return out

    variants = {}
    if not args.no_variants:
        del w
        torch.cuda.empty_cache()
        for vname in (VARIANT, "ctx4x8192_v151936_bf16", "edge_16384x131072_f32"):
            variants[vname] = time_variant(vname)
        w = synth.make(name, device=dev, seed=synth.WORKLOADS[name][4])

    # Gradient of the KL w.r.t. the quant logits (row pass + reduction +
    # gradient pass writing fp32 [N, V]) on the same context.
    grad = None
    if not args.no_grad:
        gout = torch.empty_like(w.base)
        st.set_timing(True)
        for _ in range(3):
            st.run_grad(w.base, w.quant, w.token_ids, out=gout, scale=1.0 / N)
            st.result()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        gms = []
        gsteps = max(3, min(args.steps, 10))
        a.record(stream)
        for _ in range(gsteps):
            st.run_grad(w.base, w.quant, w.token_ids, out=gout, scale=1.0 / N)
            st.result()
            gms.append(st.second_pass_timing())
        b.record(stream)
        torch.cuda.synchronize(dev)
        step_ms = a.elapsed_time(b) / gsteps
        kms = sum(gms) / len(gms)
        gbytes = 3 * N * V * eb  # reads b and q, writes the fp32 gradient
        grad = {"workload": name, "grad_dtype": "f32", "steps": gsteps, "ms_per_step": step_ms,
                "value": N / (step_ms / 1000.0), "unit": "rows/s",
                "grad_pass_ms": kms, "grad_pass_gbs": gbytes / (kms / 1000.0) / 1e9,
                "grad_pass_frac": gbytes / (kms / 1000.0) / 1e9 / peak,
                "algorithmic_bytes_per_grad_launch": gbytes,
                "step_gbs": (gbytes + in_bytes) / (step_ms / 1000.0) / 1e9}
        del gout
        torch.cuda.empty_cache()

    # Top-128 compression of the base rows + KL against it on the same
    # context: per-row thresholds, the row pass in its top-k scan form (it
    # copies out the lanes holding candidates), the reduction and the top-k
    # selection over the copies. Each logit is read from memory once, so
    # the step is timed against the inputs' bytes.
    topk = None
    if not args.no_topk:
        for _ in range(2):
            st.run_topk(w.base, w.quant, w.token_ids, k=128)
            st.result()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        tsteps = max(2, min(args.steps, 5))
        kms, rms = [], []
        a.record(stream)
        for _ in range(tsteps):
            out = st.run_topk(w.base, w.quant, w.token_ids, k=128)
            st.result()
            kms.append(st.second_pass_timing())
            rms.append(st.timing()[0])
        b.record(stream)
        torch.cuda.synchronize(dev)
        tms = a.elapsed_time(b) / tsteps
        kpass = sum(kms) / len(kms)
        topk = {"workload": name, "k": 128, "steps": tsteps, "ms_per_step": tms,
                "value": N / (tms / 1000.0), "unit": "rows/s",
                "step_gbs": in_bytes / (tms / 1000.0) / 1e9,
                "step_frac": in_bytes / (tms / 1000.0) / 1e9 / peak,
                "scan_row_pass_ms": sum(rms) / len(rms),
                "threshold_and_select_ms": kpass,
                "exact_path_rows": st.topk_exact_rows(),
                "algorithmic_bytes_per_step": in_bytes,
                "mean_kl_topk": float(out["kl_topk"].mean().item())}
        del out

    # End to end through the public host-memory entry point: pinned host
    # buffers in, the result struct out, copies inside the timed region.
    e2e = None
    if args.e2e_steps > 0:
        hb = w.base.cpu().pin_memory()
        hq = w.quant.cpu().pin_memory()
        ht = w.token_ids.cpu().pin_memory()
        st.run_host(hb, hq, ht)
        st.result()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.e2e_steps):
            st.run_host(hb, hq, ht)
            st.result()
        b.record(stream)
        torch.cuda.synchronize(dev)
        ems = a.elapsed_time(b) / args.e2e_steps
        e2e = {"value": N / (ems / 1000.0), "unit": "rows/s",
               "h2d_bytes_per_step": in_bytes + 4 * N, "d2h_bytes_per_step": RESULT_BYTES,
               "ms_per_step": ems, "path": "kld_stats_run_host (pinned host buffers)"}
        del hb, hq, ht

    split_row = None
    if not args.no_split_row and args.rows is None:
        del w
        torch.cuda.empty_cache()
        split_row = split_row_latency(dev, stream, max(1, args.split_calls))

    cpu = cpu_mt = None
    if not args.no_cpu_baseline:
        cpu, cpu_mt = cpu_baseline(name)

    line = {
        "metric": METRIC, "value": value, "unit": "rows/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": args.dtype, "data": "synthetic",
        "config": {"workload": name, "rows_per_gpu": N, "vocab": V, "logit_dtype": args.dtype,
                   "global_rows": total_rows,
                   "parallelism": "one GPU, whole statistic per step (kld_stats_run)",
                   "l2": "inputs (9.96 GB per step per GPU) exceed the 126 MB L2; no flush"},
        "roofline": roofline, "cpu_baseline": cpu, "cpu_baseline_all_cores": cpu_mt, "e2e": e2e,
        "gpu_launches": 2 * args.steps, "clocks": clocks,
        "gbs": in_bytes / (ms_per_step / 1000.0) / 1e9,
        "mean_kld": res["mean_kld"], "top1_agree_pct": res["top1_agree_pct"], "ppl": res["ppl"],
        "ppl_base": res["ppl_base"], "rms_dp": res["rms_dp"], "mean_dp": res["mean_dp"],
        "variants": variants, "split_row": split_row, "grad": grad, "topk": topk,
    }
    if args.rows is not None or args.dtype != "f32" or args.split_calls != SPLIT_CALLS:
        line["config"]["override"] = {"rows": N, "dtype": args.dtype,
                                      "split_calls": args.split_calls,
                                      "note": "profiling run, not the benchmark workload"}
    print(json.dumps(line), flush=True)

    st.close()


if __name__ == "__main__":
    main()
