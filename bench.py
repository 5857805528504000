"""Benchmark of one Hybrid Tree Attention verification call (one layer) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference] [--num-splits S]

A step is one full verification call (prefix split-KV kernel, then the tree
pass fused with the log-sum-exp merge) over one batch of synthetic inputs
already resident in HBM.  Inputs rotate over enough buffer sets that every
step's K/V are not in L2 (126 MB) when it starts.  The metric is the
microseconds per layer call (lower is better) and, for the prefix kernel,
the achieved HBM bandwidth against the measured peak.

Under torchrun (N > 1) every rank runs its own calls on its own GPU (weak
scaling, no data-path collective); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from tree_masked_verification_b200 import hta  # noqa: E402
from tree_masked_verification_b200.inputs import (ACCEPT_WORKLOADS, WORKLOADS, bf16_bits,  # noqa: E402
                                                  accept_inputs, paged_cache)

METRIC = "µs per layer verify-attention call; achieved HBM GB/s vs B200 peak @32k prefix"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def workload_config(w, S, n_sets):
    tree = {"levels": "/".join(map(str, w.widths)), "random": "random", "chain": "chain"}[w.tree]
    if w.kind == "prefix":
        tree = "none (prefix-only attention)"
    lens = w.prefix_lens()
    call = {"prefix": "longspec_hta_prefix_attention",
            "window": "longspec_hta_window_verify"}.get(w.kind, "longspec_hta_verify")
    if w.block_size:
        call += "_paged"
    return {"workload": w.name, "call": call, "block_size": w.block_size or None,
            "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D, "T": w.T,
            "L_cap": w.L_cap, "L_mean": float(lens.mean()), "tree": tree,
            "k_peaked": w.k_peaked, "num_splits": S,
            "l2": f"inputs rotate over {n_sets} buffer sets ({n_sets}x the K/V bytes > 2x L2)"
            if n_sets > 1 else "K/V bytes per call > 2x L2"}


PREFIX_KERNEL_SOURCES = ("tree_masked_verification_b200/csrc/prefix_tc.cu",
                         "tree_masked_verification_b200/csrc/hta_kernels.h",
                         "tree_masked_verification_b200/csrc/hta_common.cuh")


def prefix_source_sha():
    """First 16 hex digits of the SHA-256 of the prefix kernel's sources
    (the kernel file and the two headers it compiles with, concatenated)."""
    import hashlib
    h = hashlib.sha256()
    for rel in PREFIX_KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload_name):
    """DRAM bytes per launch of the prefix kernel from the committed ncu
    summary, if that summary was taken on this workload with the current
    kernel sources and the default build (else None)."""
    if os.environ.get("LONGSPEC_HTA_LIB"):
        return None          # another build than the one profiled
    path = os.path.join(ROOT, "profiles", f"prefix_tc_kernel_{workload_name}.json")
    try:
        with open(path) as f:
            prof = json.load(f)
        sha = prefix_source_sha()
    except (OSError, ValueError):
        return None
    if prof.get("source_sha256_16") != sha:
        return None
    return int(prof["dram_bytes_read"] + prof["dram_bytes_write"])


def prefix_algorithmic_bytes(w):
    """Bytes the prefix kernel must move at minimum: K and V of the L_b
    prefix keys of every (b, KV head) (2 * D * 2 bytes per key and head),
    plus Q once.  The split partials are not counted."""
    lens = w.visible_lens().astype(np.int64)
    return int(lens.sum()) * w.Hkv * 2 * w.D * 2 + w.B * w.Hq * w.T * w.D * 2


def floors(w, peak_gbs):
    """The three lower bounds of the prefix pass at this pool's peaks (us):
    HBM (algorithmic bytes / measured copy bandwidth), tensor (the MMA work
    as issued, 128-row tiles of the G*T packed rows, / measured bf16 cuBLAS
    throughput; also the useful part alone) and exp2 (one per score / the
    exp2 unit's 16 results per clock per SM at the maximum SM clock)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        tflops, sm_mhz = float(pk["bf16_tflops"]), float(pk.get("sm_max_mhz", 1965.0))
    except Exception:
        tflops, sm_mhz = 1590.0, 1965.0
    keys = int(w.visible_lens().astype(np.int64).sum()) * w.Hkv
    rows = w.G * w.T
    padded = -(-rows // 128) * 128
    useful = 4.0 * rows * keys * w.D
    issued = 4.0 * padded * keys * w.D
    exps = float(rows * keys)
    return {"hbm_us": prefix_algorithmic_bytes(w) / (peak_gbs * 1e9) * 1e6,
            "tensor_us": issued / (tflops * 1e12) * 1e6,
            "tensor_useful_us": useful / (tflops * 1e12) * 1e6,
            "exp2_us": exps / (16 * 148 * sm_mhz * 1e6) * 1e6,
            "basis": f"measured {peak_gbs:.0f} GB/s, {tflops:.0f} TFLOP/s bf16 (burst), "
                     f"16 exp2/clk/SM x 148 SMs at {sm_mhz:.0f} MHz"}


def pct(xs, q):
    xs = sorted(xs)
    return xs[min(len(xs) - 1, max(0, int(round(q * (len(xs) - 1)))))]


def host_cpu():
    """The host the CPU baseline ran on: logical CPUs available to this
    process and the CPU model string."""
    try:
        nproc = len(os.sched_getaffinity(0))
    except AttributeError:
        nproc = os.cpu_count()
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": nproc, "cpu_model": model}


class NvmlSampler:
    """SM clock and throttle reasons read through NVML about every
    `period_s` by a background thread, so that even a timed region of a
    millisecond holds samples; only those stamped inside it are kept."""
    NAMES = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
             ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))

    def __init__(self, cuda_index, period_s=0.0005):
        import threading
        import pynvml
        self.nv = pynvml
        pynvml.nvmlInit()
        self.h = None
        try:
            pr = torch.cuda.get_device_properties(cuda_index)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            self.h = pynvml.nvmlDeviceGetHandleByIndex(cuda_index)
        self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
        self.period = period_s
        self.samples = []
        self.stop_flag = threading.Event()
        self.thread = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv, h = self.nv, self.h
        reasons_fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop_flag.is_set():
            try:
                mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                bits = int(reasons_fn(h))
            except Exception:
                break
            self.samples.append((time.time(), mhz, bits))
            time.sleep(self.period)

    def start(self):
        self.thread.start()

    def stop(self, t_begin=None, t_end=None):
        self.stop_flag.set()
        self.thread.join(timeout=2)
        try:
            self.nv.nvmlShutdown()
        except Exception:
            pass
        inside = [r for r in self.samples if t_begin is not None and t_begin <= r[0] <= t_end]
        use = inside or self.samples
        if not use:
            return None
        reasons = sorted({n for _, _, bits in use for n, m in self.NAMES if bits & m})
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": self.max_mhz,
                "samples": len(use), "samples_in_timed_region": len(inside),
                "reasons": reasons, "source": "NVML, ~0.5 ms period"}


def clock_sampler(cuda_index):
    try:
        return NvmlSampler(cuda_index)
    except Exception:
        return ClockSampler(cuda_index)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms; only the
    samples stamped inside the timed region are kept (used when NVML cannot
    be loaded)."""
    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self, t_begin=None, t_end=None):
        """Median SM clock and throttle reasons of the samples taken between
        the host wall times t_begin and t_end (all samples if none fall in)."""
        import datetime
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        rows = []
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(f[2]), float(f[3]),
                             {n for n, v in zip(names, f[6:10]) if v.lower() == "active"}))
            except ValueError:
                continue
        inside = [r for r in rows if t_begin is not None and t_begin - 0.05 <= r[0] <= t_end + 0.05]
        use = inside or rows
        if not use:
            return None
        reasons = set().union(*(r[3] for r in use))
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": use[-1][2],
                "samples": len(use), "samples_in_timed_region": len(inside),
                "reasons": sorted(reasons), "source": "nvidia-smi, 200 ms period"}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    """The largest of the ranks' values (every rank gets it)."""
    if world == 1:
        return x
    dev = "cpu" if torch.distributed.get_backend() == "gloo" else "cuda"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_us_per_call(max_elapsed_ms: float, steps: int, world: int) -> float:
    """Whole-job time per call: every rank ran `steps` calls of its own, so
    the job finished world * steps calls in the slowest rank's time."""
    return max_elapsed_ms * 1e3 / (steps * world)


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


# --------------------------------------------------------------------------
# CPU oracle: the reported baseline (cpu_baseline) and the reference arm
# --------------------------------------------------------------------------
_ORACLE_CACHE = {}


def _oracle_head_problem(w, b, kvh):
    """The oracle problem of one (b, KV head) group (B = 1, Hkv = 1)."""
    import oracle
    from tree_masked_verification_b200.inputs import bf16_bits
    key = (w.name, b, kvh)
    if key not in _ORACLE_CACHE:
        inp = w.generate_head(b, kvh)
        _ORACLE_CACHE.clear()
        if w.kind == "window":
            from oracle import window as oracle_window
            args = [bf16_bits(inp["q"]), bf16_bits(inp["k_prefix"]), bf16_bits(inp["v_prefix"]),
                    inp["prefix_len"].numpy(), bf16_bits(inp["k_tree"]), bf16_bits(inp["v_tree"]),
                    inp["parent"].numpy()]
            _ORACLE_CACHE[key] = lambda rows: oracle_window.window_attention(
                *args, w.L_cap, scale=w.scale, rows=rows)
            return _ORACLE_CACHE[key]
        _ORACLE_CACHE[key] = oracle.Problem(
            bf16_bits(inp["q"]), bf16_bits(inp["k_prefix"]), bf16_bits(inp["v_prefix"]),
            inp["prefix_len"].numpy(), bf16_bits(inp["k_tree"]), bf16_bits(inp["v_tree"]),
            inp["parent"].numpy(), scale=w.scale)
    return _ORACLE_CACHE[key]


def oracle_rows_timed(w, heads, budget_s, rows_per_head=None, row_offset=0):
    """Runs the fp64 oracle (single thread) over the packed rows of the given
    (b, KV head) groups until `budget_s` is spent; returns (seconds, rows).
    Input generation is outside the timed part."""
    done, spent = 0, 0.0
    M = w.G * w.T
    for b, kvh in heads:
        p = _oracle_head_problem(w, b, kvh)
        n = M if rows_per_head is None else min(M, rows_per_head)
        rows = np.array([[0, ((row_offset + r) % M) // w.T, ((row_offset + r) % M) % w.T]
                         for r in range(n)], dtype=np.int32)
        t0 = time.perf_counter()
        if w.kind == "prefix":
            p.prefix_partial(0, w.L_cap, rows)
        elif w.kind == "window":
            p(rows)
        else:
            p.attention(rows)
        spent += time.perf_counter() - t0
        done += n
        if spent >= budget_s:
            break
    return spent, done


def cpu_baseline(w, budget_s=10.0):
    heads = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    spent, rows = oracle_rows_timed(w, heads, budget_s)
    total_rows = w.B * w.Hq * w.T
    us_per_call = spent / rows * total_rows * 1e6
    return {"value": us_per_call, "unit": "µs", "cores": 1, "kind": "oracle", **host_cpu(),
            "sample": f"{rows} of {total_rows} query rows (whole KV-head groups, fp64, one "
                      f"thread, {spent:.1f} s), scaled to one full call"}


def run_reference(args, world, rank):
    w = WORKLOADS[args.workload]
    if rank != 0:
        return
    total_rows = w.B * w.Hq * w.T
    heads = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    # a step is a bounded sample of the call: as many query rows as keep the
    # whole run within --ref-budget seconds (at least one row, at most
    # --ref-rows), from the time of one row measured first
    spent1, _ = oracle_rows_timed(w, heads[:1], 0.0, rows_per_head=1)
    fit = int(args.ref_budget / max(1, args.warmup + args.steps) / max(spent1, 1e-9))
    per_step = max(1, min(w.G * w.T, args.ref_rows, fit))
    times = []
    for i in range(args.warmup + args.steps):
        spent, rows = oracle_rows_timed(w, heads[:1], 0.0, rows_per_head=per_step,
                                        row_offset=i * per_step)
        if i >= args.warmup:
            times.append(spent / rows)
    sec_per_row = sum(times) / len(times)
    us = sec_per_row * total_rows * 1e6
    line = {
        "impl": "reference", "metric": METRIC, "value": us, "unit": "µs",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sec_per_row * per_step * 1e3, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, None, 1),
        "cpu_baseline": {"value": us, "unit": "µs", "cores": 1, "kind": "oracle", **host_cpu(),
                         "sample": f"{per_step} query rows per step of {total_rows}, fp64, "
                                   f"one thread, scaled to one full call"},
        "e2e": {"value": us, "unit": "µs", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------
def run_ours(args, world, rank, local):
    w = WORKLOADS[args.workload]
    if args.block_size >= 0:
        w = w.replace(block_size=args.block_size)
    dev = torch.device("cuda", torch.cuda.current_device())
    cpu = w.generate()
    if w.block_size:
        cpu["k_cache"], cpu["v_cache"], cpu["block_table"] = paged_cache(
            cpu["k_prefix"], cpu["v_prefix"], cpu["prefix_len"].tolist(), w.block_size, w.seed)
    kv_bytes = 2 * cpu["k_prefix"].numel() * 2
    n_sets = 1 if kv_bytes > 2 * L2_BYTES else int(math.ceil(2 * L2_BYTES / kv_bytes)) + 1
    sets = []
    base = {k: v.to(dev) for k, v in cpu.items()}
    for i in range(n_sets):
        sets.append(base if i == 0 else {k: v.clone() for k, v in base.items()})
    dims = hta.dims_of(base["q"], base["k_prefix"], w.scale)
    S, chunk = hta.chunking(dims, args.num_splits)
    ws = hta.new_workspace(dims, args.num_splits, dev)
    if w.kind == "window":   # one chunk: the window's W/128 + 1 tiles
        S, chunk = 1, (w.L_cap // 128 + 1) * 128
        ws = hta.new_window_workspace(dims, dev)
    out = torch.empty_like(base["q"])
    lse = torch.empty(base["q"].shape[:3], dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def call(i, events=None):
        s = sets[i % n_sets]
        if w.block_size:
            fn = hta.prefix_attention_paged if w.kind == "prefix" else hta.verify_paged
            tree = () if w.kind == "prefix" else (s["k_tree"], s["v_tree"], s["parent"])
            fn(s["q"], s["k_cache"], s["v_cache"], s["block_table"], s["prefix_len"], *tree,
               L_cap=w.L_cap, out=out, lse=lse, workspace=ws, scale=w.scale,
               num_splits=args.num_splits, prefix_events=events, stream=stream)
        elif w.kind == "prefix":
            hta.prefix_attention(s["q"], s["k_prefix"], s["v_prefix"], s["prefix_len"], out=out,
                                 lse=lse, workspace=ws, scale=w.scale, num_splits=args.num_splits,
                                 prefix_events=events, stream=stream)
        elif w.kind == "window":
            if events is not None:
                events[0].record(stream)
            hta.window_verify(s["q"], s["k_prefix"], s["v_prefix"], s["prefix_len"], s["k_tree"],
                              s["v_tree"], s["parent"], out=out, lse=lse, workspace=ws,
                              scale=w.scale, stream=stream)
            if events is not None:    # around the whole call: no hook between its kernels
                events[1].record(stream)
        else:
            hta.verify(s["q"], s["k_prefix"], s["v_prefix"], s["prefix_len"], s["k_tree"],
                       s["v_tree"], s["parent"], out=out, lse=lse, workspace=ws, scale=w.scale,
                       num_splits=args.num_splits, prefix_events=events, stream=stream)

    for i in range(args.warmup):
        call(i)
    torch.cuda.synchronize()
    if hta.get_status(ws) != hta.OK:
        raise RuntimeError("device status error during warm-up")

    # --graph: the timed calls replay a CUDA graph of G calls (G divides K),
    # so the host's per-call cost (binding, checks, launches) is paid once
    graph, G = None, 1
    if args.graph:
        G = max(d for d in range(1, min(args.steps, 200) + 1) if args.steps % d == 0)
        graph = torch.cuda.CUDAGraph()
        cap, saved = torch.cuda.Stream(), stream
        cap.wait_stream(saved)
        stream = cap                      # the calls below launch on the capture stream
        with torch.cuda.graph(graph, stream=cap):
            for i in range(G):
                call(i)
        stream = saved
        graph.replay()
        torch.cuda.synchronize()
        if hta.get_status(ws) != hta.OK:
            raise RuntimeError("device status error in the graph warm-up")

    # timed region 1 (the headline): back-to-back calls, nothing between the
    # two kernels of a call (an event there would serialise them)
    sampler = clock_sampler(local if world > 1 else 0)
    sampler.start()
    time.sleep(0.3)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    wall0 = time.time()
    t_start.record(stream)
    if graph is not None:
        for _ in range(args.steps // G):
            graph.replay()
    else:
        for i in range(args.steps):
            call(i)
    t_end.record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    barrier(world)
    clocks = sampler.stop(wall0, wall1)
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_end), world)
    if hta.get_status(ws) != hta.OK:
        raise RuntimeError("device status error in the timed region")

    # timed region 2 (the roofline): the same calls with CUDA events recorded
    # around the prefix kernel on the launching stream
    n2 = min(args.steps, 2000)   # calls of the second pass (per-call events)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(n2)]
    ev_end = [torch.cuda.Event(enable_timing=True) for _ in range(n2)]
    for (a, b), c in zip(ev, ev_end):   # torch creates the CUDA event on first record
        a.record(stream)
        b.record(stream)
        c.record(stream)
    barrier(world)
    torch.cuda.synchronize()
    for i in range(n2):
        call(i, ev[i])
        ev_end[i].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    prefix_ms = [a.elapsed_time(b) for a, b in ev]
    call_ms = [a.elapsed_time(c) for (a, _), c in zip(ev, ev_end)]
    prefix_avg_ms = max_over_ranks(sum(prefix_ms) / len(prefix_ms), world)
    if hta.get_status(ws) != hta.OK:
        raise RuntimeError("device status error in the roofline region")

    # host cost of one call (argument checks, tensor-map lookup, launches),
    # the GPU running behind it
    torch.cuda.synchronize()
    n_host = min(args.steps, 100)
    h0 = time.perf_counter()
    for i in range(n_host):
        call(i)
    host_us = (time.perf_counter() - h0) / n_host * 1e6
    torch.cuda.synchronize()
    c_abi_us = c_abi_host_us(w, sets[0], out, lse, ws, dims, stream, n_host, args.num_splits)
    torch.cuda.synchronize()

    ms_per_step = elapsed_ms / args.steps
    us_per_call = job_us_per_call(elapsed_ms, args.steps, world)
    peak, peak_kind = peaks()
    pbytes = prefix_algorithmic_bytes(w)
    achieved = pbytes / (prefix_avg_ms * 1e-3) / 1e9
    call_bytes = w.algorithmic_bytes()

    # end to end through the host-buffer entry point (copies inside the region)
    e2e = run_e2e(args, w, cpu, dims, dev, stream, world)

    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": us_per_call, "unit": "µs", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": f"synthetic (seeded N(0,1) bf16; tree: {workload_config(w, S, n_sets)['tree']})",
        "config": {**workload_config(w, S, n_sets),
                   "launch": f"CUDA graph of {G} calls, replayed" if graph is not None else "eager"},
        "roofline": {"bound": "hbm", "kernel": "prefix_tc_kernel", "achieved": achieved,
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": profiled_traffic(w.name),
                     "algorithmic_bytes": pbytes, "avg_launch_us": prefix_avg_ms * 1e3},
        "call_roofline": {"bytes": call_bytes, "achieved_gbs": call_bytes / (ms_per_step * 1e-3) / 1e9,
                          "frac_measured": call_bytes / (ms_per_step * 1e-3) / 1e9 / peak,
                          "frac_nominal_8tbs": call_bytes / (ms_per_step * 1e-3) / 8e12},
        "distribution": {
            "call_us": {"p10": pct(call_ms, 0.1) * 1e3, "p50": pct(call_ms, 0.5) * 1e3,
                        "p90": pct(call_ms, 0.9) * 1e3},
            "prefix_us": {"p10": pct(prefix_ms, 0.1) * 1e3, "p50": pct(prefix_ms, 0.5) * 1e3,
                          "p90": pct(prefix_ms, 0.9) * 1e3},
            "host_api_us_per_call": host_us,
            "c_abi_host_us_per_call": c_abi_us,
            "note": "per-call CUDA events of the roofline pass (events between the kernels "
                    "serialise them, so these run a little above the headline value)"},
        "floors": floors(w, peak),
        "gpu_launches": 2 * args.steps,
        "timing": "value: CUDA events around the K back-to-back calls; roofline: a second pass "
                  "of the same calls with events around each prefix launch",
        "build": {"library": os.path.basename(hta.library_path()), **hta.build_info()},
        "clocks": clocks,
        "e2e": e2e,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_budget)
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------
# greedy acceptance (the step after a verification call)
# --------------------------------------------------------------------------
def run_accept(args, world, rank, local):
    """Latency of one greedy-acceptance call: argmax of B*(T+1) logits rows
    of V bf16 values, then the tree walk.  HBM-bound on the logits read."""
    B, T, V = ACCEPT_WORKLOADS[args.accept]
    dev = torch.device("cuda", torch.cuda.current_device())
    cpu = accept_inputs(B, T, V, seed=17 + rank, p_match=0.8)
    lbytes = cpu["logits"].numel() * 2
    n_sets = int(math.ceil(2 * L2_BYTES / lbytes)) + 1
    base = {k: cpu[k].to(dev) for k in ("logits", "draft_tokens", "parent")}
    sets = [base] + [{k: v.clone() for k, v in base.items()} for _ in range(n_sets - 1)]
    ws = hta.new_accept_workspace(B, T, V, dev)
    n_acc = torch.empty(B, dtype=torch.int32, device=dev)
    path = torch.empty(B, T, dtype=torch.int32, device=dev)
    bonus = torch.empty(B, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def call(i):
        s = sets[i % n_sets]
        hta.accept_greedy(s["logits"], s["draft_tokens"], s["parent"], accept_len=n_acc, path=path,
                          bonus=bonus, workspace=ws, stream=stream)

    for i in range(args.warmup):
        call(i)
    torch.cuda.synchronize()
    if hta.get_status(ws) != hta.OK:
        raise RuntimeError("device status error during warm-up")
    graph, G = None, 1
    if args.graph:   # replays of a CUDA graph of G calls (G divides K)
        G = max(d for d in range(1, min(args.steps, 200) + 1) if args.steps % d == 0)
        graph = torch.cuda.CUDAGraph()
        cap, saved = torch.cuda.Stream(), stream
        cap.wait_stream(saved)
        stream = cap
        with torch.cuda.graph(graph, stream=cap):
            for i in range(G):
                call(i)
        stream = saved
        graph.replay()
        torch.cuda.synchronize()
        if hta.get_status(ws) != hta.OK:
            raise RuntimeError("device status error in the graph warm-up")
    sampler = clock_sampler(local if world > 1 else 0)
    sampler.start()
    time.sleep(0.3)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    wall0 = time.time()
    t0.record(stream)
    if graph is not None:
        for _ in range(args.steps // G):
            graph.replay()
    else:
        for i in range(args.steps):
            call(i)
    t1.record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    barrier(world)
    clocks = sampler.stop(wall0, wall1)
    elapsed_ms = max_over_ranks(t0.elapsed_time(t1), world)
    if hta.get_status(ws) != hta.OK:
        raise RuntimeError("device status error in the timed region")

    # acceptance followed by the KV commit of the accepted path (8 KV heads,
    # D 128, contiguous cache) on the device, back to back: every call
    # appends up to (tree depth) rows, so the cache is sized for all calls
    Hkv, D = 8, 128
    n_pipe = min(args.steps, 2000)
    par = cpu["parent"].numpy()
    depth = np.zeros(par.shape, dtype=np.int64)
    for i in range(T):
        depth[:, i] = np.where(par[:, i] < 0, 1, depth[np.arange(B), np.maximum(par[:, i], 0)] + 1)
    L_cap = int((n_pipe + args.warmup + 1) * depth.max())
    kcache = torch.zeros(B, Hkv, L_cap, D, dtype=torch.bfloat16, device=dev)
    vcache = torch.zeros_like(kcache)
    ktree = torch.randn(B, Hkv, T, D, device=dev).to(torch.bfloat16)
    vtree = torch.randn_like(ktree)
    lens = torch.zeros(B, dtype=torch.int32, device=dev)

    def pipe(i):
        call(i)
        hta.commit(kcache, vcache, lens, ktree, vtree, n_acc, path, workspace=ws, stream=stream)

    for i in range(args.warmup):
        pipe(i)
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    p0.record(stream)
    for i in range(n_pipe):
        pipe(i)
    p1.record(stream)
    torch.cuda.synchronize()
    pipe_ms = max_over_ranks(p0.elapsed_time(p1), world)
    if hta.get_status(ws) != hta.OK:
        raise RuntimeError("device status error in the accept + commit region")

    # end to end: logits, tokens and parents from pinned host memory, the
    # three results back to the host, every call
    host = {k: cpu[k].pin_memory() for k in ("logits", "draft_tokens", "parent")}
    n_e2e = min(args.e2e_steps * 10, args.steps)
    outs = [torch.empty(B, dtype=torch.int32).pin_memory(), torch.empty(B, T, dtype=torch.int32).pin_memory(),
            torch.empty(B, dtype=torch.int32).pin_memory()]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(n_e2e):
        s = sets[i % n_sets]
        for k in host:
            s[k].copy_(host[k], non_blocking=True)
        call(i)
        for o, d in zip(outs, (n_acc, path, bonus)):
            o.copy_(d, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)

    if rank != 0:
        return
    us = job_us_per_call(elapsed_ms, args.steps, world)
    peak, peak_kind = peaks()
    abytes = lbytes + 2 * B * T * 4 + 3 * B * 4 + B * T * 4
    achieved = abytes / (elapsed_ms / args.steps * 1e-3) / 1e9
    line = {
        "metric": "greedy tree acceptance latency per call", "value": us, "unit": "µs",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": elapsed_ms / args.steps, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) logits, one planted "
        "maximum per row; LongSpec 4/16/16/16/16 tree; draft token = parent row's maximum w.p. 0.8)",
        "config": {"workload": args.accept, "B": B, "T": T, "V": V, "input_sets": n_sets,
                   "launch": f"CUDA graph of {G} calls, replayed" if graph is not None else "eager",
                   "l2": f"{n_sets} rotating logits sets ({n_sets * lbytes / 1e6:.0f} MB > L2)"},
        "roofline": {"bound": "hbm", "kernel": "argmax_slices_kernel + accept_kernel",
                     "achieved": achieved, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": None, "algorithmic_bytes": abytes},
        "gpu_launches": 2 * args.steps,
        "clocks": clocks,
        "accept_then_commit": {
            "us_per_call": job_us_per_call(pipe_ms, n_pipe, world), "calls": n_pipe,
            "gpu_launches": 3 * n_pipe,
            "note": "accept_greedy + commit (8 KV heads, D 128, contiguous cache) per call, "
                    "back to back; the prefix grows by the accepted length every call"},
        "e2e": {"value": job_us_per_call(e2e_ms, n_e2e, world), "unit": "µs",
                "h2d_bytes_per_step": sum(v.numel() * v.element_size() for v in host.values()),
                "d2h_bytes_per_step": sum(o.numel() * 4 for o in outs), "steps": n_e2e},
    }
    if world == 1 and not args.no_cpu_baseline:
        import oracle.accept as oracle_accept
        bits = bf16_bits(cpu["logits"])
        tok, par = cpu["draft_tokens"].numpy(), cpu["parent"].numpy()
        n, t_cpu = 0, time.perf_counter()
        while n == 0 or time.perf_counter() - t_cpu < min(args.cpu_budget, 5.0):
            oracle_accept.accept_greedy(bits, tok, par)
            n += 1
        line["cpu_baseline"] = {"value": (time.perf_counter() - t_cpu) / n * 1e6, "unit": "µs",
                                "cores": 1, "kind": "oracle", **host_cpu(),
                                "sample": f"{n} whole calls of the numpy oracle on the same inputs"}
    print(json.dumps(line), flush=True)


def c_abi_host_us(w, s, out, lse, ws, dims, stream, n, num_splits=0):
    """Host time of one longspec_hta_verify_ex call on its own: the C entry
    point called in a loop with its arguments converted once, so the figure
    holds the library's checks, tensor-map lookups and launches but not the
    Python binding's marshalling (the GPU runs behind).  None for calls other
    than the contiguous verification."""
    import ctypes
    if w.kind != "verify" or w.block_size:
        return None
    fn = hta.load().longspec_hta_verify_ex
    opts = hta.Options(num_splits, hta.PREFIX_TCGEN05, None, None)
    args = (ctypes.byref(dims), s["q"].data_ptr(), s["k_prefix"].data_ptr(), s["v_prefix"].data_ptr(),
            s["prefix_len"].data_ptr(), s["k_tree"].data_ptr(), s["v_tree"].data_ptr(),
            s["parent"].data_ptr(), out.data_ptr(), lse.data_ptr(), ws.data_ptr(),
            ws.numel(), ctypes.byref(opts), stream.cuda_stream)
    if fn(*args) != hta.OK:
        raise RuntimeError("longspec_hta_verify_ex failed")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(n):
        fn(*args)
    return (time.perf_counter() - t0) / n * 1e6


def run_e2e(args, w, cpu, dims, dev, stream, world):
    if w.block_size:
        names = ("q", "k_cache", "v_cache", "block_table", "prefix_len") + (
            () if w.kind == "prefix" else ("k_tree", "v_tree", "parent"))
    elif w.kind == "prefix":
        names = ("q", "k_prefix", "v_prefix", "prefix_len")
    elif w.kind == "window":
        names = ("q", "k_prefix", "v_prefix", "prefix_len", "k_tree", "v_tree", "parent")
    else:
        names = tuple(cpu.keys())
    host = {k: cpu[k].pin_memory() for k in names}
    out = torch.empty_like(host["q"]).pin_memory()
    lse = torch.empty(host["q"].shape[:3], dtype=torch.float32).pin_memory()
    if w.kind in ("prefix", "window") or w.block_size:
        # no host-buffer entry point for these calls: the same copies in and
        # out around the device call, all on `stream`
        dsts = {k: torch.empty_like(v, device=dev) for k, v in host.items()}
        dout = torch.empty_like(dsts["q"])
        dlse = torch.empty(dsts["q"].shape[:3], dtype=torch.float32, device=dev)
        ws = (hta.new_window_workspace(dims, dev) if w.kind == "window"
              else hta.new_workspace(dims, args.num_splits, dev))

        def device_call():
            s = dsts
            if w.block_size:
                fn = hta.prefix_attention_paged if w.kind == "prefix" else hta.verify_paged
                tree = () if w.kind == "prefix" else (s["k_tree"], s["v_tree"], s["parent"])
                fn(s["q"], s["k_cache"], s["v_cache"], s["block_table"], s["prefix_len"], *tree,
                   L_cap=w.L_cap, out=dout, lse=dlse, workspace=ws, scale=w.scale,
                   num_splits=args.num_splits, stream=stream)
            elif w.kind == "window":
                hta.window_verify(s["q"], s["k_prefix"], s["v_prefix"], s["prefix_len"], s["k_tree"],
                                  s["v_tree"], s["parent"], out=dout, lse=dlse, workspace=ws,
                                  scale=w.scale, stream=stream)
            else:
                hta.prefix_attention(s["q"], s["k_prefix"], s["v_prefix"], s["prefix_len"], out=dout,
                                     lse=dlse, workspace=ws, scale=w.scale,
                                     num_splits=args.num_splits, stream=stream)

        def call():
            with torch.cuda.stream(stream):
                for k, v in host.items():
                    dsts[k].copy_(v, non_blocking=True)
                device_call()
                out.copy_(dout, non_blocking=True)
                lse.copy_(dlse, non_blocking=True)
    else:
        arena = torch.empty(hta.host_arena_bytes(dims), dtype=torch.uint8, device=dev)

        def call():
            hta.verify_host(host["q"], host["k_prefix"], host["v_prefix"], host["prefix_len"],
                            host["k_tree"], host["v_tree"], host["parent"], out, lse, arena,
                            scale=w.scale, stream=stream)

    steps = max(1, min(args.steps, args.e2e_steps))
    for _ in range(min(args.warmup, 3)):
        call()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(steps):
        call()
    b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms_max = max_over_ranks(a.elapsed_time(b), world)
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out.numel() * out.element_size() + lse.numel() * lse.element_size()
    return {"value": job_us_per_call(ms_max, steps, world), "unit": "µs", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama3-8b-32k", choices=sorted(WORKLOADS))
    ap.add_argument("--num-splits", type=int, default=0)
    ap.add_argument("--block-size", type=int, default=-1,
                    help="paged prefix cache block size for the workload (0 = contiguous; "
                         "default: the workload's own)")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--ref-rows", type=int, default=16)
    ap.add_argument("--ref-budget", type=float, default=120.0,
                    help="seconds of oracle work for the whole --impl reference run")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--graph", action="store_true",
                    help="time the calls as replays of a captured CUDA graph")
    ap.add_argument("--accept", default=None, choices=sorted(ACCEPT_WORKLOADS),
                    help="time greedy acceptance on this workload instead of attention")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.accept:
            run_accept(args, world, rank, local)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
