"""Benchmark: exact attention forward TFLOP/s on B200 (bf16, causal counts half
the FLOPs), as a fraction of the measured dense-bf16 tensor-core peak.

One step = one forward of the whole workload (one kernel launch) on inputs
already resident in device memory.  Default workload: the Llama-style GQA
causal layer, B=2, Hq=32, Hkv=8, N=8192, d=128, K scaled by 2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mine|reference]

With N > 1 (launched by torch.distributed.run) every rank runs its own
replica of the workload on its own GPU; there is no data exchange between
ranks (the work units are independent), so scaling is weak.  With
`--shard heads` the ranks instead split one problem by kv-head groups
(strong scaling); one NCCL all-gather of O after the timed region reports
what collecting it costs.  Rank 0 prints one JSON line.  `--impl reference`
times the CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_io_aware_92_b200 import workloads as wl  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}


# Cycles of the spin kernel queued before each single-call start event (about
# 0.5 ms at B200 clocks).  The GPU is still busy with it while the host
# queues the timed call, so the events measure device time only and not the
# host's call overhead.
LAUNCH_COVER_CYCLES = 1_000_000


def flush_l2(buf):
    """Evict the L2 between timed calls: write `buf` (256 MiB, twice the L2),
    then read it back, so that the write-backs of its dirty lines happen here
    and not inside the next timed call."""
    buf.zero_()
    buf.sum()


def record_start(ev):
    """Record a start event behind a spin kernel (LAUNCH_COVER_CYCLES)."""
    import torch
    torch.cuda._sleep(LAUNCH_COVER_CYCLES)
    ev.record()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return FALLBACK_PEAKS, "fallback"


def kernel_source_hash() -> str:
    """sha256[:16] of what defines the timed forward kernel and its launch:
    the kernel header, the PTX helpers, and the host functions that build
    its tensor maps and launch it (their text in fa_api.cu)."""
    import hashlib
    import re
    csrc = os.path.join(ROOT, "exact_io_aware_92_b200", "csrc")
    h = hashlib.sha256()
    for name in ("fa_fwd_sm100.cuh", "sm100_ptx.cuh"):
        with open(os.path.join(csrc, name), "rb") as fh:
            h.update(fh.read())
    with open(os.path.join(csrc, "fa_api.cu")) as fh:
        api = fh.read()
    for head in (r"\nint make_map\(", r"\ntemplate <int D>\nint launch_bf16\("):
        m = re.search(head + r".*?\n}\n", api, re.S)
        if m is None:
            raise RuntimeError(f"kernel_source_hash: {head!r} not found in fa_api.cu")
        h.update(m.group(0).encode())
    return h.hexdigest()[:16]


def dist_env():
    """(rank, world size, local rank) from the launcher's environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def replica_seed(w: wl.Workload, rank: int) -> int:
    """Each rank times its own replica of the workload, drawn from its own seed."""
    return w.seed + 1000 * rank


def reduce_max(x: float, device) -> float:
    """Max of x over the ranks of the default process group (x itself
    without one): the slowest rank sets the job's time."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(flops_per_step: float, steps: int, ms_max: float, world: int) -> float:
    """Whole-job TFLOP/s: `world` replicas each ran `steps` steps in at most
    ms_max milliseconds."""
    return world * flops_per_step * steps / (ms_max * 1e-3) / 1e12


def head_shard(Hkv: int, group: int, world: int, rank: int):
    """Head sharding of one problem: rank r takes the kv heads [g0, g1) and
    the query heads [h0, h1) = [g0 * group, g1 * group) that share them, so
    no rank needs another's K or V (work units are independent)."""
    if Hkv % world:
        raise ValueError(f"{Hkv} kv heads do not split over {world} ranks")
    per = Hkv // world
    g0, g1 = rank * per, (rank + 1) * per
    return g0, g1, g0 * group, g1 * group


def assemble_heads(parts):
    """O (or LSE) of the whole problem from the ranks' head slices, given in
    rank order: the slices are concatenated along the head axis (axis 1)."""
    import torch
    return torch.cat(list(parts), dim=1)


class ClockSampler:
    """SM clock, power and clock-event reasons of the GPU the timed region runs
    on, sampled every 10 ms through NVML in a background thread.  The device is
    found by the UUID torch reports (CUDA_VISIBLE_DEVICES renumbers devices,
    NVML does not).  Only samples taken between region_start() and
    region_stop() are reported; without NVML the record says so.  Reading
    only: nothing here changes a setting of the GPU."""
    # every clock-event reason bit NVML defines, by the name the report uses
    REASONS = (("gpu_idle", 0x1), ("applications_clocks_setting", 0x2), ("sw_power_cap", 0x4),
               ("hw_slowdown", 0x8), ("sync_boost", 0x10), ("sw_thermal_slowdown", 0x20),
               ("hw_thermal_slowdown", 0x40), ("hw_power_brake_slowdown", 0x80),
               ("display_clock_setting", 0x100))

    def __init__(self, torch_index: int):
        import threading
        self.samples = []  # (t, sm_mhz, power_w, reasons bitmask)
        self.t0 = self.t1 = None
        self.stop_evt = threading.Event()
        self.thread = None
        self.nvml = None
        self.handle = None
        self.max_mhz = None
        self.instant_field = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(torch_index).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle,
                                                                  pynvml.NVML_CLOCK_SM))
            self.instant_field = getattr(pynvml, "NVML_FI_DEV_POWER_INSTANT", None)
            self.nvml = pynvml
        except Exception:
            self.nvml = None

    def _power_w(self):
        """(board power as nvidia-smi's power.draw reports it, averaged by the
        driver over about a second; NVML's instantaneous power field where it
        exists, else None).  The instantaneous field updates far more slowly
        than the 10 ms sampling, so only its maximum is reported."""
        nv = self.nvml
        avg = nv.nvmlDeviceGetPowerUsage(self.handle) / 1000.0
        inst = None
        if self.instant_field is not None:
            try:
                v = nv.nvmlDeviceGetFieldValues(self.handle, [self.instant_field])[0]
                if v.nvmlReturn == nv.NVML_SUCCESS:
                    inst = float(v.value.uiVal) / 1000.0
            except Exception:
                inst = None
        return avg, inst

    def _run(self):
        nv = self.nvml
        while not self.stop_evt.is_set():
            try:
                t = time.monotonic()
                sm = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                pw = self._power_w()
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append((t, float(sm), pw, int(rs)))
            except Exception:
                pass
            self.stop_evt.wait(self.PERIOD_S)

    # Poll period.  A contract region of 20 launches lasts under 20 ms, so the
    # sampler polls every millisecond to see the clocks inside it.
    PERIOD_S = 0.001

    def start(self):
        import threading
        if self.nvml is not None:
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()

    def region_start(self):
        self.t0 = time.monotonic()

    def region_stop(self):
        self.t1 = time.monotonic()

    def stop(self):
        if self.nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        self.stop_evt.set()
        self.thread.join(timeout=5)
        inside = [x for x in self.samples
                  if self.t0 is not None and self.t1 is not None and self.t0 <= x[0] <= self.t1]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples"]}
        reasons = set()
        for _, _, _, rs in inside:
            for name, bit in self.REASONS:
                if rs & bit:
                    reasons.add(name)
        sm = [x[1] for x in inside]
        pw = [x[2][0] for x in inside]
        inst = [x[2][1] for x in inside if x[2][1] is not None]
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.max_mhz,
                "sm_mhz_min": min(sm), "reasons": sorted(reasons), "samples": len(inside),
                "power_w_1s_avg_median": statistics.median(pw),
                "power_w_1s_avg_max": max(pw),
                "power_w_instant_max": max(inst) if inst else None,
                "source": f"NVML, every {self.PERIOD_S * 1e3:g} ms, timed region only"}


def oracle_sample_rows(w: wl.Workload, rows_per_head: int, seed: int = 1234) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return np.stack([np.sort(rng.choice(w.N, rows_per_head, replace=False))
                     for _ in range(w.B * w.Hq)])


def sample_flops(w: wl.Workload, rows: np.ndarray, seqlens) -> float:
    """Metric FLOPs of the sampled query rows: 4*d per visible key, with the
    causal count halved as the metric defines it (whole rows otherwise)."""
    total = 0.0
    for bh in range(rows.shape[0]):
        L = w.N if seqlens is None else int(seqlens[bh // w.Hq])
        total += 4.0 * w.d * L * rows.shape[1]
    return total / 2 if w.causal else total


def oracle_sample(w: wl.Workload, inp: wl.Inputs, target_s: float):
    """A seeded sample of query rows per (batch, head) on which one oracle run
    takes about target_s on this host (at least 4 rows per head, at most all
    rows): the sample doubles, or jumps to the estimated size, until a run
    reaches a quarter of the target."""
    import oracle
    threads = oracle.num_threads()
    scale = float(np.float32(w.scale))
    rows_per_head = 4
    while True:
        rows = oracle_sample_rows(w, rows_per_head)
        t0 = time.perf_counter()
        oracle.attention_forward(inp.q_bits, inp.k_bits, inp.v_bits, causal=w.causal, scale=scale,
                                 seqlens=inp.seqlens, rows=rows, threads=threads)
        dt = time.perf_counter() - t0
        if dt > target_s / 4 or rows_per_head >= w.N:
            return rows, rows_per_head, dt, threads
        rows_per_head = min(w.N, rows_per_head * max(2, int(target_s / 4 / max(dt, 1e-3))))


def run_oracle_rows(w: wl.Workload, inp: wl.Inputs, rows, threads) -> float:
    """Seconds for one oracle run on the given query rows."""
    import oracle
    t0 = time.perf_counter()
    oracle.attention_forward(inp.q_bits, inp.k_bits, inp.v_bits, causal=w.causal,
                             scale=float(np.float32(w.scale)), seqlens=inp.seqlens, rows=rows,
                             threads=threads)
    return time.perf_counter() - t0


def time_oracle(w: wl.Workload, inp: wl.Inputs, budget_s: float):
    """The CPU oracle on a bounded sample of query rows of the same workload."""
    rows, rows_per_head, dt, threads = oracle_sample(w, inp, budget_s)
    f = sample_flops(w, rows, inp.seqlens)
    return {"value": f / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"{rows_per_head} seeded query rows per (batch, head) of {w.name} "
                      f"({rows.size} rows, every visible key), {dt:.1f} s wall"}, dt


# The reference arm's whole warm-up + timed run stays within about this many
# seconds, whatever --steps and --warmup are.
REF_TOTAL_S = 150.0


def run_reference(args, w: wl.Workload):
    """The oracle as the reference arm: one run on a fixed row sample per step,
    the sample sized so that all warm-up and timed steps fit REF_TOTAL_S."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    inp = wl.draw_workload(w)
    total = args.warmup + args.steps
    target = max(0.05, min(args.ref_budget, REF_TOTAL_S / max(total, 1)))
    rows, rows_per_head, _, threads = oracle_sample(w, inp, target)
    f = sample_flops(w, rows, inp.seqlens)
    per_step = []
    for s in range(total):
        dt = run_oracle_rows(w, inp, rows, threads)
        if s >= args.warmup:
            per_step.append(dt)
    ms = statistics.median(per_step) * 1e3
    value = f / (ms * 1e-3) / 1e12
    cpu = {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
           "sample": f"{rows_per_head} seeded query rows per (batch, head) of {w.name} "
                     f"({rows.size} rows, every visible key) per step; median of "
                     f"{len(per_step)} timed steps of {ms / 1e3:.2f} s"}
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded, bf16-rounded N(0,1))",
        "config": workload_config(w),
        "cpu_baseline": cpu,
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


METRIC = "attention fwd TFLOP/s (bf16, causal=1/2 FLOPs) and % of B200 dense BF16 peak"
# Second denominator: NVIDIA's per-GPU B200 BF16 figure (4.5 PFLOP/s) assumes 2:4
# sparsity; the dense figure is half of it.
NOMINAL_BF16_TFLOPS = 2250.0


def workload_config(w: wl.Workload):
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d,
            "causal": w.causal, "k_scale": w.k_scale, "scale": w.scale,
            "seqlens": None if w.seqlen_range is None else f"uniform {w.seqlen_range}"}


def run_mine(args, w: wl.Workload):
    import torch
    import torch.distributed as dist
    from exact_io_aware_92_b200 import _lib, attention

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    heads = args.shard == "heads"
    if heads:
        # One problem split by kv-head groups: every rank draws the same
        # inputs and keeps its heads.
        inp = wl.draw(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed, k_scale=w.k_scale,
                      seqlen_range=w.seqlen_range)
        g0, g1, h0, h1 = head_shard(w.Hkv, w.Hq // w.Hkv, world, rank)
        inp.q_bits = np.ascontiguousarray(inp.q_bits[:, h0:h1])
        inp.k_bits = np.ascontiguousarray(inp.k_bits[:, g0:g1])
        inp.v_bits = np.ascontiguousarray(inp.v_bits[:, g0:g1])
    else:
        # Each rank: its own replica of the workload (seed offset by rank).
        inp = wl.draw(w.B, w.Hq, w.Hkv, w.N, w.d, replica_seed(w, rank), k_scale=w.k_scale,
                      seqlen_range=w.seqlen_range)
    q, k, v = (torch.from_numpy(x).view(torch.bfloat16).to(dev)
               for x in (inp.q_bits, inp.k_bits, inp.v_bits))
    sl = None if inp.seqlens is None else torch.from_numpy(inp.seqlens).to(dev)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flops = wl.flops(w, inp.seqlens)
    if heads:
        flops = flops * q.shape[1] / w.Hq  # this rank's share of the problem
    # whole-job throughput: replicas add up; shards of one problem do not
    job_world = 1 if heads else world
    job_flops = flops * world if heads else flops
    in_bytes = sum(t.numel() * t.element_size() for t in (q, k, v))
    stream = torch.cuda.current_stream(dev)

    def step():
        attention.fwd(q, k, v, causal=w.causal, scale=w.scale, seqlens=sl, out=o, lse=lse,
                      status=status)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if attention.check_status(status) != 0:
        raise RuntimeError("kernel reported a time-out during warm-up")

    sampler = ClockSampler(local)
    barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # The region opens before the first launch is queued: the GPU starts on
    # it at once, so samples from here on fall inside the timed launches.
    sampler.region_start()
    start.record(stream)
    for _ in range(args.steps):
        step()
    end.record(stream)
    end.synchronize()
    sampler.region_stop()
    torch.cuda.synchronize(dev)
    barrier()
    clocks = sampler.stop()
    ms_total = start.elapsed_time(end)
    if attention.check_status(status) != 0:
        raise RuntimeError("kernel reported a time-out in the timed region")
    ms_max = reduce_max(ms_total, dev)
    ms_per_step = ms_max / args.steps
    value = job_throughput(job_flops, args.steps, ms_max, job_world)
    gather_ms = None
    if heads and world > 1:
        # One all-gather (NCCL) brings O to every rank in head order; timed
        # apart from the forward, as the cost a caller pays to collect it.
        parts = [torch.empty_like(o) for _ in range(world)]
        g_0, g_1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        g_0.record(stream)
        dist.all_gather(parts, o)
        full_o = assemble_heads(parts)
        g_1.record(stream)
        torch.cuda.synchronize(dev)
        gather_ms = reduce_max(g_0.elapsed_time(g_1), dev)
        assert full_o.shape[1] == w.Hq
        del parts, full_o
    kernel_tflops = flops / (ms_total / args.steps * 1e-3) / 1e12

    # End to end through the C ABI on host buffers: pinned host inputs are
    # copied in, the forward runs, O and LSE are copied back, every step.
    q_h, k_h, v_h = (torch.from_numpy(x).pin_memory() for x in (inp.q_bits, inp.k_bits, inp.v_bits))
    o_h = torch.empty(q_h.shape, dtype=torch.int16).pin_memory()
    lse_h = torch.empty(lse.shape, dtype=torch.float32).pin_memory()
    sl_h = None if inp.seqlens is None else torch.from_numpy(inp.seqlens).pin_memory()
    # Steps through the asynchronous host-buffer call: each queues its copies
    # in, its forward and its copies out of O and LSE; consecutive steps are
    # chained (the next step's copies in overlap this step's tail).  The
    # stream is synchronised once after the last step.
    e2e_steps = max(2, min(args.steps, 10))
    for _ in range(2):
        attention.fwd_hostio(q_h, k_h, v_h, o_h, lse_h, q, k, v, o, lse, causal=w.causal,
                             scale=w.scale, seqlens_h=sl_h, seqlens_d=sl)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        attention.fwd_hostio(q_h, k_h, v_h, o_h, lse_h, q, k, v, o, lse, causal=w.causal,
                             scale=w.scale, seqlens_h=sl_h, seqlens_d=sl, wait=False)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    if attention.check_status() != 0:
        raise RuntimeError("kernel reported a time-out in the end-to-end leg")
    e2e_ms = reduce_max(e0.elapsed_time(e1), dev)
    e2e_value = job_throughput(job_flops, e2e_steps, e2e_ms, job_world)
    h2d = in_bytes + (0 if sl is None else sl.numel() * 4)
    d2h = o.numel() * 2 + lse.numel() * 4
    # The copy rates of this host link alone (plain pinned copies of the same
    # bytes, one direction at a time): what bounds the end-to-end step.
    c0, c1, c2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    c0.record(stream)
    for t_d, t_h in ((q, q_h), (k, k_h), (v, v_h)):
        t_d.view(torch.int16).copy_(t_h.view(torch.int16), non_blocking=True)
    c1.record(stream)
    o_h.copy_(o.view(torch.int16), non_blocking=True)
    lse_h.copy_(lse, non_blocking=True)
    c2.record(stream)
    torch.cuda.synchronize(dev)
    h2d_ms, d2h_ms = c0.elapsed_time(c1), c1.elapsed_time(c2)
    # both directions at once, on two streams (what the overlapped call needs)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    b0, b1, b2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    torch.cuda.synchronize(dev)
    b0.record(stream)
    s_in.wait_event(b0)
    s_out.wait_event(b0)
    with torch.cuda.stream(s_in):
        for t_d, t_h in ((q, q_h), (k, k_h), (v, v_h)):
            t_d.view(torch.int16).copy_(t_h.view(torch.int16), non_blocking=True)
        b1.record(s_in)
    with torch.cuda.stream(s_out):
        o_h.copy_(o.view(torch.int16), non_blocking=True)
        lse_h.copy_(lse, non_blocking=True)
        b2.record(s_out)
    torch.cuda.synchronize(dev)
    both_ms = max(b0.elapsed_time(b1), b0.elapsed_time(b2))
    link = {"h2d_gbs": in_bytes / h2d_ms / 1e6, "d2h_gbs": d2h / d2h_ms / 1e6,
            "both_directions_ms": both_ms,
            "copy_bound_ms_per_step": max(h2d_ms, d2h_ms, both_ms),
            "e2e_ms_per_step": e2e_ms / e2e_steps,
            "note": "plain pinned copies of one step's bytes: each direction alone, "
                    "then both at once on two streams"}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks, src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    traffic = None
    traffic_file = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(traffic_file):
        with open(traffic_file) as f:
            tj = json.load(f)
        if tj.get("kernel_source_sha256_16") == kernel_source_hash():
            traffic = tj.get(w.name)
    # the oracle baseline is timed at N = 1 only, on the whole workload
    cpu, _ = (time_oracle(w, inp, budget_s=args.cpu_budget)
              if world == 1 and not args.no_cpu_baseline else (None, None))
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "strong" if heads else "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded, bf16-rounded N(0,1))",
        "config": workload_config(w),
        "run": {"l2": (f"no flush: inputs {in_bytes / 2**20:.0f} MiB > L2 126 MiB"
                       if in_bytes > L2_BYTES else
                       f"not flushed: inputs {in_bytes / 2**20:.1f} MiB fit in L2"),
                "parallelism": (f"kv-head shards x{world}" if heads and world > 1 else
                                f"replicas x{world}" if world > 1 else "single GPU")},
        "roofline": {"bound": "tensor", "achieved": kernel_tflops, "peak": peak,
                     "unit": "TFLOP/s", "frac": kernel_tflops / peak, "traffic": traffic,
                     "peak_source": f"{src} bf16_tflops (burst; kernel timed back to back)"},
        "pct_of_peak": 100.0 * kernel_tflops / peak,
        "pct_of_nominal_peak": 100.0 * kernel_tflops / NOMINAL_BF16_TFLOPS,
        "clocks": clocks,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "link": link},
        "gpu_launches": args.steps,
        "cpu_baseline": cpu,
    }
    if gather_ms is not None:
        line["o_allgather_ms"] = gather_ms
    print(json.dumps(line), flush=True)
    return 0


def report_all_workloads(args):
    """Throughput of each path on its workloads (one GPU), one JSON object
    per line; not the contract line.  --only picks one section."""
    import torch
    dev = torch.device("cuda", 0)
    sections = {"forward": report_forward, "varlen": report_varlen, "decode": report_decode,
                "backward": report_backward, "fp8": report_fp8, "mufu": report_mufu}
    for name, fn in sections.items():
        if args.only in (None, name):
            fn(args, dev)


def report_forward(args, dev):
    """The bf16 forward on each of the five workloads."""
    import torch
    from exact_io_aware_92_b200 import attention
    peaks, src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    for w in wl.ALL:
        inp = wl.draw_workload(w)
        q, k, v = (torch.from_numpy(x).view(torch.bfloat16).to(dev)
                   for x in (inp.q_bits, inp.k_bits, inp.v_bits))
        sl = None if inp.seqlens is None else torch.from_numpy(inp.seqlens).to(dev)
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=dev)
        flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
        in_bytes = sum(t.numel() * t.element_size() for t in (q, k, v))
        for _ in range(args.warmup):
            attention.fwd(q, k, v, causal=w.causal, scale=w.scale, seqlens=sl, out=o, lse=lse)
        torch.cuda.synchronize(dev)
        times = []
        for _ in range(args.steps):
            if in_bytes < L2_BYTES:
                flush_l2(flush)  # inputs smaller than L2: evict them between steps
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            record_start(e0)
            attention.fwd(q, k, v, causal=w.causal, scale=w.scale, seqlens=sl, out=o, lse=lse)
            e1.record()
            e1.synchronize()
            times.append(e0.elapsed_time(e1))
        ms = statistics.median(times)
        f = wl.flops(w, inp.seqlens)
        algo_bytes = in_bytes + o.numel() * 2 + lse.numel() * 4
        extra = {}
        if inp.seqlens is not None:
            # query rows inside each sequence only: 4 Hq d sum(len^2)
            useful = 4.0 * w.Hq * w.d * float(np.sum(inp.seqlens.astype(np.float64) ** 2))
            extra = {"tflops_useful": useful / ms / 1e9, "flops_useful": useful}
        print(json.dumps({"workload": w.name, "ms_median": ms, "tflops": f / ms / 1e9,
                          **extra,
                          "frac_of_peak": f / ms / 1e9 / peak,
                          "frac_of_nominal_peak": f / ms / 1e9 / NOMINAL_BF16_TFLOPS,
                          "hbm_gbs": algo_bytes / ms / 1e6,
                          "flops": f, "algorithmic_bytes": algo_bytes,
                          "l2": "flushed between steps" if in_bytes < L2_BYTES else "inputs > L2",
                          "peak_source": src}), flush=True)


def report_fp8(args, dev):
    """The FP8 E4M3 forward (fa_fwd_fp8) on the GQA workload; FLOPs counted
    as for the bf16 forward, against the measured bf16 peak and twice it
    (the nominal FP8:bf16 dense ratio)."""
    import torch
    from exact_io_aware_92_b200 import attention
    peaks, src = load_peaks()
    w = wl.LLAMA_GQA_FP8
    inp = wl.draw_fp8_workload(w)
    q, k = torch.from_numpy(inp.q).to(dev), torch.from_numpy(inp.k).to(dev)
    vt = torch.from_numpy(inp.vt()).to(dev)
    o = torch.empty((w.B, w.Hq, w.N, w.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=dev)
    kw = dict(descale_q=inp.descale_q, descale_k=inp.descale_k, descale_v=inp.descale_v,
              causal=w.causal, scale=w.scale, out=o, lse=lse)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        attention.fwd_fp8(q, k, vt, **kw)
    torch.cuda.synchronize(dev)
    times = []
    for _ in range(args.steps):
        flush_l2(flush)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        record_start(e0)
        attention.fwd_fp8(q, k, vt, **kw)
        e1.record()
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    ms = statistics.median(times)
    f = wl.flops(w)
    tf = f / ms / 1e9
    print(json.dumps({"workload": w.name, "ms_median": ms, "tflops": tf,
                      "frac_of_bf16_peak": tf / float(peaks["bf16_tflops"]),
                      "frac_of_fp8_peak_2x_bf16": tf / (2 * float(peaks["bf16_tflops"])),
                      "flops": f, "l2": "flushed between steps", "peak_source": src}), flush=True)


def report_backward(args, dev):
    """The backward (fa_bwd) on the GPT-2 and Llama GQA workloads.  FLOPs are
    counted as 2.5x the forward's (the five N^2 d products of the gradient);
    this design executes seven, since the dQ kernel recomputes S and dP."""
    import torch
    from exact_io_aware_92_b200 import attention
    peaks, src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    for w in (wl.GPT2, wl.LLAMA_GQA):
        inp = wl.draw_workload(w)
        q, k, v = (torch.from_numpy(x).view(torch.bfloat16).to(dev)
                   for x in (inp.q_bits, inp.k_bits, inp.v_bits))
        g = torch.Generator(device=dev).manual_seed(w.seed + 100)
        do = torch.randn(q.shape, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
        o, lse = attention.fwd(q, k, v, causal=w.causal, scale=w.scale)
        ws = torch.empty(attention.bwd_workspace_size(w.B, w.Hq, w.N), dtype=torch.uint8,
                         device=dev)
        flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
        for _ in range(args.warmup):
            attention.bwd(q, k, v, o, do, lse, causal=w.causal, scale=w.scale, workspace=ws)
        torch.cuda.synchronize(dev)
        times = []
        for _ in range(args.steps):
            flush_l2(flush)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            record_start(e0)
            attention.bwd(q, k, v, o, do, lse, causal=w.causal, scale=w.scale, workspace=ws)
            e1.record()
            e1.synchronize()
            times.append(e0.elapsed_time(e1))
        ms = statistics.median(times)
        f = 2.5 * wl.flops(w, inp.seqlens)
        print(json.dumps({"workload": w.name + "@backward", "ms_median": ms,
                          "tflops": f / ms / 1e9, "frac_of_peak": f / ms / 1e9 / peak,
                          "tflops_executed": 1.4 * f / ms / 1e9, "flops": f,
                          "launches_per_call": 3, "l2": "flushed between steps",
                          "peak_source": src}), flush=True)
        del q, k, v, do, o, lse, ws, flush


def report_varlen(args, dev):
    """The BERT-shaped workload in the packed layout (no padded rows)."""
    import torch
    from exact_io_aware_92_b200 import attention
    peaks, src = load_peaks()
    w = wl.BERT
    inp = wl.draw_workload(w)
    lengths = [int(x) for x in inp.seqlens]
    q, k, v = (torch.from_numpy(wl.pack(x, lengths)).view(torch.bfloat16).to(dev)
               for x in (inp.q_bits, inp.k_bits, inp.v_bits))
    cu = torch.from_numpy(wl.cu_seqlens(lengths)).to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.Hq, q.shape[0]), dtype=torch.float32, device=dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        attention.fwd_varlen(q, k, v, cu, max(lengths), causal=False, scale=w.scale, out=o,
                             lse=lse)
    torch.cuda.synchronize(dev)
    times = []
    for _ in range(args.steps):
        flush_l2(flush)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        record_start(e0)
        attention.fwd_varlen(q, k, v, cu, max(lengths), causal=False, scale=w.scale, out=o,
                             lse=lse)
        e1.record()
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    ms = statistics.median(times)
    useful = 4.0 * w.Hq * w.d * float(sum(L * L for L in lengths))
    print(json.dumps({"workload": w.name + "@packed", "ms_median": ms,
                      "tflops_useful": useful / ms / 1e9,
                      "frac_of_peak": useful / ms / 1e9 / float(peaks["bf16_tflops"]),
                      "flops_useful": useful, "l2": "flushed between steps",
                      "peak_source": src}), flush=True)


def report_mufu(args, dev):
    """The exponential unit's rate, measured (fa_measure_ex2_rate), beside
    the rate at which the tensor pipe consumes score elements: one ex2 per
    element against 4d FLOPs of MMA at 8192 dense bf16 FLOP per clock per SM.
    Below 1, the fraction is the share of the tensor peak the MUFU pipe
    alone allows unless part of the exponentials run on the FMA pipe."""
    from exact_io_aware_92_b200 import attention
    rate = attention.measure_ex2_rate(dev)
    out = {"probe": "mufu_ex2", "ex2_per_clk_per_sm": rate,
           "instruction": "ex2.approx.ftz.f32"}
    for d in (64, 128):
        consumed = 8192.0 / (4 * d)  # score elements per clock per SM at the tensor peak
        out[f"tensor_elems_per_clk_d{d}"] = consumed
        out[f"mufu_cap_frac_of_tensor_peak_d{d}"] = min(1.0, rate / consumed)
    print(json.dumps(out), flush=True)


def report_decode(args, dev):
    """The split-KV decode path: HBM bandwidth against the measured copy rate,
    with 1 and with 4 new query rows per sequence (4 and 32 rows per kv head)."""
    for w in (wl.DECODE, wl.DECODE_NQ4):
        report_decode_one(args, dev, w)


def report_decode_one(args, dev, w):
    import torch
    from exact_io_aware_92_b200 import attention
    peaks, src = load_peaks()
    inp = wl.draw_workload(w)
    q, k, v = (torch.from_numpy(x).view(torch.bfloat16).to(dev)
               for x in (inp.q_bits, inp.k_bits, inp.v_bits))
    sl = torch.from_numpy(inp.seqlens).to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.nq), dtype=torch.float32, device=dev)
    ws = torch.empty(attention.decode_workspace_size(w.B, w.Hq, w.Hkv, w.nq, w.N, w.d),
                     dtype=torch.uint8, device=dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        attention.fwd_decode(q, k, v, causal=w.causal, scale=w.scale, seqlens=sl, workspace=ws,
                             out=o, lse=lse)
    torch.cuda.synchronize(dev)
    times = []
    for _ in range(args.steps):
        flush_l2(flush)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        record_start(e0)
        attention.fwd_decode(q, k, v, causal=w.causal, scale=w.scale, seqlens=sl, workspace=ws,
                             out=o, lse=lse)
        e1.record()
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    ms = statistics.median(times)
    # algorithmic bytes: the valid cache rows of K and V, Q, O and LSE
    kv = 2 * int(np.sum(inp.seqlens)) * w.Hkv * w.d * 2
    qo = 2 * q.numel() * 2 + lse.numel() * 4
    gbs = (kv + qo) / ms / 1e6
    flops = 4.0 * w.Hq * w.nq * w.d * float(np.sum(inp.seqlens))
    print(json.dumps({"workload": w.name, "ms_median": ms, "hbm_gbs": gbs,
                      "frac_of_hbm_peak": gbs / float(peaks["hbm_gbs"]),
                      "algorithmic_bytes": kv + qo, "tflops": flops / ms / 1e9,
                      "launches_per_call": 2, "l2": "flushed between steps",
                      "peak_source": src}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["mine", "reference"], default="mine")
    ap.add_argument("--workload", default=wl.LLAMA_GQA.name, choices=[w.name for w in wl.ALL])
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of CPU work for the oracle baseline sample")
    ap.add_argument("--ref-budget", type=float, default=8.0,
                    help="seconds of CPU work per reference-arm step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--shard", choices=["replicas", "heads"], default="replicas",
                    help="N > 1: one replica of the workload per rank (weak scaling), or "
                         "one problem split by kv-head groups (strong scaling)")
    ap.add_argument("--only", choices=["forward", "varlen", "decode", "backward", "fp8", "mufu"],
                    default=None, help="with --all-workloads: run one section")
    ap.add_argument("--all-workloads", action="store_true",
                    help="report per-workload throughput for the five workloads instead")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch size (profiling a smaller case)")
    args = ap.parse_args()
    if args.all_workloads:
        return report_all_workloads(args)
    w = wl.BY_NAME[args.workload]
    if args.batch is not None:
        import dataclasses
        w = dataclasses.replace(w, B=args.batch, name=f"{w.name}@B{args.batch}")
    if args.impl == "reference":
        return run_reference(args, w)
    return run_mine(args, w)


if __name__ == "__main__":
    sys.exit(main())
