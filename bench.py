#!/usr/bin/env python
"""Benchmark of the fused matmul-sample (FMMS) step; prints one JSON line.

One step = one fused LM-head matmul + temperature + Gumbel noise + argmax call
(fs_sample_ex) over one batch of B rows of a Qwen3-8B-shaped head
(d=4096, V=151936, bf16, T=0.7, per-row seeds) with inputs resident in HBM.
Weights (1.24 GB) exceed the 126 MB L2, so no flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--batch B]
  python bench.py --impl reference ...   # the CPU oracle, timed the same way

Under torchrun each rank runs an independent replica (the path has no
data-path exchange at one GPU per replica); timings are the max over ranks.
"""
import argparse
import contextlib
import hashlib
import json
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "FMMS µs/call & HBM GB/s (% roofline), d=4096 V=151936 bf16, B=1–256"
UNIT = "us/call"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
KERNEL_SOURCES = ["lm_head_exact_fmms_b200/csrc/fmms_kernel.cuh",
                  "lm_head_exact_fmms_b200/csrc/noise.cuh",
                  "lm_head_exact_fmms_b200/csrc/sm100.cuh",
                  "lm_head_exact_fmms_b200/csrc/fmms_common.cuh"]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--batch", type=int, default=64)
    ap.add_argument("--workload", default="qwen3-8b")
    ap.add_argument("--impl", default="fmms", choices=["fmms", "reference"])
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tp", action="store_true",
                    help="split the vocabulary across the ranks instead of running independent "
                         "replicas; the kernels exchange the per-row keys through each other's "
                         "memory (fs_sample_tp)")
    ap.add_argument("--tp-nccl", action="store_true",
                    help="with --tp: exchange the keys with an int64 MAX all-reduce (NCCL) after "
                         "the kernel instead")
    return ap.parse_args()


# ----------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def kernel_source_hash():
    """Hash of the kernel's code: comments and whitespace are left out, so
    that editing a comment does not retire the recorded traffic."""
    import re
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel)) as f:
            src = f.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()[:16]


def committed_traffic(workload_key):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken
    on the current kernel source for this workload; else None."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        t = json.load(f)
    if t.get("kernel_source_sha") != kernel_source_hash():
        return None
    entry = t.get("workloads", {}).get(workload_key)
    if entry is None:
        return None
    # per call, like the achieved figure: one fused launch per 256 rows
    return entry.get("dram_bytes_per_launch") * entry.get("fused_launches_per_call", 1)


class ClockSampler:
    """Samples SM clock and clock-event reasons while the timed region runs
    (NVML, the library nvidia-smi reads; nvidia-smi itself as fallback)."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index, period=0.01):
        self.index, self.period = index, period
        self.samples, self.reasons = [], set()
        self.stamped = []          # (host time, SM MHz, reason bits) of every NVML sample
        self.window = None         # (t0, t1): keep only samples taken inside it
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._nvml = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nvml = None

    def _reasons(self):
        n = self._nvml
        fn = getattr(n, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(n, "nvmlDeviceGetCurrentClocksThrottleReasons")
        return fn(self._h)

    def _sample(self):
        # Stamped at the midpoint of the two queries: on some hosts a query
        # takes milliseconds, as long as a whole short timed region.
        try:
            t = time.perf_counter()
            mhz = self._nvml.nvmlDeviceGetClockInfo(self._h, self._nvml.NVML_CLOCK_SM)
            bits = self._reasons()
            self.stamped.append((0.5 * (t + time.perf_counter()), mhz, bits))
        except Exception:
            pass

    MIN_INTERVAL_S = 0.0005  # at most 2,000 queries a second from the polling loop

    def sample_now(self):
        """One sample from the calling thread (the host polls the GPU with
        it while a timed region drains, so even a region of a few
        milliseconds holds samples), at most one per MIN_INTERVAL_S; in
        between it only sleeps, so a long region does not keep the driver
        busy with queries."""
        if self._nvml is None:
            time.sleep(self.MIN_INTERVAL_S)
            return
        last = self.stamped[-1][0] if self.stamped else -1e30
        if time.perf_counter() - last < self.MIN_INTERVAL_S:
            time.sleep(0.0002)
            return
        self._sample()

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(max(self.period, self.MIN_INTERVAL_S))

    def start(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        else:
            import subprocess
            self._proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index),
                 "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)

    def stop(self):
        if self._nvml is not None:
            self._stop.set()
            self._thread.join()
        elif getattr(self, "_proc", None) is not None:
            self._proc.terminate()
            out, _ = self._proc.communicate()
            for line in out.strip().splitlines():
                try:
                    sm, mx, act = [x.strip() for x in line.split(",")]
                    self.samples.append(int(sm))
                    self.max_mhz = int(mx)
                    bits = int(act, 16)
                    for b, name in self.REASONS.items():
                        if bits & b:
                            self.reasons.add(name)
                except Exception:
                    pass

    def set_window(self, t0, t1):
        """Keep only the samples taken between host times t0 and t1 (the
        timed region: the sampler may start earlier, during the warm-up, so
        that it is already answering when a region of milliseconds begins)."""
        self.window = (t0, t1)

    def _collect(self):
        if self._nvml is None:
            return
        t0, t1 = self.window if self.window is not None else (-1e30, 1e30)
        self.samples = [m for t, m, _ in self.stamped if t0 <= t <= t1]
        self.reasons = set()
        for t, _, bits in self.stamped:
            if t0 <= t <= t1:
                for b, name in self.REASONS.items():
                    if bits & b:
                        self.reasons.add(name)

    def summary(self):
        self._collect()
        s = sorted(self.samples)
        med = s[len(s) // 2] if s else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(s)}


@contextlib.contextmanager
def nvtx(name):
    """An NVTX range around a benchmark section, so that a profiler's
    timeline shows which section a kernel belongs to; nothing happens if
    NVTX is unavailable.  Pushed and popped once per section, outside the
    per-step loop."""
    try:
        import torch
        torch.cuda.nvtx.range_push(name)
        pushed = True
    except Exception:
        pushed = False
    try:
        yield
    finally:
        if pushed:
            try:
                torch.cuda.nvtx.range_pop()
            except Exception:
                pass


def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def algorithmic(B, d, V, masked):
    """Bytes that must cross HBM and flops of one call."""
    nbytes = V * d * 2 + B * d * 2 + B * 4
    if masked:
        nbytes += B * ((V + 31) // 32) * 4
    return nbytes, 2.0 * B * V * d


# A timed region at least this long runs at the board's power limit, so its
# tensor roofline is the sustained bf16 peak; a shorter one (a kernel timed
# in isolation, back to back for milliseconds) takes the burst peak.
SUSTAINED_REGION_S = 1.0


def regime_of(region_s):
    return "sustained" if region_s >= SUSTAINED_REGION_S else "burst"


def roofline(B, d, V, masked, kernel_us, peaks, peak_kind, traffic, regime="burst"):
    """Roofline of one call: the bound is the larger of (algorithmic bytes /
    measured copy bandwidth) and (flops / measured bf16 peak of the regime:
    burst for a short region, sustained for one of seconds at the power
    limit).  `fracs` carries the achieved rate against every peak, so a point
    near the ridge shows both."""
    nbytes, flops = algorithmic(B, d, V, masked)
    tc_key = "bf16_tflops_sustained" if regime == "sustained" else "bf16_tflops"
    t_mem = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (peaks[tc_key] * 1e12)
    gbs = nbytes / (kernel_us * 1e-6) / 1e9
    tfs = flops / (kernel_us * 1e-6) / 1e12
    if t_mem >= t_tc:
        r = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    else:
        r = {"bound": "tensor", "achieved": tfs, "peak": peaks[tc_key], "unit": "TFLOP/s"}
    r["frac"] = r["achieved"] / r["peak"]
    r["traffic"] = traffic
    r["regime"] = regime
    r["peak_source"] = ("%s %s (MEASURED_PEAKS.json)" % (peak_kind, tc_key if r["bound"] == "tensor"
                                                        else "hbm_gbs")
                        if peak_kind == "measured" else "fallback")
    r["fracs"] = {"hbm": round(gbs / peaks["hbm_gbs"], 4),
                  "tensor_burst": round(tfs / peaks["bf16_tflops"], 4),
                  "tensor_sustained": round(tfs / peaks["bf16_tflops_sustained"], 4)}
    r["algorithmic_bytes"] = nbytes
    r["algorithmic_flops"] = flops
    return r


# ------------------------------------------------------------ the GPU arm
def time_calls(fn, steps, warmup, stream, world=1, sampler=None, cooldown_s=1.0, per_call=True):
    """Times exactly `steps` calls after `warmup` untimed ones.  Returns
    (region ms, per-call event durations in us, or None without per_call).
    Events recorded between the calls keep each kernel from overlapping the
    one before it (a programmatic dependent launch overlaps only kernels
    adjacent in the stream), so the region that gives the throughput is
    timed without them (per_call=False) and the per-call percentiles come
    from a pass of their own.  A short idle period first lets the clocks
    recover from the power limit a previous heavy section may have left them
    at."""
    import torch
    torch.cuda.synchronize()
    time.sleep(cooldown_s)
    if sampler:
        sampler.start()  # answering by the time the region starts; samples outside it are dropped
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    n_ev = steps if per_call else 0
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    r0 = torch.cuda.Event(enable_timing=True)
    r1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    t_host0 = time.perf_counter()
    r0.record(stream)
    for i in range(steps):
        if per_call:
            starts[i].record(stream)
        fn(warmup + i)
        if per_call:
            ends[i].record(stream)
    r1.record(stream)
    while not r1.query():     # poll, sampling the clocks while the queued calls run
        if sampler:
            sampler.sample_now()
        else:
            time.sleep(0.0005)
    torch.cuda.synchronize()
    t_host1 = time.perf_counter()
    barrier(world)
    if sampler:
        sampler.stop()
        sampler.set_window(t_host0, t_host1)
    per = [s.elapsed_time(e) * 1e3 for s, e in zip(starts, ends)] if per_call else None
    return r0.elapsed_time(r1), per


def median(xs):
    s = sorted(xs)
    return s[len(s) // 2]


def percentiles(xs, qs=(10, 50, 90)):
    """Nearest-rank percentiles of the per-call kernel times."""
    s = sorted(xs)
    return [s[min(len(s) - 1, max(0, (q * len(s) + 99) // 100 - 1))] for q in qs]


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(H, W, wl, B, rs, budget_s=12.0, max_rows=64):
    """The oracle as it stands, on this host's cores, over a bounded sample of
    the workload's rows; scaled to us per B-row call."""
    import numpy as np
    import oracle
    Hc, Wc = H.cpu(), W.cpu()
    rsc = rs.cpu() if rs is not None else None
    times = []
    t_start = time.time()
    for r in range(min(B, max_rows)):
        t0 = time.perf_counter()
        oracle.sample(Hc, Wc, T=wl.temperature, seed=0, row_seeds=rsc, step=0,
                      rows=np.array([r], dtype=np.int32))
        times.append(time.perf_counter() - t0)
        if time.time() - t_start > budget_s:
            break
    per_row = sum(times) / len(times)
    return {"value": per_row * B * 1e6, "unit": UNIT, "cores": oracle.num_threads(),
            "cpu": cpu_model(), "kind": "oracle",
            "sample": "%d of the %d rows of one B=%d call (full vocabulary each), fp64 oracle; "
                      "value = mean row time x %d rows" % (len(times), B, B, B),
            "seconds": round(sum(times), 2)}


def oracle_per_workload(slice_rows=8192, reps=3):
    """The oracle timed on this host's cores for one row of every workload:
    `reps` rows over a vocabulary slice of at most `slice_rows` tokens (the
    whole head for the tiny one), scaled by V / slice to a full-vocabulary
    row, which is one B=1 call."""
    import numpy as np
    import oracle
    from lm_head_exact_fmms_b200 import synth
    out = []
    for name, wl in synth.WORKLOADS.items():
        Vs = min(wl.V, slice_rows)
        Ws = synth.make_weight(Vs, wl.d, wl.w_std)
        H = synth.make_hidden(reps, wl.d)
        rs = synth.make_row_seeds(reps) if wl.per_row_seeds else None
        mask = synth.make_mask(reps, Vs, wl.mask_allowed) if wl.groups else None
        times = []
        for r in range(reps):
            rows = np.array([r], dtype=np.int32)
            t0 = time.perf_counter()
            if wl.groups:
                oracle.sample_grouped(H, Ws, wl.groups, T=wl.temperature, mask=mask, rows=rows)
            else:
                oracle.sample(H, Ws, T=wl.temperature, row_seeds=rs, rows=rows)
            times.append(time.perf_counter() - t0)
        per_row = sorted(times)[len(times) // 2] * wl.V / Vs
        out.append({"workload": name, "d": wl.d, "V": wl.V,
                    "us_per_row": round(per_row * 1e6, 1),
                    "sample": "median of %d rows x %d-token slice, scaled by V/%d"
                              % (reps, Vs, Vs)})
    return {"cores": oracle.num_threads(), "cpu": cpu_model(), "kind": "oracle",
            "points": out}


def run_gpu(args, world, rank, local):
    import torch

    from lm_head_exact_fmms_b200 import binding, synth

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    binding.load_library()
    wl = synth.WORKLOADS[args.workload]
    B = args.batch
    stream = torch.cuda.current_stream()
    peaks, peak_kind = load_peaks()

    W = synth.make_weight(wl.V, wl.d, wl.w_std, device=dev)
    H = synth.make_hidden(B, wl.d, device=dev)
    rs = synth.make_row_seeds(B, device=dev) if wl.per_row_seeds else None
    mask = synth.make_mask(B, wl.V, wl.mask_allowed).to(dev) if wl.mask_allowed else None
    out = torch.empty(B, dtype=torch.int32, device=dev)
    ws = torch.zeros(binding.fs_workspace_bytes(B, wl.V, wl.groups or 0), dtype=torch.uint8,
                     device=dev)
    grouped = bool(wl.groups)
    tp = args.tp and world > 1 and not grouped
    if tp:
        from lm_head_exact_fmms_b200 import tp as tpmod
        lo, hi = tpmod.shard_bounds(wl.V, world)[rank]
        W_full = W
        W = W_full[lo:hi].contiguous()
        del W_full
        torch.cuda.empty_cache()
        if args.tp_nccl or B > 256:
            keys = torch.empty(B, dtype=torch.int64, device=dev)

            def step(i):
                binding.fs_sample_shard_keys(H, W, lo, wl.V, temperature=wl.temperature, seed=0,
                                             row_seeds=rs, step=i, out_keys=keys, workspace=ws,
                                             stream=stream)
                tpmod.reduce_keys(keys)
                binding.fs_keys_to_tokens(keys, out_idx=out, stream=stream)
        else:
            exchange = tpmod.FusedExchange()

            def step(i):
                exchange.sample(H, W, lo, wl.V, temperature=wl.temperature, seed=0, row_seeds=rs,
                                step=i, out_idx=out, workspace=ws, stream=stream)
    elif grouped:
        def step(i):
            binding.fs_sample_grouped(H, W, wl.groups, temperature=wl.temperature, seed=0,
                                      row_seeds=rs, step=i, mask_bits=mask, out_idx=out,
                                      workspace=ws, stream=stream)
    else:
        def step(i):
            binding.fs_sample_ex(H, W, temperature=wl.temperature, seed=0, row_seeds=rs, step=i,
                                 mask_bits=mask, out_idx=out, workspace=ws, stream=stream)

    # Every 0.5 ms while the region lasts milliseconds; every 5 ms for long runs (the host's
    # polling loop adds samples at up to the same 0.5 ms rate).
    sampler = ClockSampler(local, period=0.0 if args.steps <= 200 else 0.005)
    with nvtx("fmms: timed steps"):
        region_ms, _ = time_calls(step, args.steps, args.warmup, stream, world, sampler,
                                  per_call=False)
    region_ms = max_over_ranks(region_ms, world)
    us_per_call = region_ms * 1e3 / args.steps
    nbytes, flops = algorithmic(B, wl.d, wl.V, mask is not None)
    # fused kernel per 256 rows, plus the group merge (grouped) or the decode (tp)
    fused_tp = tp and not (args.tp_nccl or B > 256)
    # tensor-parallel: + the token decode after the all-reduce, or the bounded
    # wait that copies the exchanged tokens
    launches_per_call = (B + 255) // 256 * (2 if grouped else 1) + (1 if tp else 0)
    # The fused kernel's average time per launch over the timed region (the
    # stream holds nothing else in flat mode; with a merge or exchange kernel
    # per call this is the call's time divided by its fused launches).
    fused_launches = (B + 255) // 256
    kernel_us = us_per_call / fused_launches
    if tp:
        # each rank streams its shard; the roofline below is per rank
        nbytes = nbytes * W.shape[0] // wl.V

    # e2e: host buffers through the public C entry point (H2D + kernel + D2H).
    Hh = H.cpu().pin_memory()
    Oh = torch.empty(B, dtype=torch.int32).pin_memory()

    def step_host(i):
        binding.fs_sample_host(Hh, W, temperature=wl.temperature, seed=0, row_seeds=rs, step=i,
                               out_idx_host=Oh, stream=stream)

    if tp or grouped:
        # the host-buffer entry point is flat and single-GPU: time H2D + the step + D2H here
        def step_host(i):
            H.copy_(Hh, non_blocking=True)
            step(i)
            Oh.copy_(out, non_blocking=True)
    with nvtx("fmms: end-to-end steps (host buffers)"):
        e2e_ms, _ = time_calls(step_host, args.steps, args.warmup, stream, world, per_call=False)
    e2e_ms = max_over_ranks(e2e_ms, world)

    result = {
        "metric": METRIC, "value": round(us_per_call, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(region_ms / args.steps, 6),
        "higher_is_better": False, "scaling": "strong" if tp else "weak", "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic: seeded H ~ N(0,1), W ~ N(0, %g^2) bf16 (random-init %s head)"
                % (wl.w_std, wl.name),
        "config": workload_config(wl, B, world, tp, fused_tp),
        "samples_per_s": round(B * world / (us_per_call * 1e-6), 1),
        "hbm_gbs_per_gpu": round(nbytes / (us_per_call * 1e-6) / 1e9, 1),
        "kernel_us": round(kernel_us, 3),
        "roofline": roofline(B, wl.d, W.shape[0], mask is not None, kernel_us, peaks, peak_kind,
                             None if tp else committed_traffic("%s/B%d" % (wl.name, B)),
                             regime_of(region_ms * 1e-3)),
        "e2e": {"value": round(e2e_ms * 1e3 / args.steps, 3), "unit": UNIT,
                "h2d_bytes_per_step": B * wl.d * 2, "d2h_bytes_per_step": B * 4,
                "entry_point": "fs_sample_host (pinned host H in, host tokens out)"},
        "gpu_launches": args.steps * launches_per_call,
        "clocks": sampler.summary(),
    }

    # The single-GPU characterisation (batch sweep, other modes) runs at N=1
    # only: at N > 1 it would hold the other GPUs idle while rank 0 works.
    if rank == 0 and world == 1 and not args.no_sweep:
        with nvtx("fmms: batch sweep"):
            result["sweep"] = sweep(torch, binding, synth, W, wl, dev, stream, peaks, peak_kind,
                                    compare_single=True)
        with nvtx("fmms: library GEMM for context"):
            result["library_gemm"] = library_gemm_points(torch, synth, W, wl, dev)
        with nvtx("fmms: sustained decode"):
            result["sustained"] = sustained_point(torch, binding, synth, W, wl, dev, stream, peaks,
                                                  peak_kind, local)
        with nvtx("fmms: sustained large batch"):
            # the tensor-bound batch over a long region, against the sustained bf16 peak
            result["sustained_b256"] = sustained_point(torch, binding, synth, W, wl, dev, stream,
                                                       peaks, peak_kind, local, B=256,
                                                       est_us=300.0)
        # The other LM-head shapes, each at its own batch sizes.
        result["sweeps"] = {}
        for other in ("qwen3-1.7b", "large"):
            owl = synth.WORKLOADS[other]
            with nvtx("fmms: batch sweep, %s head" % other):
                Wo = synth.make_weight(owl.V, owl.d, owl.w_std, device=dev)
                result["sweeps"][other] = {
                    "workload": "%s LM head d=%d V=%d T=%g, fused fs_sample_ex"
                                % (other, owl.d, owl.V, owl.temperature),
                    "points": sweep(torch, binding, synth, Wo, owl, dev, stream, peaks, peak_kind)}
                del Wo
                torch.cuda.empty_cache()
        with nvtx("fmms: grouped + masked"):
            result["grouped_masked"] = grouped_points(torch, binding, synth, dev, stream, peaks,
                                                      peak_kind, W)
        with nvtx("fmms: online grouped"):
            result["online_grouped"] = online_grouped_point(torch, binding, synth, dev, stream, W)
        with nvtx("fmms: unfused"):
            result["unfused"] = unfused_point(torch, binding, synth, W, wl, dev, stream, B)
        with nvtx("fmms: several samples per row"):
            result["multi_sample"] = multi_point(torch, binding, synth, W, wl, dev, stream, B)
        with nvtx("fmms: CUDA graph"):
            result["cuda_graph"] = graph_point(torch, binding, synth, W, wl, dev, B)
        with nvtx("fmms: top-k"):
            result["top_k"] = topk_point(torch, binding, synth, W, wl, dev, stream, B)
        with nvtx("fmms: tiny head"):
            result["tiny"] = tiny_point(torch, binding, synth, dev, stream)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not grouped:
        result["cpu_baseline"] = cpu_baseline(H, W, wl, B, rs)
        if not args.no_sweep:
            result["cpu_baseline"]["per_workload"] = oracle_per_workload()
    if fused_tp:
        exchange.close()  # every rank, after its last call
    return result


def sweep(torch, binding, synth, W, wl, dev, stream, peaks, peak_kind, steps=200, warmup=10,
          compare_single=False):
    """Each of the workload's batch sizes, `steps` back-to-back calls after a
    one-second idle: a short region, so the burst tensor peak applies."""
    rows = []
    for B in wl.batches:
        H = synth.make_hidden(B, wl.d, device=dev)
        rs = synth.make_row_seeds(B, device=dev) if wl.per_row_seeds else None
        out = torch.empty(B, dtype=torch.int32, device=dev)

        def step(i):
            binding.fs_sample_ex(H, W, temperature=wl.temperature, seed=0, row_seeds=rs, step=i,
                                 out_idx=out, stream=stream)

        region_ms, _ = time_calls(step, steps, warmup, stream, per_call=False)
        _, per = time_calls(step, steps, warmup, stream, cooldown_s=0.2)
        kus = region_ms * 1e3 / steps / binding.fs_fused_launches(B)
        rf = roofline(B, wl.d, wl.V, False, kus, peaks, peak_kind,
                      committed_traffic("%s/B%d" % (wl.name, B)), regime_of(region_ms * 1e-3))
        row = {"B": B, "us_per_call": round(region_ms * 1e3 / steps, 3),
               "kernel_us": round(kus, 3),
               # per call with an event on each side (no overlap with the call before)
               "event_us_p10_p50_p90": [round(x, 3) for x in percentiles(per)],
               "bound": rf["bound"],
               "achieved": round(rf["achieved"], 1), "unit": rf["unit"],
               "frac": round(rf["frac"], 4), "fracs": rf["fracs"], "regime": rf["regime"],
               "traffic": rf["traffic"],
               # the library's automatic choice (fs_plan_batch): CTA pairs from a 112-row tile
               "cta_pairs": binding.fs_uses_cta_pairs(B)}
        if compare_single and row["cta_pairs"]:
            # the same call on the single-CTA kernel, for comparison
            binding.fs_set_cta_pairs(0)
            try:
                r1, _ = time_calls(step, steps, warmup, stream, per_call=False)
            finally:
                binding.fs_set_cta_pairs(-1)
            row["single_cta_kernel_us"] = round(r1 * 1e3 / steps, 3)
        rows.append(row)
    return rows


def library_gemm_points(torch, synth, W, wl, dev, batches=(64, 128, 256), steps=100):
    """For context only: the logits GEMM alone, H W^T in bf16 through torch
    (cuBLAS), which writes B x V bf16 logits and samples nothing."""
    rows = []
    for B in batches:
        H = synth.make_hidden(B, wl.d, device=dev)
        out = torch.empty(B, wl.V, dtype=torch.bfloat16, device=dev)
        region_ms, _ = time_calls(lambda i: torch.matmul(H, W.t(), out=out), steps, 10,
                                  torch.cuda.current_stream(), per_call=False)
        rows.append({"B": B, "us_per_call": round(region_ms * 1e3 / steps, 3)})
    return {"what": "torch.matmul(H, W.T) bf16 -> bf16 logits [B, V] (cuBLAS), no sampling",
            "points": rows}


def sustained_point(torch, binding, synth, W, wl, dev, stream, peaks, peak_kind, local, B=64,
                    seconds=2.5, est_us=200.0):
    """A long run: calls of B rows back to back for about `seconds` (est_us:
    the expected time per call; the board sits at its power limit and the SM
    clock gives way), with the clocks sampled throughout.  Reports the kernel
    time, the median SM clock, the kernel time in clock cycles (time x median
    MHz) and the roofline of the sustained regime: the copy bandwidth, or
    the sustained bf16 peak where the matmul bounds the call."""
    H = synth.make_hidden(B, wl.d, device=dev)
    rs = synth.make_row_seeds(B, device=dev) if wl.per_row_seeds else None
    out = torch.empty(B, dtype=torch.int32, device=dev)

    def step(i):
        binding.fs_sample_ex(H, W, temperature=wl.temperature, seed=0, row_seeds=rs, step=i,
                             out_idx=out, stream=stream)

    calls = max(100, int(seconds / (est_us * 1e-6)))
    sampler = ClockSampler(local, period=0.01)
    region_ms, _ = time_calls(step, calls, 20, stream, sampler=sampler, per_call=False)
    kus = region_ms * 1e3 / calls
    clk = sampler.summary()
    rf = roofline(B, wl.d, wl.V, False, kus, peaks, peak_kind, None, regime_of(region_ms * 1e-3))
    return {"B": B, "calls": calls, "region_s": round(region_ms * 1e-3, 3),
            "us_per_call": round(region_ms * 1e3 / calls, 3), "kernel_us": round(kus, 3),
            "sm_mhz_median": clk["sm_mhz"], "clock_samples": clk["samples"],
            "reasons": clk["reasons"],
            "kcycles_per_call": round(kus * clk["sm_mhz"] / 1e3, 1) if clk["sm_mhz"] else None,
            "bound": rf["bound"], "achieved": round(rf["achieved"], 1), "unit": rf["unit"],
            "frac": round(rf["frac"], 4), "fracs": rf["fracs"], "regime": rf["regime"]}


def grouped_points(torch, binding, synth, dev, stream, peaks, peak_kind, W8, steps=100):
    """The grouped + masked workload at each of its batch sizes."""
    wl = synth.WORKLOADS["grouped-masked"]
    W = W8 if (W8.shape[0] == wl.V and W8.shape[1] == wl.d) else \
        synth.make_weight(wl.V, wl.d, wl.w_std, device=dev)
    rows = []
    for B in wl.batches:
        H = synth.make_hidden(B, wl.d, device=dev)
        mask = synth.make_mask(B, wl.V, wl.mask_allowed).to(dev)
        out = torch.empty(B, dtype=torch.int32, device=dev)

        def step(i):
            binding.fs_sample_grouped(H, W, wl.groups, temperature=wl.temperature, seed=0, step=i,
                                      mask_bits=mask, out_idx=out, stream=stream)

        region_ms, _ = time_calls(step, steps, 10, stream, per_call=False)
        us = region_ms * 1e3 / steps
        rf = roofline(B, wl.d, wl.V, True, us, peaks, peak_kind,
                      committed_traffic("%s/B%d" % (wl.name, B)), regime_of(region_ms * 1e-3))
        rows.append({"B": B, "us_per_call": round(us, 3), "bound": rf["bound"],
                     "achieved": round(rf["achieved"], 1), "unit": rf["unit"],
                     "frac": round(rf["frac"], 4), "fracs": rf["fracs"], "regime": rf["regime"],
                     "traffic": rf["traffic"],
                     "launches_per_call": 2 * binding.fs_fused_launches(B, "grouped")})
    return {"workload": "grouped-masked d=%d V=%d G=%d, 50%% mask, T=%g (fused kernel + merge)"
                        % (wl.d, wl.V, wl.groups, wl.temperature), "points": rows}


def online_grouped_point(torch, binding, synth, dev, stream, W8, B=64, steps=100):
    """Online grouped sampling on the grouped + masked head: each of the G
    groups summarised by its own call on its slice of W (as when only one
    group's weights are on chip at a time), then the summaries merged."""
    wl = synth.WORKLOADS["grouped-masked"]
    W = W8 if (W8.shape[0] == wl.V and W8.shape[1] == wl.d) else \
        synth.make_weight(wl.V, wl.d, wl.w_std, device=dev)
    G = wl.groups
    bounds = [(g * wl.V) // G for g in range(G + 1)]
    if any(b % 8 for b in bounds):
        return {"B": B, "us_per_call": None, "error": "group boundaries not multiples of 8"}
    H = synth.make_hidden(B, wl.d, device=dev)
    mask = synth.make_mask(B, wl.V, wl.mask_allowed).to(dev)
    summ = torch.empty(G, B, 3, dtype=torch.float32, device=dev)
    out = torch.empty(B, dtype=torch.int32, device=dev)
    slices = [W[bounds[g]:bounds[g + 1]] for g in range(G)]  # contiguous row ranges
    ws = torch.zeros(binding.fs_workspace_bytes_summary(B, max(b1 - b0 for b0, b1 in
                                                              zip(bounds, bounds[1:]))),
                     dtype=torch.uint8, device=dev)

    def step(i):
        for g in range(G):
            binding.fs_summarize_group(H, slices[g], bounds[g], wl.V, temperature=wl.temperature,
                                       seed=0, step=i, mask_bits=mask, out_summary=summ[g],
                                       workspace=ws, stream=stream)
        binding.fs_merge_groups(summ, seed=0, step=i, out_idx=out, stream=stream)

    region_ms, _ = time_calls(step, steps, 10, stream, per_call=False)
    return {"B": B, "groups": G, "us_per_call": round(region_ms * 1e3 / steps, 3),
            "launches_per_call": 2 * G + 1,
            "note": "one fs_summarize_group per group (fused kernel + summary merge) and one "
                    "fs_merge_groups"}


def multi_point(torch, binding, synth, W, wl, dev, stream, B, S=4, steps=100):
    """num_samples > 1: S exact draws per row from one pass over W."""
    H = synth.make_hidden(B, wl.d, device=dev)
    rs = synth.make_row_seeds(B, device=dev) if wl.per_row_seeds else None
    out = torch.empty(B, S, dtype=torch.int32, device=dev)
    ws = torch.zeros(binding.fs_workspace_bytes_multi(B, wl.V, S), dtype=torch.uint8, device=dev)

    def step(i):
        binding.fs_sample_multi(H, W, S, temperature=wl.temperature, seed=0, row_seeds=rs, step=i,
                                out_idx=out, workspace=ws, stream=stream)

    region_ms, _ = time_calls(step, steps, 10, stream, per_call=False)
    return {"B": B, "num_samples": S, "us_per_call": round(region_ms * 1e3 / steps, 3),
            "samples_per_s": round(B * S / (region_ms * 1e-3 / steps), 1)}


def graph_point(torch, binding, synth, W, wl, dev, B, calls=10, replays=30):
    """The same step captured ten calls at a time in a CUDA graph, to separate
    the kernel from per-call launch overhead."""
    try:
        H = synth.make_hidden(B, wl.d, device=dev)
        rs = synth.make_row_seeds(B, device=dev) if wl.per_row_seeds else None
        out = torch.empty(B, dtype=torch.int32, device=dev)
        ws = torch.zeros(binding.fs_workspace_bytes(B, wl.V, 0), dtype=torch.uint8, device=dev)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for i in range(3):
                binding.fs_sample_ex(H, W, temperature=wl.temperature, row_seeds=rs, step=i,
                                     out_idx=out, workspace=ws, stream=s)
        s.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for i in range(calls):
                binding.fs_sample_ex(H, W, temperature=wl.temperature, row_seeds=rs, step=i,
                                     out_idx=out, workspace=ws, stream=s)
        torch.cuda.synchronize()
        time.sleep(1.0)
        for _ in range(2):
            g.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(replays):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / (replays * calls)
        del g
        return {"B": B, "us_per_call": round(us, 3), "calls_per_graph": calls}
    except Exception as exc:   # report, do not break the bench line
        return {"B": B, "us_per_call": None, "error": str(exc)[:200]}


def tiny_point(torch, binding, synth, dev, stream, copies=64, steps=640, graph_calls=64,
               replays=10):
    """The tiny head (d=256, V=4096, 2 MiB of W): launch latency, not
    bandwidth.  Each call reads the next of `copies` distinct W tensors
    (128 MiB in all, above the 126 MB L2), so no call finds its W in L2.
    Reported per call through the stream and inside a CUDA graph."""
    wl = synth.WORKLOADS["tiny"]
    B = wl.batches[0]
    try:
        Ws = [synth.make_weight(wl.V, wl.d, wl.w_std, seed=1234 + c, device=dev)
              for c in range(copies)]
        H = synth.make_hidden(B, wl.d, device=dev)
        out = torch.empty(B, dtype=torch.int32, device=dev)
        ws = torch.zeros(binding.fs_workspace_bytes(B, wl.V, 0), dtype=torch.uint8, device=dev)

        def step(i):
            binding.fs_sample_ex(H, Ws[i % copies], temperature=wl.temperature, seed=0, step=i,
                                 out_idx=out, workspace=ws, stream=stream)

        region_ms, _ = time_calls(step, steps, 3 * copies, stream, per_call=False)
        _, per = time_calls(step, steps, 3 * copies, stream, cooldown_s=0.2)
        res = {"workload": "tiny head d=%d V=%d B=%d, %d rotating W copies (%d MiB)"
                           % (wl.d, wl.V, B, copies, copies * wl.V * wl.d * 2 >> 20),
               "us_per_call": round(region_ms * 1e3 / steps, 3),
               "event_us_p10_p50_p90": [round(x, 3) for x in percentiles(per)]}
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for i in range(graph_calls):
                binding.fs_sample_ex(H, Ws[i % copies], temperature=wl.temperature, seed=0,
                                     step=i, out_idx=out, workspace=ws, stream=s)
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(replays):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        res["graph_us_per_call"] = round(e0.elapsed_time(e1) * 1e3 / (replays * graph_calls), 3)
        del g
        return res
    except Exception as exc:   # report, do not break the bench line
        return {"us_per_call": None, "error": str(exc)[:200]}


def topk_point(torch, binding, synth, W, wl, dev, stream, B, K=50, steps=100):
    """Top-k sampling: the fused kernel writes fp32 logits to HBM, then a
    per-block candidate launch and a per-row select launch sample each row."""
    H = synth.make_hidden(B, wl.d, device=dev)
    rs = synth.make_row_seeds(B, device=dev) if wl.per_row_seeds else None
    out = torch.empty(B, dtype=torch.int32, device=dev)
    logits = torch.empty(B, wl.V, dtype=torch.float32, device=dev)

    def step(i):
        binding.fs_sample_topk(H, W, K, temperature=wl.temperature, seed=0, row_seeds=rs, step=i,
                               out_idx=out, logits=logits, stream=stream)

    region_ms, _ = time_calls(step, steps, 10, stream, per_call=False)
    return {"B": B, "K": K, "us_per_call": round(region_ms * 1e3 / steps, 3),
            "launches_per_call": 3 * ((B + 255) // 256)}


def unfused_point(torch, binding, synth, W, wl, dev, stream, B, steps=100):
    H = synth.make_hidden(B, wl.d, device=dev)
    rs = synth.make_row_seeds(B, device=dev) if wl.per_row_seeds else None
    out = torch.empty(B, dtype=torch.int32, device=dev)
    logits = torch.empty(B, wl.V, dtype=torch.float32, device=dev)

    def step(i):
        binding.fs_sample_unfused(H, W, temperature=wl.temperature, seed=0, row_seeds=rs, step=i,
                                  out_idx=out, logits=logits, stream=stream)

    region_ms, _ = time_calls(step, steps, 10, stream, per_call=False)
    return {"us_per_call": round(region_ms * 1e3 / steps, 3),
            "extra_hbm_bytes_per_call": 2 * B * wl.V * 4,
            "note": "matmul writes fp32 logits [B,V], a second kernel reads them back"}


# ------------------------------------------------------ the reference arm
def workload_config(wl, B, world, tp=False, fused_tp=False):
    """The `config` object of the JSON line (both arms print the same one)."""
    grouped = bool(wl.groups)
    return {"workload": "%s LM head, d=%d V=%d B=%d T=%g%s%s, fused %s"
                        % (wl.name, wl.d, wl.V, B, wl.temperature,
                           ", per-row seeds" if wl.per_row_seeds else "",
                           (", G=%d, %d%% mask" % (wl.groups, round(100 * wl.mask_allowed)))
                           if grouped else "",
                           "fs_sample_grouped" if grouped else "fs_sample_ex"),
            "batch_per_gpu": B, "global_batch": B * world, "d": wl.d, "V": wl.V,
            "parallelism": ("tensor-parallel vocabulary x%d (%s)" % (
                world, "fused peer-memory exchange" if fused_tp else "NCCL all-reduce"))
            if tp else ("replicas x%d" % world),
            "l2": "no flush: W (%.2f GB) exceeds the 126 MB L2" % (wl.V * wl.d * 2 / 1e9)}


def run_reference(args, world, rank):
    """The CPU oracle timed on this host's cores, on the same workload, metric
    and unit; each step is a bounded sample (one row over a vocabulary slice)."""
    if rank != 0:
        return None
    import numpy as np
    import torch

    import oracle
    from lm_head_exact_fmms_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    B = args.batch
    H = synth.make_hidden(B, wl.d)
    # a vocabulary slice of the head; the full head would take minutes per step
    total = args.steps + args.warmup
    budget = 120.0 / max(total, 1)
    probe_V = 4096
    Wp = synth.make_weight(probe_V, wl.d, wl.w_std)
    rs = synth.make_row_seeds(B) if wl.per_row_seeds else None
    t0 = time.perf_counter()
    oracle.sample(H, Wp, T=wl.temperature, row_seeds=rs, rows=np.array([0], dtype=np.int32))
    t_probe = max(time.perf_counter() - t0, 1e-6)
    Vs = int(max(64, min(wl.V, probe_V * budget / t_probe)))
    Ws = synth.make_weight(Vs, wl.d, wl.w_std)
    times = []
    for i in range(total):
        r = np.array([i % B], dtype=np.int32)
        t0 = time.perf_counter()
        oracle.sample(H, Ws, T=wl.temperature, row_seeds=rs, step=i, rows=r)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    scale = (wl.V / Vs) * B
    value = sum(times) / len(times) * scale * 1e6
    cores = oracle.num_threads()
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(sum(times) / len(times) * 1e3, 3), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, B, world, args.tp and world > 1 and not wl.groups,
                                  args.tp and world > 1 and not wl.groups
                                  and not (args.tp_nccl or B > 256)),
        "cpu_baseline": {"value": round(value, 1), "unit": UNIT, "cores": cores, "cpu": cpu_model(),
                         "kind": "oracle",
                         "sample": "each step: 1 row x %d-token vocabulary slice; value scaled "
                                   "by (V/%d) x B" % (Vs, Vs)},
        "e2e": {"value": round(value, 1), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        res = run_reference(args, world, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    world, rank, local = dist_setup()
    res = run_gpu(args, world, rank, local)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
