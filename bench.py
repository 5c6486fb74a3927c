#!/usr/bin/env python
"""Benchmark of the MoE dispatch/combine hot path (layout -> dispatch -> combine)
on the DeepSeek-V3-shaped low-latency decode workload: 8 logical ranks x 128
tokens (B = 1024), d = 7168, E = 256, top-8, int8 dynamic quantization.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode] [--flush-mb 512] [--no-cpu-baseline]

One step = one pass of the whole path over one batch: ep_layout, ep_dispatch,
ep_combine through the C ABI, captured once as a CUDA graph and replayed.  The
expert output buffer that combine reads is resident (the identity expert: the
dequantized receive rows), since the expert computation is not part of
dispatch/combine.  Up to three buffer sets are used in rotation, so consecutive
steps touch disjoint memory (more than the 126 MB L2 per step); when only one
set fits, L2 is flushed (a 512 MB memset) between steps, outside the events.
Per-kernel durations: isolated (one launch after an L2 read-flush, CUDA events
around it; the roofline figure) and overlapped (graphs of back-to-back launches).

Prints one JSON line (rank 0).  value = algorithmic HBM bytes of the three
kernels / step time, whole job (all ranks), in GB/s.
--impl reference times the CPU oracle (the reference arm for this path) on the
host cores, one bounded sample of the workload per step.
With N > 1 (torchrun), every rank runs an independent replica (the EP ranks are
logical partitions of one GPU; nothing is exchanged between GPUs).
"""
import argparse
import hashlib
import json
import re
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "dispatch+combine HBM GB/s and tokens/s at d=7168,E=256,k=8; % of B200 HBM peak"
SPEC_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
PROFILES = os.path.join(ROOT, "profiles")
_CSRC = "combine_ep_layout_12_b200/csrc/"
KERNEL_SOURCES = {  # every source file a kernel's code comes from
    "layout": [_CSRC + f for f in ("ep_layout.cu", "ep_layout_dev.cuh", "ep_internal.cuh")],
    "dispatch": [_CSRC + f for f in ("ep_dispatch.cu", "ep_dispatch_dev.cuh", "ep_internal.cuh")],
    "combine": [_CSRC + f for f in ("ep_combine.cu", "ep_internal.cuh")],
    "layout_dispatch": [_CSRC + f for f in ("ep_fused.cu", "ep_layout_dev.cuh", "ep_dispatch_dev.cuh",
                                            "ep_internal.cuh")],
}


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    p.add_argument("--workload", default="decode")
    p.add_argument("--flush-mb", type=int, default=512, help="L2 flush between steps when only one buffer set fits")
    p.add_argument("--sets", type=int, default=3, help="buffer sets used in rotation")
    p.add_argument("--e2e-steps", type=int, default=None, help="steps of the end-to-end loop (default min(K, 200))")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=10.0, help="target CPU time of the oracle baseline")
    p.add_argument("--sweep", default=None,
                   help="comma-separated workloads or 'all': per-workload table instead of the JSON line")
    p.add_argument("--sweep-out", default=None, help="where --sweep writes its JSON document")
    p.add_argument("--shard", action="store_true",
                   help="time the multi-GPU form on this GPU (P slabs, two micro-batches, dual-batch overlap)")
    p.add_argument("--profile-launches", type=int, default=0, metavar="N",
                   help="for profiler captures: build --workload with one buffer set and run N times each "
                        "of ep_layout, ep_dispatch, ep_layout_dispatch and ep_combine, each after an L2 "
                        "read-flush; prints no JSON line")
    return p.parse_args(argv)


# ----------------------------------------------------------------------------- distributed plumbing


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    import torch.distributed as dist
    from datetime import timedelta
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=timedelta(seconds=120))
    return dist if world > 1 else None


def aggregate(dist, seconds, units, device=None):
    """Whole-job numbers over ranks: time = max over ranks, units = sum over ranks."""
    if dist is None:
        return seconds, units
    import torch
    t = torch.tensor([seconds], dtype=torch.float64, device=device)
    u = torch.tensor([units], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


def barrier(dist, device=None):
    if dist is not None:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ----------------------------------------------------------------------------- clocks


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {
        "hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
        "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
        "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
        "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
        "hw_power_brake": "nvmlClocksEventReasonHwPowerBrakeSlowdown",
    }

    def __init__(self, index, period=0.01):
        self.samples = []
        self.period = period
        self.ok = False
        self.window = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as exc:  # no NVML: report that instead of numbers
            self.error = repr(exc)
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.th = threading.Thread(target=self._run, daemon=True)
            self.th.start()

    def mark(self, t0, t1):
        self.window = (t0, t1)

    def stop(self):
        if self.ok:
            self._stop.set()
            self.th.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "error", "")}
        t0, t1 = self.window if self.window else (-1e30, 1e30)
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        used = inside
        note = None
        if len(inside) < 3:  # short timed region: widen to the neighbouring samples
            used = sorted(self.samples, key=lambda s: abs(s[0] - 0.5 * (t0 + t1)))[:5]
            note = "timed region shorter than the sampling period; nearest samples used"
        mhz = [s[1] for s in used]
        reasons = set()
        for s in used:
            for name, attr in self.REASONS.items():
                bit = getattr(self.nv, attr, 0)
                if bit and (s[2] & bit):
                    reasons.add(name)
        out = {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
               "reasons": sorted(reasons), "samples": len(used)}
        if note:
            out["note"] = note
        return out


# ----------------------------------------------------------------------------- helpers


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def trimmed_mean(xs, trim=0.1):
    """Mean of xs without the lowest and highest `trim` fraction."""
    xs = sorted(xs)
    n = int(len(xs) * trim)
    xs = xs[n:len(xs) - n] if len(xs) > 2 * n else xs
    return sum(xs) / len(xs)


def code_text(src):
    """C/C++/CUDA source without comments and with whitespace runs collapsed, so a
    change to comments alone does not count as a change of the kernel."""
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def source_hash(name, read=None):
    """Hash of the code of every source file a kernel is built from; read(rel) gives
    a file's text (default: the working tree)."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[name]:
        if read is None:
            with open(os.path.join(ROOT, rel)) as f:
                text = f.read()
        else:
            text = read(rel)
        h.update(code_text(text).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload, kernel, with_shape=False):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source (else None); with_shape: also the workload the
    capture ran on (a smaller variant with the same per-launch traffic, or the
    workload itself)."""
    path = os.path.join(PROFILES, "traffic.json")
    try:
        with open(path) as f:
            j = json.load(f)
        rec = j[workload][kernel]
        if rec.get("source_sha") != source_hash(kernel):
            return (None, None) if with_shape else None
        b = float(rec["dram_bytes_per_launch"])
        return (b, rec.get("captured_on", workload)) if with_shape else b
    except Exception:
        return (None, None) if with_shape else None


def oracle_sample_prepare(w, inp, t0, n_tokens):
    """Inputs of one oracle sample: tokens [t0, t0 + n_tokens) (one logical rank's
    batch when n_tokens = T) taken as a one-rank problem, plus stand-in expert
    outputs (the identity expert: dequantized receive rows, made here once and not
    timed, since the expert computation is not part of dispatch/combine)."""
    import oracle
    from combine_ep_layout_12_b200 import metrics
    B = n_tokens
    cfg = oracle.make_cfg(B, w.d, w.k, 1, B, w.E, w.n_zero, w.n_copy, w.n_const, w.quant_mode)
    sl = slice(t0, t0 + B)
    st = {"cfg": cfg, "idx": np.ascontiguousarray(inp["topk_idx"][sl]),
          "x": np.ascontiguousarray(inp["x"][sl]), "wts": np.ascontiguousarray(inp["topk_weights"][sl]),
          "act": None if inp.get("active") is None else np.ascontiguousarray(inp["active"][sl]),
          "smooth": inp["smooth"], "a1": inp["a1"], "a2": inp["a2"], "v": inp["v"],
          "expert_smooth": w.smooth == "expert", "quant_mode": w.quant_mode, "d": w.d}
    rx, rsc, compact, n_r = _oracle_dispatch(st)
    if w.quant_mode != 0:
        eo = np.zeros((max(n_r, 1), w.d), np.uint16)
        if n_r:
            f = rx[:n_r].astype(np.float32)
            if w.quant_mode == 2:
                f = f * rsc[:n_r, None]
            eo[:n_r] = (f.view(np.uint32) >> 16).astype(np.uint16)
    else:
        eo = rx
    st["eo"] = eo
    nr, bsp = metrics.routing_counts(w.with_(B=B), st["idx"], n_r, active=st["act"])
    st["bytes"] = sum(metrics.kernel_bytes(w.with_(B=B, P=1, M=B), nr, bsp, smooth=inp["smooth"] is not None,
                                           masked=st["act"] is not None).values())
    return st


def _oracle_dispatch(st):
    """Layout, quantization and the scatter into a compact receive buffer (one row
    per routed pick, the same bytes as the real layout)."""
    import oracle
    cfg = st["cfg"]
    lay = oracle.layout(cfg, st["idx"], active=st["act"])
    dp = lay["dst_pos"]
    compact = np.full(dp.shape, -1, np.int32)
    routed = dp >= 0
    n_r = int(routed.sum())
    compact[routed] = np.arange(n_r, dtype=np.int32)
    if st["expert_smooth"]:
        rx, rsc = oracle.dispatch_expert_smooth(cfg, st["x"], st["smooth"], st["idx"], compact, max(n_r, 1))
    else:
        q, ts = oracle.quantize(cfg, st["x"], st["smooth"])
        rx, rsc = oracle.dispatch(cfg, q, ts, compact, max(n_r, 1))
    return rx, rsc, compact, n_r


def oracle_sample_run(st):
    """One timed oracle pass over a prepared sample: layout, quantize, scatter, combine."""
    import oracle
    _, _, compact, _ = _oracle_dispatch(st)
    oracle.combine(st["cfg"], st["eo"], st["idx"], st["wts"], compact, st["x"], st["a1"], st["a2"],
                   st["v"], active=st["act"])


def _oracle_worker_main(conn):
    """One oracle process: receives its sample once, then runs `reps` passes per
    request and answers with the seconds they took."""
    st = conn.recv()
    while True:
        msg = conn.recv()
        if msg[0] != "run":
            break
        t = time.perf_counter()
        for _ in range(msg[1]):
            oracle_sample_run(st)
        conn.send(time.perf_counter() - t)
    conn.close()


class OracleWorkers:
    """One spawned oracle process per host core (at most `cap`), each holding one
    logical rank's batch of the workload; run(reps) makes every process do reps
    passes at once and returns each one's seconds."""

    def __init__(self, w, inp, n_tok, cap=32):
        import multiprocessing as mp
        ctx = mp.get_context("spawn")  # never fork a process that has a CUDA context
        self.n = max(1, min(os.cpu_count() or 1, cap))
        n_ranks = max(1, w.B // n_tok)
        self.states = [oracle_sample_prepare(w, inp, (i % n_ranks) * n_tok, n_tok) for i in range(self.n)]
        self.conns, self.procs = [], []
        for st in self.states:
            a, b = ctx.Pipe()
            pr = ctx.Process(target=_oracle_worker_main, args=(b,), daemon=True)
            pr.start()
            a.send(st)
            self.conns.append(a)
            self.procs.append(pr)
        self.run(1)  # warm: imports and the oracle library loaded in every process

    def run(self, reps):
        for c in self.conns:
            c.send(("run", reps))
        return [c.recv() for c in self.conns]

    def close(self):
        for c in self.conns:
            try:
                c.send(("stop",))
            except Exception:
                pass
        for pr in self.procs:
            pr.join(timeout=10)


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_baseline(w, inp, target_s):
    """The oracle on the host: single-threaded, then one process per core (up to 32)
    each running one logical rank's batch, all at once for about target_s seconds.
    value = algorithmic bytes of all processes' passes / the slowest process's time."""
    n_tok = min(w.B, max(w.T, 1))
    st = oracle_sample_prepare(w, inp, 0, n_tok)
    oracle_sample_run(st)
    t = time.perf_counter()
    reps1 = 0
    while time.perf_counter() - t < min(2.0, target_s / 4) or reps1 < 1:
        oracle_sample_run(st)
        reps1 += 1
    t1 = (time.perf_counter() - t) / reps1
    single = st["bytes"] / t1 / 1e9
    pool = OracleWorkers(w, inp, n_tok)
    try:
        reps = max(1, int(round(target_s / t1)))
        secs = pool.run(reps)
    finally:
        pool.close()
    nbytes = sum(s["bytes"] for s in pool.states) * reps
    return {"value": nbytes / max(secs) / 1e9, "unit": "GB/s", "cores": pool.n, "kind": "oracle",
            "cpu_model": cpu_model(), "host_cpus": os.cpu_count(),
            "single_thread_value": single,
            "sample": "%d oracle processes (spawned, one per host core up to 32), each running %d passes "
                      "of one logical rank's %d tokens of the %s workload at once; plain C oracle; "
                      "value = all passes' algorithmic bytes / the slowest process's %.1f s; "
                      "single_thread_value: one process alone" % (pool.n, reps, n_tok, w.name, max(secs))}


# ----------------------------------------------------------------------------- reference arm


def run_reference(args):
    world, rank, local = dist_env()
    if world > 1 and rank != 0:
        return 0
    from combine_ep_layout_12_b200 import workloads as wl
    w = wl.get(args.workload)
    inp = wl.generate(w)
    n_tok = min(w.B, max(w.T, 1))
    pool = OracleWorkers(w, inp, n_tok)
    try:
        for _ in range(args.warmup):
            pool.run(1)
        total = 0.0
        for _ in range(args.steps):  # a step: every process does one pass at once
            total += max(pool.run(1))
    finally:
        pool.close()
    nbytes = sum(s["bytes"] for s in pool.states) * args.steps
    value = nbytes / total / 1e9
    sample = ("%d oracle processes (spawned, one per host core up to 32), each doing one pass of one "
              "logical rank's %d tokens of the %s workload per step; plain C oracle; step time = the "
              "slowest process's pass" % (pool.n, n_tok, w.name))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": config_dict(w),
        "tokens_per_s": pool.n * n_tok * args.steps / total,
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": pool.n, "kind": "oracle",
                         "cpu_model": cpu_model(), "host_cpus": os.cpu_count(), "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_dict(w):
    """The workload only (both arms report the same dict); how it was timed goes
    under the line's "method" key."""
    return {"workload": w.name, "B": w.B, "d": w.d, "E": w.E, "k": w.k, "P": w.P, "M": w.M,
            "n_zero": w.n_zero, "n_copy": w.n_copy, "n_const": w.n_const,
            "quant_mode": w.quant_mode, "payload": "int8" if w.quant_mode != 0 else "bf16",
            "routing": w.routing, "layout": "packed [B*k, d]" if w.layout == 1 else "low-latency [E, P*M, d]",
            "parallelism": "replicas (logical EP ranks inside each GPU)"}


# ----------------------------------------------------------------------------- our arm


class Workbench:
    """Device buffers of one workload, rotated over `R` sets, plus the CUDA graphs
    that time it: steps (ep_layout_dispatch -> ep_combine) and per-kernel loops."""

    def __init__(self, w, inp, device, stream, max_sets, flush_mb):
        import torch
        from combine_ep_layout_12_b200 import metrics, runner
        self.w, self.device, self.stream = w, device, stream
        set_bytes = w.rows * w.d * (1 if w.quant_mode != 0 else 2) + w.rows * 12 + 4 * w.B * w.d
        if w.quant_mode != 0:
            set_bytes += w.rows * w.d * 2
        free = torch.cuda.mem_get_info(device)[0]
        if set_bytes > 0.9 * free:
            raise MemoryError("%s needs %.1f GB of device memory, %.1f GB free"
                              % (w.name, set_bytes / 1e9, free / 1e9))
        # consecutive steps touch disjoint memory when two or more sets fit; with
        # one set, L2 is flushed between steps instead
        self.R = int(max(1, min(max_sets, (0.8 * free) // max(set_bytes, 1))))
        self.sets = []
        for _ in range(self.R):
            dev_inp = runner.to_device(inp, device)
            pipe = runner.Pipeline(w, device)
            with torch.cuda.stream(stream):
                pipe.layout(dev_inp, stream)
                pipe.dispatch(dev_inp, stream)
            stream.synchronize()
            assert pipe.buf.check(stream) == 0, "device error bits set"
            dp = pipe.buf.dst_pos
            rows = dp[dp >= 0].long()
            if w.quant_mode != 0:  # identity expert: expert_out rows = dequantized receive rows
                deq = pipe.buf.recv_x[rows].float()
                if w.quant_mode == 2:
                    deq = deq * pipe.buf.recv_scale[rows].unsqueeze(1)
                pipe.expert_out[rows] = deq.to(torch.bfloat16)
            self.sets.append((pipe, dev_inp))
        torch.cuda.synchronize(device)
        self.n_routed = int((self.sets[0][0].buf.dst_pos >= 0).sum().item())
        _, b_sp = metrics.routing_counts(w, inp["topk_idx"], self.n_routed, active=inp.get("active"))
        self.kbytes = metrics.kernel_bytes(w, self.n_routed, b_sp, smooth=inp["smooth"] is not None,
                                           masked=inp.get("active") is not None)
        self.step_bytes = sum(self.kbytes.values())
        self.flush = None
        if self.R == 1 and flush_mb:
            self.flush = torch.empty(flush_mb << 20, dtype=torch.uint8, device=device)
        self.S = 2 * self.R if self.R > 1 else 1
        units = w.d // 16 if w.quant_mode != 0 else w.d // 8
        # ep_layout_dispatch runs as one grid when T <= 128, k <= 8 and a row fits 128 threads
        self.one_grid = w.B > 0 and w.T <= 128 and w.k <= 8 and units <= 1024
        self.launches_per_step = 2 if self.one_grid else 3

    def capture(self, fn):
        import torch
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            fn()
        return g

    def steps_graph(self, n):
        def body():
            for i in range(n):
                if self.flush is not None:
                    self.flush.zero_()
                p, d = self.sets[i % self.R]
                p.step(d, self.stream)
        return self.capture(body)

    def kernel_graph(self, names):
        def body():
            for i in range(self.S):
                p, d = self.sets[i % self.R]
                for name in names:
                    if self.flush is not None:
                        self.flush.zero_()
                    getattr(p, name)(d, self.stream)
        return self.capture(body)

    def replay(self, g, n):
        """Replays g n times between two CUDA events; returns milliseconds."""
        import torch
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(self.stream):
            a.record(self.stream)
            for _ in range(n):
                g.replay()
            b.record(self.stream)
        b.synchronize()
        return a.elapsed_time(b)

    def read_flush(self):
        """Read a buffer three times the L2 size (one reduction kernel): afterwards
        L2 holds only clean lines of that buffer, so the next kernel reads its inputs
        from DRAM and its writes evict nothing that needs writing back, as under a
        profiler's cache flush.  Not launched with a programmatic edge, so the next
        kernel cannot start before it has finished."""
        import torch
        if self._rf_src is None:
            self._rf_src = torch.ones(self.READ_FLUSH_BYTES // 4, dtype=torch.float32, device=self.device)
            self._rf_out = torch.zeros((), dtype=torch.float32, device=self.device)
        torch.sum(self._rf_src, dim=0, out=self._rf_out)

    READ_FLUSH_BYTES = 384 << 20
    _rf_src = None
    _rf_out = None

    def isolated_times(self, reps, keys=("layout", "dispatch", "combine", "layout_dispatch")):
        """Per-launch milliseconds of each library call run alone: read_flush() (L2
        holds only clean lines of another buffer, the inputs are in DRAM), a CUDA
        event, the one call, a CUDA event; eager launches, so the call neither
        overlaps nor follows another launch of the library.  The median over `reps`
        such launches per call (buffer sets in rotation), as a trimmed mean: event
        times come in steps of about 1 us on this GPU, and the mean of many jittered
        samples resolves below the step where a median would sit on it.  The span
        between the events also holds the processing of the two event records:
        event_pair is the same measurement with nothing between the events, and it
        is subtracted (the difference follows ncu's gpu__time_duration of the same
        launches to within about 0.5 us); raw keeps the spans as measured."""
        import torch
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]

        def timed(name):
            with torch.cuda.stream(self.stream):
                for i in range(reps):
                    p, d = self.sets[i % self.R]
                    self.read_flush()
                    ev[i][0].record(self.stream)
                    if name:
                        getattr(p, name)(d, self.stream)
                    ev[i][1].record(self.stream)
            self.stream.synchronize()
            return trimmed_mean([a.elapsed_time(b) for a, b in ev])

        timed("layout")  # warm-up
        raw = {key: timed(key) for key in keys}
        pair = timed(None)
        out = {key: max(v - pair, 0.0) for key, v in raw.items()}
        out["event_pair"] = pair
        out["raw"] = raw
        return out

    def kernel_times(self, launches):
        """Per-launch milliseconds of each kernel and of the one-call layout+dispatch,
        from graphs of S back-to-back launches replayed about `launches / S` times.
        With one buffer set each launch is preceded by an L2 flush inside the graph;
        that memset is timed too and subtracted."""
        graphs = {"layout": ["layout"], "dispatch": ["dispatch"], "combine": ["combine"],
                  "layout+dispatch": ["layout", "dispatch"], "layout_dispatch": ["layout_dispatch"]}
        n_rep = max(1, launches // self.S)
        out = {}
        for key, names in graphs.items():
            g = self.kernel_graph(names)
            self.replay(g, 1)
            out[key] = self.replay(g, n_rep) / (n_rep * self.S)
        if self.flush is not None:
            def fbody():
                for _ in range(self.S):
                    self.flush.zero_()
            g = self.capture(fbody)
            self.replay(g, 1)
            f = self.replay(g, n_rep) / (n_rep * self.S)
            out = {k: v - f * (2 if k == "layout+dispatch" else 1) for k, v in out.items()}
        return out, n_rep


def run_ours(args):
    import torch
    from combine_ep_layout_12_b200 import build as ep_build
    from combine_ep_layout_12_b200 import runner
    from combine_ep_layout_12_b200 import workloads as wl

    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    ep_build.build()
    if args.sweep:
        return run_sweep(args, device)
    if args.profile_launches:
        return run_profile_launches(args, device)
    if args.shard:
        return run_shard(args, device)

    w = wl.get(args.workload)
    inp = wl.generate(w)
    stream = torch.cuda.Stream(device)
    wb = Workbench(w, inp, device, stream, args.sets, args.flush_mb)
    R, S, sets = wb.R, wb.S, wb.sets
    K = args.steps

    # one graph per set holding one step: warm-up and the per-step latency loop;
    # graphs of S consecutive steps over the sets: the timed throughput loop
    step_graphs = [wb.capture(lambda p=p, d=d: p.step(d, stream)) for p, d in sets]
    multi_graph = wb.steps_graph(S)
    rem_graph = wb.steps_graph(K % S) if K % S else None

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            if wb.flush is not None:
                wb.flush.zero_()
            step_graphs[i % R].replay()
        multi_graph.replay()
        if rem_graph is not None:
            rem_graph.replay()
    stream.synchronize()

    clocks = ClockSampler(device.index if device.index is not None else 0)
    clocks.start()
    time.sleep(0.05)
    # timed region: exactly K steps, as K // S replays of the S-step graph plus
    # one replay of a (K % S)-step graph
    t0_ev, t1_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dist, device)
    torch.cuda.synchronize(device)
    t_wall0 = time.perf_counter()
    with torch.cuda.stream(stream):
        t0_ev.record(stream)
        for _ in range(K // S):
            multi_graph.replay()
        if rem_graph is not None:
            rem_graph.replay()
        t1_ev.record(stream)
    torch.cuda.synchronize(device)
    barrier(dist, device)
    local_s = t0_ev.elapsed_time(t1_ev) / 1e3
    if wb.flush is not None:  # the flush memsets are inside the step graphs: take them out
        fg = wb.capture(lambda: [wb.flush.zero_() for _ in range(S)])
        wb.replay(fg, 1)
        local_s -= wb.replay(fg, max(1, K // S)) / 1e3 * (K / (max(1, K // S) * S))

    # per-step latency: single-step graph replays, CUDA events around each
    n_lat = min(K, 500)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * n_lat)]
    with torch.cuda.stream(stream):
        for i in range(n_lat):
            if wb.flush is not None:
                wb.flush.zero_()
            ev[2 * i].record(stream)
            step_graphs[i % R].replay()
            ev[2 * i + 1].record(stream)
    torch.cuda.synchronize(device)
    step_ms = [ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(n_lat)]

    kern_ms, n_rep = wb.kernel_times(K)
    iso_ms = wb.isolated_times(min(max(K, 30), 200))
    t_wall2 = time.perf_counter()
    clocks.mark(t_wall0, t_wall2)
    time.sleep(0.03)
    clocks.stop()
    for p, _ in sets:
        assert p.buf.check(stream) == 0, "device error bits set during the timed steps"

    job_s, job_bytes = aggregate(dist, local_s, float(wb.step_bytes * K), device)
    _, job_tokens = aggregate(dist, local_s, float(w.B * K), device)
    value = job_bytes / job_s / 1e9

    peak, peak_kind = measured_peak()
    # per kernel: isolated (one launch alone after an L2 read-flush, events around it;
    # the figure the roofline uses) and overlapped (graphs of back-to-back launches,
    # where a launch may start while the previous one drains: throughput, not latency)
    kernels = {}
    tot = sum(iso_ms[n] for n in ("layout", "dispatch", "combine"))
    for name in ("layout", "dispatch", "combine"):
        ms = iso_ms[name]
        ach = wb.kbytes[name] / (ms * 1e-3) / 1e9
        kernels[name] = {"us": 1e3 * ms, "bytes": wb.kbytes[name], "achieved_gbs": ach,
                         "frac_of_measured": ach / peak, "frac_of_8tbs": ach / SPEC_HBM_GBS,
                         "share": ms / tot, "us_overlapped": 1e3 * kern_ms[name],
                         "achieved_gbs_overlapped": wb.kbytes[name] / (kern_ms[name] * 1e-3) / 1e9}
    for name in kernels:
        kernels[name]["traffic"], kernels[name]["traffic_captured_on"] = recorded_traffic(w.name, name, True)
    dom = max(("dispatch", "combine", "layout"), key=lambda n: kernels[n]["share"])
    traffic = kernels[dom]["traffic"]
    roofline = {"bound": "hbm", "kernel": dom, "achieved": kernels[dom]["achieved_gbs"], "peak": peak,
                "unit": "GB/s", "frac": kernels[dom]["achieved_gbs"] / peak, "traffic": traffic,
                "peak_source": ("%s copy bandwidth (MEASURED_PEAKS.json hbm_gbs)" % peak_kind)
                if peak_kind == "measured" else "fallback 6.65 TB/s",
                "frac_of_8tbs_spec": kernels[dom]["achieved_gbs"] / SPEC_HBM_GBS,
                "algorithmic_bytes": wb.kbytes[dom],
                "duration": "isolated: trimmed mean over single eager launches, each after a read of a buffer "
                            "three times the L2 size, of the span between CUDA events around the launch, "
                            "minus the span of an empty event pair (%.2f us); raw span %.2f us"
                            % (1e3 * iso_ms["event_pair"], 1e3 * iso_ms["raw"][dom]),
                "traffic_captured_on": kernels[dom]["traffic_captured_on"],
                "traffic_note": "dram__bytes_read.sum + dram__bytes_write.sum of one ncu capture of this "
                                "kernel (per launch), recorded in profiles/traffic.json; null once the "
                                "kernel source has changed since. traffic_captured_on names the workload "
                                "the capture ran on: decode_e64 has the decode launch's tokens, hidden "
                                "size, picks and routed rows (so its traffic per launch) on a 64-expert "
                                "receive buffer that keeps the multi-pass capture near 1.4 GB"}

    # end to end through the public API with host buffers (eager calls, no graph).
    # Every step uploads its inputs from pinned host memory and reads its y back.
    # Streamed: uploads, steps and read-backs go on three streams ordered by
    # events, so step i's upload and step i-1's read-back overlap step i's kernels
    # and each other (the two copy directions use separate copy engines); a buffer
    # set is reused only after its previous step has finished and its y has been
    # read.  Serial: the same work on one stream, one step after another.
    e2e = None
    e2e_serial = None
    if not args.no_e2e:
        Ke = args.e2e_steps if args.e2e_steps is not None else min(K, 200)
        host = runner.to_device(inp, device, pin=True)
        y_host = [torch.empty((w.B, w.d), dtype=torch.bfloat16).pin_memory() for _ in range(R)]
        names = ("x", "topk_idx", "topk_weights")
        h2d = sum(host[n].numel() * host[n].element_size() for n in names)
        d2h = y_host[0].numel() * y_host[0].element_size()
        s_in = torch.cuda.Stream(device)
        s_out = torch.cuda.Stream(device)
        ev_in = [torch.cuda.Event() for _ in range(Ke)]
        ev_done = [torch.cuda.Event() for _ in range(Ke)]
        ev_out = [torch.cuda.Event() for _ in range(Ke)]
        t_begin = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        barrier(dist, device)
        torch.cuda.synchronize(device)
        t_begin.record(s_in)
        for i in range(Ke):
            p, d = sets[i % R]
            if i >= R:
                s_in.wait_event(ev_done[i - R])  # the set's inputs were read by step i - R
            with torch.cuda.stream(s_in):
                for n in names:
                    d[n].copy_(host[n], non_blocking=True)
            ev_in[i].record(s_in)
            stream.wait_event(ev_in[i])
            if i >= R:
                stream.wait_event(ev_out[i - R])  # the set's y was read back
            with torch.cuda.stream(stream):
                if wb.flush is not None:
                    wb.flush.zero_()
                p.step(d, stream)
            ev_done[i].record(stream)
            s_out.wait_event(ev_done[i])
            with torch.cuda.stream(s_out):
                y_host[i % R].copy_(p.y, non_blocking=True)
            ev_out[i].record(s_out)
        t_end.record(s_out)
        torch.cuda.synchronize(device)
        barrier(dist, device)
        loc = t_begin.elapsed_time(t_end) / 1e3
        js, jb = aggregate(dist, loc, float(wb.step_bytes * Ke), device)
        e2e = {"value": jb / js / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": Ke, "ms_per_step": 1e3 * js / Ke,
               "mode": "streamed: uploads, steps and read-backs on three event-ordered streams"}

        e0 = [torch.cuda.Event(enable_timing=True) for _ in range(Ke)]
        e1 = [torch.cuda.Event(enable_timing=True) for _ in range(Ke)]
        barrier(dist, device)
        torch.cuda.synchronize(device)
        with torch.cuda.stream(stream):
            for i in range(Ke):
                p, d = sets[i % R]
                if wb.flush is not None:
                    wb.flush.zero_()
                e0[i].record(stream)
                for n in names:
                    d[n].copy_(host[n], non_blocking=True)
                p.step(d, stream)
                y_host[0].copy_(p.y, non_blocking=True)
                e1[i].record(stream)
        torch.cuda.synchronize(device)
        barrier(dist, device)
        loc = sum(a.elapsed_time(b) for a, b in zip(e0, e1)) / 1e3
        js, jb = aggregate(dist, loc, float(wb.step_bytes * Ke), device)
        e2e_serial = {"value": jb / js / 1e9, "unit": "GB/s", "ms_per_step": 1e3 * js / Ke,
                      "mode": "serial: one stream, events around each step"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, inp, args.cpu_seconds)

    del step_graphs, multi_graph, rem_graph
    if dist is not None:
        dist.barrier(device_ids=[device.index])
        dist.destroy_process_group()
    if rank != 0:
        return 0
    cfg = config_dict(w)
    method = {
        "l2": ("%d buffer sets in rotation: consecutive steps touch disjoint memory "
               "(%.0f MB algorithmic per step, L2 126 MB)" % (R, wb.step_bytes / 1e6)) if R > 1 else
              ("flushed between steps (%d MB memset, timed alone and subtracted)" % args.flush_mb),
        "timing": ("K steps as replays of a CUDA graph of %d consecutive steps (ep_layout_dispatch -> "
                   "ep_combine, programmatic launch edges), CUDA events around the whole timed region; "
                   "step_latency_us_median: single-step graph replays with events around each" % S),
    }
    lps = wb.launches_per_step
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": 1e3 * job_s / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": cfg,
        "method": method,
        "tokens_per_s": job_tokens / job_s,
        "bytes_per_step": wb.step_bytes,
        "step_latency_us_median": 1e3 * statistics.median(step_ms),
        "kernels": kernels,
        "layout_then_dispatch_us": 1e3 * kern_ms["layout+dispatch"],
        "layout_dispatch_one_call_us": 1e3 * kern_ms["layout_dispatch"],
        "layout_dispatch_one_call_us_isolated": 1e3 * iso_ms["layout_dispatch"],
        "layout_dispatch_one_call_traffic": recorded_traffic(w.name, "layout_dispatch"),
        "comm_gbs_dispatch": wb.n_routed * w.d * (1 if w.quant_mode != 0 else 2)
        / (kern_ms["dispatch"] * 1e-3) / 1e9,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "e2e_serial": e2e_serial,
        "clocks": clocks.summary(),
        "gpu_launches": lps * K,
        "gpu_launches_latency_loop": lps * n_lat,
        "gpu_launches_kernel_loops": (5 + lps) * n_rep * S,
        "gpu_launches_isolated": 5 * min(max(K, 30), 200),
    }
    print(json.dumps(line), flush=True)
    return 0


def run_profile_launches(args, device):
    """Isolated launches of every call for a profiler: one buffer set, each call
    after a read-flush (so each starts on a clean L2 with its inputs in DRAM)."""
    import torch
    from combine_ep_layout_12_b200 import workloads as wl
    w = wl.get(args.workload)
    stream = torch.cuda.Stream(device)
    wb = Workbench(w, wl.generate(w), device, stream, 1, 0)
    p, d = wb.sets[0]
    with torch.cuda.stream(stream):
        for _ in range(args.profile_launches):
            for name in ("layout", "dispatch", "layout_dispatch", "combine"):
                wb.read_flush()
                getattr(p, name)(d, stream)
    stream.synchronize()
    assert p.buf.check(stream) == 0, "device error bits set"
    print("profile launches done: %s x %d" % (w.name, args.profile_launches), flush=True)
    return 0


def run_shard(args, device):
    """The multi-GPU form on one GPU: the P logical ranks of --workload in one process,
    each with its own slab allocation, reached through the pointer tables a multi-GPU
    run fills with mapped peer slabs; the ranks' kernels in turn on one stream, then on
    a stream per rank (as P GPUs run them).  Times, as CUDA graphs replayed K times:
    - one step of one micro-batch: every rank's layout, dispatch (with the in-kernel
      count exchange) and combine;
    - two micro-batches (different routing and tokens) one after the other;
    - the same two with the dual-batch overlap (shard.dbo, two streams).
    The expert outputs are filled once and not recomputed (the experts are not part
    of the path).  Prints one JSON line per arrangement; --sweep-out also writes them
    to a file."""
    import torch
    from combine_ep_layout_12_b200 import workloads as wl
    wa = wl.get(args.workload)
    wb_ = wa.with_(name=wa.name + "_b", seed=wa.seed + 1)
    stream = torch.cuda.Stream(device)
    side = torch.cuda.Stream(device)
    lines = []
    for rank_streams in (False, True):
        lines.append(_shard_times(args, device, wa, wb_, stream, side, rank_streams))
        print(json.dumps(lines[-1]), flush=True)
        torch.cuda.empty_cache()
    if args.sweep_out:
        with open(args.sweep_out, "w") as f:
            json.dump(lines, f, indent=1)
    return 0


def _shard_times(args, device, wa, wb_, stream, side, rank_streams):
    """The three graph timings of run_shard for one arrangement of the ranks."""
    import torch
    from combine_ep_layout_12_b200 import metrics, runner, shard
    from combine_ep_layout_12_b200 import workloads as wl
    shards, inputs, nbytes = [], [], 0.0
    for w in (wa, wb_):
        inp = wl.generate(w)
        n_routed, b_sp = metrics.routing_counts(w, inp["topk_idx"], active=inp.get("active"))
        kb = metrics.kernel_bytes(w, n_routed, b_sp, smooth=inp.get("smooth") is not None,
                                  masked=inp.get("active") is not None)
        nbytes += float(sum(kb.values()))
        sh = shard.LocalShards(w, device, rank_streams=rank_streams)
        for slab in sh.slabs:
            slab.expert_out.normal_()
        shards.append(sh)
        inputs.append(shard.split_inputs(w, runner.to_device(inp, device)))
    sa, sb = shards
    ra, rb = inputs
    with torch.cuda.stream(stream):
        sa.step(ra, None, stream)
        sb.step(rb, None, stream)
    stream.synchronize()
    for sh in shards:
        for rk in sh.ranks:
            assert rk.check() == 0, "device error bits set"

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        return g

    graphs = {"one_step": capture(lambda: sa.step(ra, None, stream)),
              "two_sequential": capture(lambda: (sa.step(ra, None, stream), sb.step(rb, None, stream))),
              "two_dbo": capture(lambda: shard.dbo(sa, sb, ra, rb, None, (stream, side)))}
    K = max(3, min(args.steps, 200))
    res = {}
    for name, g in graphs.items():
        for _ in range(max(3, args.warmup)):
            g.replay()
        torch.cuda.synchronize(device)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(K):
                g.replay()
        t1.record(stream)
        t1.synchronize()
        res[name] = 1e3 * t0.elapsed_time(t1) / K
    for sh in shards:
        for rk in sh.ranks:
            assert rk.check() == 0, "device error bits set"
    one = res["one_step"]
    line = {"mode": "shard, one GPU", "ranks": "concurrent, one stream per rank" if rank_streams else "in turn, one stream",
            "workload": wa.name, "P": wa.P, "T": wa.T, "steps": K,
            "one_step_us": one, "one_step_gbs": nbytes / 2 / (one * 1e-6) / 1e9,
            "two_sequential_us": res["two_sequential"], "two_dbo_us": res["two_dbo"],
            "dbo_speedup": res["two_sequential"] / res["two_dbo"]}
    del graphs
    return line


def fit_latency_bandwidth(points):
    """Least-squares fit of t = L + V / BW over (V bytes, t seconds) points."""
    V = np.array([p[0] for p in points], dtype=np.float64)
    t = np.array([p[1] for p in points], dtype=np.float64)
    A = np.stack([np.ones_like(V), V], axis=1)
    (L, inv_bw), *_ = np.linalg.lstsq(A, t, rcond=None)
    return {"L_us": 1e6 * L, "BW_eff_gbs": (1.0 / inv_bw) / 1e9 if inv_bw > 0 else None}


def run_sweep(args, device):
    """Tokens-per-rank sweep (P = 16, T in 1..4096) and the other named workloads:
    per-kernel times and GB/s, step time, and a latency/bandwidth fit per kernel.
    Writes one JSON document to --sweep-out and prints a table."""
    import torch
    from combine_ep_layout_12_b200 import workloads as wl
    names = args.sweep.split(",") if args.sweep != "all" else (
        ["sweep_T%d_q%d" % (T, q) for q in (2, 0) for T in wl.SWEEP_T] +
        ["decode", "skewed", "prefill", "tiny_q2"])
    stream = torch.cuda.Stream(device)
    peak, _ = measured_peak()
    results = []
    for name in names:
        w = wl.get(name)
        try:
            inp = wl.generate(w)
            wb = Workbench(w, inp, device, stream, args.sets, args.flush_mb)
        except MemoryError as exc:
            results.append({"workload": name, "skipped": str(exc)})
            print("%-18s skipped: %s" % (name, exc), flush=True)
            continue
        steps = max(wb.S, min(args.steps, 600))
        g = wb.steps_graph(wb.S)
        wb.replay(g, 2)
        n = max(1, steps // wb.S)
        step_ms = wb.replay(g, n) / (n * wb.S)
        if wb.flush is not None:
            fg = wb.capture(lambda: [wb.flush.zero_() for _ in range(wb.S)])
            wb.replay(fg, 1)
            step_ms -= wb.replay(fg, n) / (n * wb.S)
        kern_ms, _ = wb.kernel_times(steps)
        iso_ms = wb.isolated_times(min(steps, 100))
        for p, _ in wb.sets:
            assert p.buf.check(stream) == 0
        rec = {"workload": name, "B": w.B, "T": w.T, "P": w.P, "d": w.d, "E": w.E, "k": w.k,
               "quant_mode": w.quant_mode, "sets": wb.R, "step_us": 1e3 * step_ms,
               "step_gbs": wb.step_bytes / (step_ms * 1e-3) / 1e9,
               "tokens_per_s": w.B / (step_ms * 1e-3), "bytes": wb.kbytes,
               "layout_dispatch_one_call_us": 1e3 * kern_ms["layout_dispatch"]}
        for k in ("layout", "dispatch", "combine"):
            rec[k + "_us"] = 1e3 * iso_ms[k]
            rec[k + "_gbs"] = wb.kbytes[k] / (iso_ms[k] * 1e-3) / 1e9
            rec[k + "_frac_of_measured"] = rec[k + "_gbs"] / peak
            rec[k + "_us_overlapped"] = 1e3 * kern_ms[k]
        rec["event_pair_us"] = 1e3 * iso_ms["event_pair"]
        rec["raw_span_us"] = {k: 1e3 * v for k, v in iso_ms["raw"].items()}
        rec["layout_dispatch_one_call_us_isolated"] = 1e3 * iso_ms["layout_dispatch"]
        results.append(rec)
        print("%-18s T=%-5d step %8.1f us %7.0f GB/s | layout %7.1f us | dispatch %8.1f us %6.0f GB/s | "
              "combine %8.1f us %6.0f GB/s" % (name, w.T, rec["step_us"], rec["step_gbs"], rec["layout_us"],
                                               rec["dispatch_us"], rec["dispatch_gbs"], rec["combine_us"],
                                               rec["combine_gbs"]), flush=True)
        del wb, g
        torch.cuda.empty_cache()
    fits = {}
    for q in (0, 2):
        pts = [r for r in results if r.get("workload", "").startswith("sweep_") and
               r.get("quant_mode") == q and "step_us" in r]
        if len(pts) >= 3:
            fits["q%d" % q] = {k: fit_latency_bandwidth([(r["bytes"][k], r[k + "_us"] * 1e-6) for r in pts])
                               for k in ("dispatch", "combine")}
            fits["q%d" % q]["step"] = fit_latency_bandwidth(
                [(sum(r["bytes"].values()), r["step_us"] * 1e-6) for r in pts])
    doc = {"peak_gbs": peak, "results": results, "fits": fits}
    if args.sweep_out:
        with open(args.sweep_out, "w") as f:
            json.dump(doc, f, indent=1)
    print(json.dumps({"fits": fits}), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
