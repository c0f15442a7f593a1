#!/usr/bin/env python
"""Decode-step throughput of the SOCKET hot path on B200.

One step = one socket_decode call for all B x Hq query heads of one layer:
soft tables -> scoring -> top-k -> sparse attention (four kernels).  Inputs
(the bucket-id index, value norms, K/V cache, queries) are resident in HBM
before the timed region; steps rotate over several independently drawn
layers, so consecutive steps share no data and every step's inputs exceed
the 126 MB L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl socket|reference]

Multi-GPU (torchrun, one rank per GPU): every rank runs the same per-GPU
workload on its own data (weak scaling, no collective on the data path);
timing is the max over ranks of the device time.  Rank 0 prints one JSON line.

--impl reference times the CPU oracle (the only reference this method has)
on a bounded sample of the same workload, on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads as wl  # noqa: E402

METRIC = "SOCKET decode steps/sec at 128K ctx; HBM GB/s vs roofline (1×B200)"
UNIT = "steps/s"
FALLBACK_HBM_GBS = 6650.0


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------

def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured (MEASURED_PEAKS.json hbm_gbs, STREAM-style copy)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback 6650 GB/s (earlier measurement on this pool)"


def tensor_peak() -> float:
    """Measured dense bf16 TFLOP/s (burst) of MEASURED_PEAKS.json, else the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"])
    except Exception:
        return 1590.0


def profiled_traffic(kernel: str, workload: str, src_files):
    """DRAM bytes per launch from a committed ncu summary, if the kernel source
    is unchanged since the counters were taken; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel]
    except Exception:
        return None
    h = hashlib.sha256()
    for s in src_files:
        with open(os.path.join(ROOT, s), "rb") as f:
            h.update(f.read())
    if rec.get("source_sha256") != h.hexdigest() or rec.get("workload") != workload:
        return None
    return rec.get("dram_bytes_per_launch_full")


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.0005):
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.error = None
        self.errors = 0
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            handle = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                    handle = h
            if handle is None:
                handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nvml = pynvml
            self.handle = handle
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing or inaccessible
            self.error = f"{type(e).__name__}: {e}"

    def _sample(self):
        nv = self.nvml
        mhz = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
        try:
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
        except AttributeError:
            r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.handle)
        self.samples.append(mhz)
        self.reasons |= int(r) & ~0x1

    def sample_now(self):
        """One sample from the calling thread (while queued GPU work runs)."""
        if self.error is None or self.samples:
            try:
                self._sample()
            except Exception as e:
                self.errors += 1
                self.error = f"{type(e).__name__}: {e}"

    def _run(self):
        # A failed query is recorded and sampling goes on (one NVML error must
        # not end the clock record of the timed region).
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception as e:
                self.errors += 1
                self.error = f"{type(e).__name__}: {e}"
            time.sleep(self.period)

    def __enter__(self):
        if self.error is None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()
            try:
                self._sample()
            except Exception:
                pass

    def summary(self):
        if self.error is not None and not self.samples:
            return {"error": self.error}
        out = {"sm_mhz": float(statistics.median(self.samples)) if self.samples else None,
               "sm_max_mhz": float(self.max_mhz), "samples": len(self.samples),
               "reasons": [n for b, n in self.REASONS.items() if self.reasons & b]}
        if self.errors:
            out["query_errors"] = self.errors
            out["last_error"] = self.error
        return out


def max_over_ranks(x: float, world: int) -> float:
    """The largest of the ranks' values (every rank gets it)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, steps: int, ms_max: float) -> float:
    """Steps per second of the whole job: every rank ran `steps` steps of its
    own data (weak scaling), and the job took the slowest rank's time."""
    return world * steps / (ms_max * 1e-3)


def step_kernel_times(evs, n: int, path: int) -> dict:
    """Mean ms of each kernel of a decode step from the events the library
    recorded around its kernels (socket_set_step_events), named after the
    kernels the step's path launched (socket_last_decode_path)."""
    import soft_lsh_top_b200 as sk

    def gap(i):
        return statistics.fmean(evs[s][i].elapsed_time(evs[s][i + 1]) for s in range(n))
    if path == sk.SOCKET_STEP_ONE_KERNEL:
        return {"small_step": gap(0)}
    if path == sk.SOCKET_STEP_FUSED:
        return {"soft_tables": gap(0), "score": gap(1), "select_attend": gap(2)}
    return {name: gap(i) for i, name in enumerate(["soft_tables", "score", "topk", "attention"])}


def kernels_per_step(path: int, L: int) -> int:
    """Library kernels one decode step launches on its path (the scoring stage
    takes one launch per 64 tables)."""
    import soft_lsh_top_b200 as sk

    if path == sk.SOCKET_STEP_ONE_KERNEL:
        return 1
    return (2 if path == sk.SOCKET_STEP_FUSED else 3) + -(-L // 64)


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------------------
# CPU oracle timing (baseline leg and reference arm)
# ----------------------------------------------------------------------------

def oracle_decode_timing(w, K, V, q, W, units_kvh, min_seconds=2.0, reps_max=50):
    """Hash the sampled units with the oracle (untimed), then time the oracle
    decode of those units (OpenMP across units).  K, V: [Hkv, Ncap, d] CPU
    tensors of one batch row; q: [Hq, d].  Returns (seconds per rep, units,
    threads, seconds to hash the units)."""
    import oracle
    S = len(units_kvh)
    ids = np.zeros((S, w.L, w.ncap), dtype=np.uint8)
    vn = np.zeros((S, w.ncap), dtype=np.float32)
    th = time.perf_counter()
    for i, h in enumerate(units_kvh):
        a, v, _ = oracle.hash_keys(K[h, : w.N], V[h, : w.N], W, w.L, w.P)
        ids[i, :, : w.N] = a
        vn[i, : w.N] = v.astype(np.float32)
    hash_s = time.perf_counter() - th
    qs = torch.stack([q[h * w.G:(h + 1) * w.G] for h in units_kvh])
    Ks = torch.stack([K[h] for h in units_kvh])
    Vs = torch.stack([V[h] for h in units_kvh])
    threads = min(S, oracle.max_threads())
    oracle.set_num_threads(threads)
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.decode(qs, W, w.L, w.P, w.tau, ids, vn, Ks, Vs, w.N, w.k, want_scores=False)
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or reps >= reps_max:
            break
    return el / reps, S, threads, hash_s


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(w, inp):
    """The oracle's decode on a bounded sample of the workload's units, with
    OpenMP over those units, and on one unit with one thread."""
    import oracle
    units = list(range(min(w.Hkv, 8)))
    K = inp["K"][0].cpu()
    V = inp["V"][0].cpu()
    q, W = inp["q"][0].cpu(), inp["W"].cpu()
    t, S, threads, hash_s = oracle_decode_timing(w, K, V, q, W, units)
    t1, S1, _, _ = oracle_decode_timing(w, K, V, q, W, units[:1], min_seconds=1.0)
    oracle.set_num_threads(oracle.max_threads())
    value = 1.0 / (t * w.U / S)
    return {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
            "nproc": os.cpu_count(), "cpu_model": cpu_model(),
            "single_thread": {"value": 1.0 / (t1 * w.U / S1), "unit": UNIT, "cores": 1,
                              "sample": f"1 unit at full N={w.N}, {t1 * 1e3:.1f} ms; steps/s scaled by {w.U}"},
            "hash_keys_per_s": S * w.N / hash_s,
            "sample": f"{S} of {w.U} (batch, kv-head) units at full N={w.N}, oracle decode (soft tables, scores, "
                      f"top-k, attention) in fp64 with {threads} threads (one per unit), {t * 1e3:.1f} ms per "
                      f"sample; steps/s scaled by {w.U}/{S}"}


def run_reference(args, world: int, rank: int):
    if rank != 0:
        return 0
    import oracle
    w = wl.WORKLOADS[args.workload]
    inp = wl.make_inputs(w, "cpu", batches=[0])
    S = min(w.Hkv, oracle.max_threads())
    units = list(range(S))
    K, V, q, W = inp["K"][0], inp["V"][0], inp["q"][0], inp["W"]
    import oracle as orc
    ids = np.zeros((S, w.L, w.ncap), dtype=np.uint8)
    vn = np.zeros((S, w.ncap), dtype=np.float32)
    for i, h in enumerate(units):
        a, v, _ = orc.hash_keys(K[h, : w.N], V[h, : w.N], W, w.L, w.P)
        ids[i, :, : w.N] = a
        vn[i, : w.N] = v.astype(np.float32)
    qs = torch.stack([q[h * w.G:(h + 1) * w.G] for h in units])
    Ks, Vs = K[:S].contiguous(), V[:S].contiguous()
    orc.set_num_threads(S)
    step = lambda: orc.decode(qs, W, w.L, w.P, w.tau, ids, vn, Ks, Vs, w.N, w.k, want_scores=False)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    per_sample = el / max(args.steps, 1)
    value = 1.0 / (per_sample * w.U / S)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": per_sample * w.U / S * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d, "L": w.L,
                   "P": w.P, "tau": w.tau, "k": w.k, "kv_dtype": w.dtype},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": S, "kind": "oracle",
                         "sample": f"each step: oracle decode of {S} of {w.U} units at full N={w.N} "
                                   f"(OpenMP over units), scaled by {w.U}/{S}"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------
# the CUDA path
# ----------------------------------------------------------------------------

def time_workload(name: str, dev, steps: int = 100, flush_l2: bool = False):
    """Decode steps of another workload on this GPU (one layer).  Workloads
    larger than L2 replay a CUDA graph back to back; the small ones (whose
    data would stay in L2 between steps) are timed one step at a time with a
    write of 2 x L2 bytes before each, so every step starts cold."""
    import soft_lsh_top_b200 as sk
    w = wl.WORKLOADS[name]
    inp = wl.make_inputs(w, dev)
    ids, vn = sk.alloc_cache_index(w.B, w.Hkv, w.ncap, w.L, dev)
    sk.socket_hash_keys(inp["K"], inp["V"], inp["W"], ids, vn, 0, w.N)
    ws, idx, out = sk.alloc_decode_buffers(w.B, w.Hq, w.Hkv, w.ncap, w.L, w.P, w.k, dev)
    step = lambda: sk.socket_decode(inp["q"], inp["W"], ids, vn, inp["K"], inp["V"], w.N, w.tau, w.k, ws, idx, out)
    for _ in range(5):
        step()
    torch.cuda.synchronize()
    peak, _ = hbm_peak()
    if flush_l2:
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        junk = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for a, b in evs:
            junk.fill_(1)
            a.record()
            step()
            b.record()
        torch.cuda.synchronize()
        us = statistics.median(a.elapsed_time(b) for a, b in evs) * 1e3
        how = "one step at a time, L2 overwritten before each step; median of CUDA-event times around the step"
        del junk
    else:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            g.replay()
        b.record()
        torch.cuda.synchronize()
        us = a.elapsed_time(b) / steps * 1e3
        how = "CUDA graph of one step replayed back to back (inputs larger than L2)"
        del g
    assert sk.read_device_error(ws) == 0
    res = {"B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "L": w.L, "P": w.P, "tau": w.tau, "k": w.k,
           "kv_dtype": w.dtype, "us_per_step": us, "steps_per_s": 1e6 / us, "bytes_per_step": w.step_bytes(),
           "step_roofline_frac": w.step_bytes() / (us * 1e-6) / 1e9 / peak, "how": how}
    del inp, ids, vn, ws, idx, out
    torch.cuda.empty_cache()
    return res


def run_socket(args, world: int, rank: int, local_rank: int):
    import soft_lsh_top_b200 as sk
    from soft_lsh_top_b200 import _build
    _build.build()  # no-op when the in-tree library is current
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    w = wl.WORKLOADS[args.workload]
    if args.batch and args.batch != w.B:
        # A smaller batch of the same workload (profiling captures); renamed so
        # nothing measured on it passes for the full workload.
        w = w.scaled(B=args.batch, name=f"{w.name}_batch{args.batch}")
    R = args.layers
    layers = []
    for li in range(R):
        wi = w.scaled(seed=w.seed + 1000 * li + 7919 * rank)
        inp = wl.make_inputs(wi, dev)
        ids, vn = sk.alloc_cache_index(w.B, w.Hkv, w.ncap, w.L, dev)
        sk.socket_hash_keys(inp["K"], inp["V"], inp["W"], ids, vn, 0, w.N)
        layers.append((inp, ids, vn))
    torch.cuda.synchronize()
    ws, idx, out = sk.alloc_decode_buffers(w.B, w.Hq, w.Hkv, w.ncap, w.L, w.P, w.k, dev)

    def step(s, q=None):
        inp, ids, vn = layers[s % R]
        sk.socket_decode(inp["q"] if q is None else q, inp["W"], ids, vn, inp["K"], inp["V"], w.N, w.tau, w.k,
                         ws, idx, out)

    for s in range(args.warmup):
        step(s)
    torch.cuda.synchronize()

    # One CUDA graph holds R consecutive decode steps, one per layer, so the
    # kernels chain by programmatic dependent launch across steps as well
    # (graph edges); the timed loop replays it K // R times and runs the
    # K % R remaining steps as direct calls.
    graph, launch = None, "direct C-ABI calls, one stream"
    if not args.no_graph:
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                for li in range(R):
                    step(li)
            for _ in range(max(1, args.warmup // R)):
                graph.replay()
            torch.cuda.synchronize()
            assert sk.read_device_error(ws) == 0
            launch = f"CUDA graph replay ({R} decode steps per graph, one per layer)"
        except Exception as exc:  # capture unsupported here: time direct calls
            graph = None
            launch = f"direct C-ABI calls, one stream (graph capture failed: {type(exc).__name__})"

    # ---- timed region: K steps back to back (kernels chain by programmatic
    # dependent launch; nothing is recorded between them).
    K = args.steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clocks:
        start.record()
        if graph is not None:
            for _ in range(K // R):
                graph.replay()
            for s in range(K % R):
                step(s)
        else:
            for s in range(K):
                step(s)
        clocks.sample_now()  # the queue still holds most of the steps
        end.record()
        torch.cuda.synchronize()
    graph = None
    barrier(world)
    ms_total = max_over_ranks(start.elapsed_time(end), world)
    assert sk.read_device_error(ws) == 0

    # ---- per-kernel durations: a second pass with events recorded by the
    # library between the kernels, on the launching stream.  The events
    # serialise the kernels, so these are each kernel's own time.
    KD = min(K, 200)
    nk = 4  # kernel slots of a step's events (socket_set_step_events)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(KD)]
    for row in evs:  # torch creates the CUDA event on first record
        for e in row:
            e.record()
    torch.cuda.synchronize()
    for s in range(KD):
        sk.socket_set_step_events(evs[s])
        step(s)
    torch.cuda.synchronize()
    sk.socket_set_step_events([])
    path = sk.socket_last_decode_path()
    kern_ms = step_kernel_times(evs, KD, path)
    assert sk.read_device_error(ws) == 0

    # ---- prefill: hashing a whole layer (socket_hash_keys), for the hash
    # kernel's roofline.  Not part of the decode step.
    inp0, ids0, vn0 = layers[0]
    for _ in range(2):
        sk.socket_hash_keys(inp0["K"], inp0["V"], inp0["W"], ids0, vn0, 0, w.N)
    torch.cuda.synchronize()
    RH = 5
    h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0.record()
    for _ in range(RH):
        sk.socket_hash_keys(inp0["K"], inp0["V"], inp0["W"], ids0, vn0, 0, w.N)
    h1.record()
    torch.cuda.synchronize()
    sk.socket_hash_check()
    hash_ms = max_over_ranks(h0.elapsed_time(h1) / RH, world)

    # ---- one selection per query head (socket_decode_per_head) on the same
    # layers: direct calls, then a pass with events between the kernels.
    ws_h, idx_h, out_h = sk.alloc_decode_buffers(w.B, w.Hq, w.Hkv, w.ncap, w.L, w.P, w.k, dev, per_head=True)

    def step_h(s):
        inp, ids, vn = layers[s % R]
        sk.socket_decode_per_head(inp["q"], inp["W"], ids, vn, inp["K"], inp["V"], w.N, w.tau, w.k,
                                  ws_h, idx_h, out_h)

    for s in range(args.warmup):
        step_h(s)
    torch.cuda.synchronize()
    KH = min(K, 100)
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    p0.record()
    for s in range(KH):
        step_h(s)
    p1.record()
    torch.cuda.synchronize()
    ph_ms = max_over_ranks(p0.elapsed_time(p1), world)
    KHD = min(KH, 50)
    evs_h = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(KHD)]
    for row in evs_h:
        for e in row:
            e.record()
    torch.cuda.synchronize()
    for s in range(KHD):
        sk.socket_set_step_events(evs_h[s])
        step_h(s)
    torch.cuda.synchronize()
    sk.socket_set_step_events([])
    ph_kern = step_kernel_times(evs_h, KHD, sk.socket_last_decode_path())
    assert sk.read_device_error(ws_h) == 0
    del ws_h, idx_h, out_h, evs_h
    torch.cuda.empty_cache()

    # ---- decode steps that append one key each (the append-mix workload):
    # hash + decode as two calls, and the fused socket_decode_append.
    wa = wl.APPEND_MIX.scaled(seed=wl.APPEND_MIX.seed + 7919 * rank)
    ia = wl.make_inputs(wa, dev)
    ids_a, vn_a = sk.alloc_cache_index(wa.B, wa.Hkv, wa.ncap, wa.L, dev)
    sk.socket_hash_keys(ia["K"], ia["V"], ia["W"], ids_a, vn_a, 0, wa.N)
    ws_a, idx_a, out_a = sk.alloc_decode_buffers(wa.B, wa.Hq, wa.Hkv, wa.ncap, wa.L, wa.P, wa.k, dev)

    def two_calls(t):
        sk.socket_hash_keys(ia["K"], ia["V"], ia["W"], ids_a, vn_a, wa.N + t, wa.N + t + 1)
        sk.socket_decode(ia["q_steps"][t], ia["W"], ids_a, vn_a, ia["K"], ia["V"], wa.N + t + 1, wa.tau, wa.k,
                         ws_a, idx_a, out_a)

    def fused(t):
        sk.socket_decode_append(ia["q_steps"][t], ia["W"], ids_a, vn_a, ia["K"], ia["V"], wa.N + t + 1, wa.tau,
                                wa.k, 1, ws_a, idx_a, out_a)

    append = {"what": "64 decode steps that each append one key (hash + decode), append-mix workload: "
                      "socket_hash_keys + socket_decode vs the fused socket_decode_append; each variant's 64 "
                      "steps captured in one CUDA graph and replayed",
              "workload": wa.name, "B": wa.B, "Hq": wa.Hq, "Hkv": wa.Hkv, "N": wa.N, "L": wa.L, "P": wa.P,
              "k": wa.k}
    for name, fn in (("two_calls", two_calls), ("fused", fused)):
        for t in range(wa.appends):  # warm-up
            fn(t)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for t in range(wa.appends):
                fn(t)
        g.replay()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a0.record()
        for _ in range(3):
            g.replay()
        a1.record()
        torch.cuda.synchronize()
        ms = a0.elapsed_time(a1) / 3
        append[name] = {"steps_per_s": wa.appends / (ms * 1e-3), "us_per_step": 1e3 * ms / wa.appends}
        del g
    # Per-kernel times of the decode step of each variant (events between its kernels).
    for name, fn in (("two_calls", two_calls), ("fused", fused)):
        ev_a = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(wa.appends)]
        for row in ev_a:
            for e in row:
                e.record()
        torch.cuda.synchronize()
        for t in range(wa.appends):
            sk.socket_set_step_events(ev_a[t])
            fn(t)
        torch.cuda.synchronize()
        sk.socket_set_step_events([])
        append[name]["decode_kernels_us"] = {
            n: 1e3 * v for n, v in step_kernel_times(ev_a, wa.appends, sk.socket_last_decode_path()).items()}
    # Prefill of this workload (L * P = 480 hyperplanes: two tensor-core passes).
    h0.record()
    for _ in range(3):
        sk.socket_hash_keys(ia["K"], ia["V"], ia["W"], ids_a, vn_a, 0, wa.N)
    h1.record()
    torch.cuda.synchronize()
    pre_ms = h0.elapsed_time(h1) / 3
    pre_keys = wa.B * wa.Hkv * wa.N
    pre_bytes = pre_keys * (2 * wa.d * wa.elem_bytes + sk.socket_ids_row_bytes(wa.L) + 4)
    append["prefill"] = {"keys": pre_keys, "ms": pre_ms, "algorithmic_bytes": pre_bytes,
                         "gbs": pre_bytes / (pre_ms * 1e-3) / 1e9}
    sk.socket_hash_check()
    assert sk.read_device_error(ws_a) == 0
    del ia, ids_a, vn_a, ws_a, idx_a, out_a
    torch.cuda.empty_cache()

    # ---- end to end through the public API with host buffers: every step
    # copies its query in from pinned host memory and its output and indices
    # back.  The copies run on a second stream, double-buffered and ordered by
    # events, so one step's transfers overlap the neighbouring steps' kernels.
    q_host = [torch.empty_like(l[0]["q"], device="cpu").pin_memory() for l in layers]
    for l, qh in zip(layers, q_host):
        qh.copy_(l[0]["q"])
    comp = torch.cuda.current_stream(dev)
    copy_stream = torch.cuda.Stream(device=dev)
    q_dev = [torch.empty_like(layers[0][0]["q"]) for _ in range(2)]
    out_dev = [out, torch.empty_like(out)]
    idx_dev = [idx, torch.empty_like(idx)]
    out_host = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    idx_host = [torch.empty(idx.shape, dtype=idx.dtype).pin_memory() for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]    # query of the step in buffer b is on the device
    ev_done = [torch.cuda.Event() for _ in range(2)]  # the step of buffer b has finished its kernels
    ev_out = [torch.cuda.Event() for _ in range(2)]   # the step of buffer b is back on the host

    def h2d(s):
        b = s % 2
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(ev_done[b])  # the step two back has read this buffer
            q_dev[b].copy_(q_host[s % R], non_blocking=True)
            ev_in[b].record(copy_stream)

    def e2e_steps(n):
        h2d(0)
        for s in range(n):
            b = s % 2
            if s + 1 < n:
                h2d(s + 1)
            comp.wait_event(ev_in[b])
            comp.wait_event(ev_out[b])  # the step two back has left this output buffer
            inp_s, ids_s, vn_s = layers[s % R]
            sk.socket_decode(q_dev[b], inp_s["W"], ids_s, vn_s, inp_s["K"], inp_s["V"], w.N, w.tau, w.k, ws,
                             idx_dev[b], out_dev[b])
            ev_done[b].record(comp)
            with torch.cuda.stream(copy_stream):
                copy_stream.wait_event(ev_done[b])
                out_host[b].copy_(out_dev[b], non_blocking=True)
                idx_host[b].copy_(idx_dev[b], non_blocking=True)
                ev_out[b].record(copy_stream)
        comp.wait_event(ev_out[(n - 1) % 2])

    e2e_steps(args.warmup)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    copy_stream.wait_event(e0)
    e2e_steps(K)
    e1.record(comp)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    assert sk.read_device_error(ws) == 0
    h2d_bytes = q_dev[0].numel() * q_dev[0].element_size()
    d2h_bytes = out.numel() * out.element_size() + idx.numel() * idx.element_size()

    result = None
    if rank == 0:
        ms_step = ms_total / K
        bytes_step = w.step_bytes()
        peak, peak_src = hbm_peak()
        # The dominant kernel: scoring (its ids and norms), or the one kernel
        # of a small step (the whole step's bytes).
        if "score" in kern_ms:
            dom_kernel, dom_bytes, dom_ms = "score_kernel", w.U * w.N * (w.L + 4), kern_ms["score"]
        else:
            dom_kernel, dom_bytes, dom_ms = "small_step_kernel", bytes_step, kern_ms["small_step"]
        dom_gbs = dom_bytes / (dom_ms * 1e-3) / 1e9
        attn_bytes = w.U * 2 * w.k * w.d * w.elem_bytes
        # The gather kernel's own rate, where the step runs it on its own.
        attn_gbs = attn_bytes / (kern_ms["attention"] * 1e-3) / 1e9 if "attention" in kern_ms else None
        keys = w.U * w.N
        hash_bytes = keys * (2 * w.d * w.elem_bytes + sk.socket_ids_row_bytes(w.L) + 4)
        hash_flops = 2.0 * keys * w.d * w.L * w.P
        bf16_peak = tensor_peak()
        hash_gbs = hash_bytes / (hash_ms * 1e-3) / 1e9
        hash_tflops = hash_flops / (hash_ms * 1e-3) / 1e12
        prefill = {
            "what": "socket_hash_keys over the whole layer (all units, N keys each); not in the decode step",
            "kernel": "hash_umma_kernel" if w.dtype == "bf16" else "hash_kernel",
            # tcgen05 passes over whole 32-table blocks of at most 256 hyperplanes
            "passes": -(-w.L // (32 * max(1, 256 // (32 * w.P)))) if w.dtype == "bf16" else 1,
            "keys": keys, "ms": hash_ms, "keys_per_s": world * keys / (hash_ms * 1e-3),
            "algorithmic_bytes": hash_bytes, "gbs": hash_gbs, "hbm_frac": hash_gbs / peak,
            "flops": hash_flops, "tflops": hash_tflops,
            "tensor_frac": hash_tflops / bf16_peak if w.dtype == "bf16" else None,
            "bound": "hbm" if hash_bytes / (peak * 1e9) >= hash_flops / (bf16_peak * 1e12) else "tensor",
        }
        # Per-head scoring reads each kv unit's ids and norms once (its heads'
        # CTAs stream them side by side) and writes a score row per head.
        ph_score_bytes = w.U * w.N * (w.L + 4) + w.U * w.G * w.N * 4
        ph_score_ms = ph_kern.get("score", ph_kern.get("small_step"))
        ph_score_gbs = ph_score_bytes / (ph_score_ms * 1e-3) / 1e9
        # Each (head, key, table) is one 4-byte shared-memory lookup: per head
        # that is the whole lookup stream, bound by the SMs' shared-memory
        # bandwidth (128 B per clock per SM) at the sampled SM clock.
        ck = clocks.summary()
        mhz = ck.get("sm_mhz") or ck.get("sm_max_mhz") or 1965.0
        n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
        smem_peak = n_sm * 128 * mhz * 1e6 / 1e9
        lookup_bytes = w.U * w.G * w.N * w.L * 4
        lookup_gbs = lookup_bytes / (ph_score_ms * 1e-3) / 1e9
        per_head = {
            "what": "socket_decode_per_head: one selection per query head (B*Hq units) on the same layers; "
                    "direct calls",
            "steps_per_s": whole_job_rate(world, KH, ph_ms), "ms_per_step": ph_ms / KH, "steps": KH,
            "kernels_ms": ph_kern,
            "score": {"hbm_algorithmic_bytes": ph_score_bytes, "hbm_gbs": ph_score_gbs, "hbm_frac": ph_score_gbs / peak,
                      "bound": "smem", "lookup_bytes": lookup_bytes, "achieved": lookup_gbs, "peak": smem_peak,
                      "unit": "GB/s", "frac": lookup_gbs / smem_peak,
                      "peak_source": f"derived: {n_sm} SMs x 128 B/clock x {mhz:.0f} MHz (sampled SM clock)"},
            "attention_gbs": (w.U * w.G * 2 * w.k * w.d * w.elem_bytes / (ph_kern["attention"] * 1e-3) / 1e9
                              if "attention" in ph_kern else None),
        }
        traffic = (profiled_traffic("score_kernel", w.name, ["soft_lsh_top_b200/csrc/score.cu",
                                                             "soft_lsh_top_b200/csrc/common.cuh"])
                   if dom_kernel == "score_kernel" else None)
        result = {
            "metric": METRIC, "value": whole_job_rate(world, K, ms_total), "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "data": "synthetic",
            "dtype": ("bf16 K/V and q, f32 scores, softmax and outputs" if w.dtype == "bf16" else "f32"),
            "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d, "L": w.L,
                       "P": w.P, "tau": w.tau, "k": w.k, "kv_dtype": w.dtype},
            "run": {"parallelism": f"replicas{world}",
                    "l2": f"inputs larger than L2: {bytes_step / 1e6:.0f} MB per step, {R} rotating layers "
                          "of independent data", "launch": launch},
            "bytes_per_step": bytes_step,
            "step_hbm_gbs": bytes_step / (ms_step * 1e-3) / 1e9,
            "step_roofline_frac": bytes_step / (ms_step * 1e-3) / 1e9 / peak,
            "kernels_ms": kern_ms,
            "roofline": {"bound": "hbm", "kernel": dom_kernel, "achieved": dom_gbs, "peak": peak,
                         "unit": "GB/s", "frac": dom_gbs / peak, "traffic": traffic,
                         "algorithmic_bytes_per_launch": dom_bytes, "peak_source": peak_src,
                         "step": {"what": "the whole decode step: ids + norms + 2 k d 2 bytes per kv "
                                          "head, over ms_per_step", "achieved": bytes_step / (ms_step * 1e-3) / 1e9,
                                  "frac": bytes_step / (ms_step * 1e-3) / 1e9 / peak, "bytes": bytes_step,
                                  "target_frac": 0.70},
                         "attention_gbs": attn_gbs},
            "gpu_launches": kernels_per_step(path, w.L) * K,
            "step_kernels": list(kern_ms),
            "clocks": clocks.summary(),
            "prefill": prefill,
            "per_head": per_head,
            "append": append,
            "e2e": {"value": whole_job_rate(world, K, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d_bytes,
                    "d2h_bytes_per_step": d2h_bytes,
                    "how": "socket_decode per step (direct calls); query copied in from pinned host memory and "
                           "output + indices copied back every step, on a copy stream double-buffered against "
                           "the kernels"},
        }
        if not args.no_workloads:
            # The other workloads of the method's long-context range, same GPU.
            result["workloads"] = {
                wl.MILLION.name: time_workload(wl.MILLION.name, dev, steps=100),
                wl.LLAMA_32K.name: time_workload(wl.LLAMA_32K.name, dev, steps=100, flush_l2=True),
                wl.TINY.name: time_workload(wl.TINY.name, dev, steps=100, flush_l2=True),
            }
        if world == 1 and not args.no_cpu_baseline:
            result["cpu_baseline"] = cpu_baseline(w, layers[0][0])
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["socket", "reference"], default="socket")
    ap.add_argument("--workload", default=wl.BATCH8_128K.name, choices=sorted(wl.WORKLOADS))
    ap.add_argument("--layers", type=int, default=3, help="independently drawn layers rotated across steps")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true", help="skip the other workloads' step times")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (profiling captures)")
    ap.add_argument("--no-graph", action="store_true", help="time direct calls instead of CUDA graph replay")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args, world, rank)
    return run_socket(args, world, rank, local_rank)


if __name__ == "__main__":
    sys.exit(main())
