#!/usr/bin/env python
"""Throughput of the bit-packed binary-weight x ternary-activation path.

Default workload: the LLaMA-7B-shaped projections (K, N) in {(4096, 4096),
(4096, 11008), (11008, 4096)} with per-128-column weight scales. One step =
the decode phase (the three M=1 activation rows ternarized and multiplied by
the three weight matrices in one fused launch), then for each shape: ternarize
the prefill activations (M=2048, E4M3 bytes) and run the tensor-core GEMM.
Weights are binarized and packed once, before timing (an offline step). The
popcount GEMM on the same prefill products is timed beside the step.

Metric: effective TOPS = sum over the step's products of 2*M*N*K, divided by
the device time of the step (CUDA-graph replay, L2 flushed between steps by a
256 MiB write). With torchrun, every rank runs the same step on its own batch
(weak scaling, no data-path collective) and the time is the max over ranks.

--impl reference times the CPU oracle (a plain C loop over unpacked values)
on a bounded row sample of the same workload. --workload selects the other
measured rows: llama_prefill, llama_decode, llama_decode_batched,
llama_decode_model, gemv_big, bert, tiny, attn, billm1, billm16, billm512, pack
(comma separated, or all).
"""
from __future__ import annotations

import argparse
import csv
import io
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time
from datetime import timedelta

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "bit-packed bin x tern GEMM effective TOPS & % roofline at LLaMA-7B shapes"
UNIT = "TOPS"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_HBM_GBS = 6650.0


# ------------------------------------------------------------------ plumbing
def dist_info():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def dist_init(backend: str):
    world, rank, local = dist_info()
    if world > 1 and not torch.distributed.is_initialized():
        torch.distributed.init_process_group(backend, timeout=timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(x: float, device=None) -> float:
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier():
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.barrier()


def weak_scaling_value(units_per_rank_step: float, steps: int, world: int, max_seconds: float):
    """Whole-job throughput: units processed by all ranks / the slowest rank's time."""
    return units_per_rank_step * steps * world / max_seconds


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": FALLBACK_HBM_GBS}, "fallback"


# DRAM traffic of the tensor-core GEMM per launch, from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum of the three prefill launches
# of `bench.py --steps 2 --warmup 1`, averaged): 11.07, 45.36 and 29.89 MB for
# K x N = 4096x4096, 4096x11008, 11008x4096 at M = 2048. Valid only for the
# kernel source it was taken on; reported as null once that file changes.
TC_TRAFFIC = {"source": "binarized_transformer_b200/csrc/gemm_tc.cu",
              "sha256": "8e7c93859df902da794099f85b99b4b2f2fca0f374fb2a490df91bffd3fb50b7",
              "bytes_per_launch": 28772693}


def tc_traffic():
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), TC_TRAFFIC["source"])
    try:
        with open(path, "rb") as f:
            ok = hashlib.sha256(f.read()).hexdigest() == TC_TRAFFIC["sha256"]
    except OSError:
        ok = False
    return TC_TRAFFIC["bytes_per_launch"] if ok else None


class ClockSampler:
    """SM clock, power and clock-event (throttle) reasons sampled while the
    timed region runs: NVML polled from a thread every 2 ms (the
    region can be far shorter than nvidia-smi's sampling period), falling back
    to `nvidia-smi -lms 50`. Read-only queries: no setting is changed."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
            "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}

    def __init__(self, cuda_index: int, interval: float = 0.002):
        self.cuda_index = cuda_index
        self.interval = interval
        self.samples = []   # (sm_mhz, power_w, reason_bits)
        self.max_mhz = None
        self.source = None
        self.proc = None
        self._stop = None

    def _nvml_handle(self, nv):
        n = nv.nvmlDeviceGetCount()
        if n == 1:
            return nv.nvmlDeviceGetHandleByIndex(0)
        uuid = str(getattr(torch.cuda.get_device_properties(self.cuda_index), "uuid", ""))
        for i in range(n):
            h = nv.nvmlDeviceGetHandleByIndex(i)
            u = nv.nvmlDeviceGetUUID(h)
            u = u.decode() if isinstance(u, bytes) else u
            if uuid and uuid in u:
                return h
        return nv.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def __enter__(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._nvml_handle(nv)
            reasons_fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self._stop = threading.Event()

            def loop():
                while not self._stop.is_set():
                    try:
                        self.samples.append((float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                             nv.nvmlDeviceGetPowerUsage(h) / 1000.0,
                                             int(reasons_fn(h))))
                    except Exception:
                        pass
                    self._stop.wait(self.interval)

            self._thread = threading.Thread(target=loop, daemon=True)
            self._thread.start()
            self.source = "nvml"
        except Exception:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.cuda_index}", f"--query-gpu={self.Q}",
                     "--format=csv,noheader,nounits", "-lms", "50"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.source = "nvidia-smi"
            except OSError:
                self.proc = None
        return self

    def __exit__(self, *exc):
        if self._stop is not None:
            self._stop.set()
            self._thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for r in csv.reader(io.StringIO(out or "")):
                if len(r) < 9:
                    continue
                bits = 0
                for nm, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        bits |= self.BITS[nm]
                self.samples.append((float(r[1]), float(r[3]), bits))
                self.max_mhz = float(r[2])

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"],
                    "samples": 0, "source": self.source}
        reasons = sorted(n for n, b in self.BITS.items() if any(s[2] & b for s in self.samples))
        return {"sm_mhz": statistics.median(s[0] for s in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples),
                "power_w_max": round(max(s[1] for s in self.samples), 1), "source": self.source}


class L2Flusher:
    """Between timed steps: write a 256 MiB buffer (twice the 126 MB L2), then
    read another 256 MiB buffer. The write evicts everything the last step left
    in L2; the read replaces the flush's own dirty lines with clean ones, so the
    timed kernels start cold and none of their reads waits behind a write-back
    of the flush."""

    def __init__(self):
        self.buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        self.rbuf = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.int32, device="cuda")

    def __call__(self):
        self.buf.zero_()
        self.rbuf.sum(dtype=torch.int64)


def event_pair():
    return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)


def gpu_head_start(us: float = 200.0):
    """Keep the GPU busy (outside the timed region) long enough for the host to
    enqueue the timed launches, so that enqueue latency is not timed."""
    torch.cuda._sleep(int(us * 2000))


# ------------------------------------------------------------------ workloads
class LlamaStep:
    """Decode GEMVs then prefill GEMMs for the three LLaMA-7B projection shapes."""

    def __init__(self, rank: int, M_prefill: int = 2048, M_decode: int = 1, prefill_path: str = "tc"):
        import binarized_transformer_b200 as bt
        self.bt = bt
        self.prefill_path = prefill_path  # "tc": tensor cores (E4M3); "popc": LOP3+POPC tiles
        self.shapes = workloads.LLAMA_SHAPES
        self.group = workloads.LLAMA_GROUP
        self.M = {"prefill": M_prefill, "decode": M_decode}
        self.w = []
        self.X = {"prefill": [], "decode": []}
        self.X_host = {"prefill": [], "decode": []}
        self.planes = {"prefill": [], "decode": []}
        self.Y = {"prefill": [], "decode": []}
        for s, (K, N) in enumerate(self.shapes):
            W = torch.from_numpy(workloads.llama_weights(s)).cuda()
            self.w.append(bt.bwta_pack_weights(W, self.group))
            del W
            for phase in ("decode", "prefill"):
                M = self.M[phase]
                Xh = torch.from_numpy(workloads.llama_acts(s, M, stream=rank)).pin_memory()
                self.X_host[phase].append(Xh)
                self.X[phase].append(Xh.cuda())
                ld = bt.ld_words_for(K)
                self.planes[phase].append((
                    torch.empty((M, ld), dtype=torch.int32, device="cuda"),
                    torch.empty((M, ld), dtype=torch.int32, device="cuda"),
                    torch.empty((M,), dtype=torch.float32, device="cuda"),
                    torch.empty((M, 32 * ld), dtype=torch.uint8, device="cuda")))
                self.Y[phase].append(torch.empty((M, N), dtype=torch.float32, device="cuda"))
        self.Y_host = {p: [torch.empty(y.shape, dtype=y.dtype).pin_memory() for y in self.Y[p]]
                       for p in self.Y}
        # the decode phase: the three projections in one fused launch
        self.decode_desc = bt.decode_jobs([(self.X["decode"][s], self.w[s][0], self.w[s][1],
                                            self.group, self.Y["decode"][s], None)
                                           for s in range(len(self.shapes))])
        torch.cuda.synchronize()

    def decode_launch(self):
        """The decode phase: ternarize the three M=1 rows and run the three GEMVs
        in one launch (weights were packed before any step, so the kernel may
        stream them before the previous kernel in the stream has finished)."""
        bt = self.bt
        M = self.M["decode"]
        ops = nbytes = 0
        for s, (K, N) in enumerate(self.shapes):
            ld = bt.ld_words_for(K)
            ops += 2 * M * N * K
            nbytes += N * ld * 4 + N * (K // self.group) * 4 + M * K * 2 + M * N * 4
        return ("decode_batched_3_projections_M1",
                lambda: bt.bwta_linear_decode_batched(None, flags=bt.GEMM_WEIGHTS_READY,
                                                      descriptors=self.decode_desc),
                ops, nbytes)

    def launches(self):
        """(name, callable, ops, alg_bytes) for every kernel launch of one step, in order."""
        bt = self.bt
        out = [self.decode_launch()]
        for phase in ("prefill",):
            for s, (K, N) in enumerate(self.shapes):
                M = self.M[phase]
                X, (m, sg, sc, a8), Y = self.X[phase][s], self.planes[phase][s], self.Y[phase][s]
                wb, ws = self.w[s]
                ld = m.shape[1]
                G = K // self.group
                if phase == "prefill" and self.prefill_path == "tc":
                    out.append((f"quantize_pack_e4m3_{phase}_{K}x{N}",
                                lambda X=X, o=(None, None, a8, sc):
                                bt.bwta_quantize_pack_acts_ex(X, planes=False, out=o),
                                0, M * K * 2 + M * 32 * ld + M * 4))
                    out.append((f"gemm_tc_{K}x{N}_M{M}",
                                lambda a8=a8, sc=sc, wb=wb, ws=ws, K=K, Y=Y:
                                bt.bwta_gemm_tc(a8, sc, wb, ws, K, self.group, out=(Y, None)),
                                2 * M * N * K, N * ld * 4 + N * G * 4 + M * 32 * ld + M * 4 + M * N * 4))
                    continue
                qa_bytes = M * K * 2 + 2 * M * ld * 4 + M * 4
                out.append((f"quantize_pack_{phase}_{K}x{N}",
                            lambda X=X, o=(m, sg, sc): bt.bwta_quantize_pack_acts(X, out=o),
                            0, qa_bytes))
                gm_bytes = N * ld * 4 + N * G * 4 + 2 * M * ld * 4 + M * 4 + M * N * 4
                # the weights are packed once, before any step: the decode GEMV may
                # prefetch them before waiting for the activation pack it follows
                flags = bt.GEMM_WEIGHTS_READY if phase == "decode" else 0
                out.append((f"{'gemv' if phase == 'decode' else 'gemm'}_{K}x{N}_M{M}",
                            lambda m=m, sg=sg, sc=sc, wb=wb, ws=ws, K=K, Y=Y, flags=flags:
                            bt.bwta_gemm(m, sg, sc, wb, ws, K, self.group, out=(Y, None),
                                         flags=flags),
                            2 * M * N * K, gm_bytes))
        return out

    def popc_launches(self):
        """The prefill products on the LOP3+POPC path (bit planes + k_gemm_tiled),
        timed beside the step so that the popcount kernel's roofline is recorded
        in every bench line."""
        bt = self.bt
        out = []
        M = self.M["prefill"]
        for s, (K, N) in enumerate(self.shapes):
            X, (m, sg, sc, _), Y = self.X["prefill"][s], self.planes["prefill"][s], self.Y["prefill"][s]
            wb, ws = self.w[s]
            ld = m.shape[1]
            G = K // self.group
            out.append((f"quantize_pack_planes_prefill_{K}x{N}",
                        lambda X=X, o=(m, sg, sc): bt.bwta_quantize_pack_acts(X, out=o),
                        0, M * K * 2 + 2 * M * ld * 4 + M * 4))
            out.append((f"gemm_popc_{K}x{N}_M{M}",
                        lambda m=m, sg=sg, sc=sc, wb=wb, ws=ws, K=K, Y=Y:
                        bt.bwta_gemm(m, sg, sc, wb, ws, K, self.group, out=(Y, None)),
                        2 * M * N * K, N * ld * 4 + N * G * 4 + 2 * M * ld * 4 + M * 4 + M * N * 4))
        return out

    def ops(self):
        return sum(op for _, _, op, _ in self.launches())

    def run(self):
        for _, fn, _, _ in self.launches():
            fn()

    def h2d_bytes(self):
        return sum(x.numel() * x.element_size() for p in self.X_host for x in self.X_host[p])

    def d2h_bytes(self):
        return sum(y.numel() * y.element_size() for p in self.Y_host for y in self.Y_host[p])

    def run_e2e(self):
        """Host fp16 activations in, host fp32 outputs out, through the public API.
        The decode phase (three rows up, one launch, three outputs down) and then
        each prefill shape (upload, pack + GEMM, download) run on three streams,
        ordered by events, so the two copy directions overlap each other and the
        kernels of the neighbouring shapes. The step starts after, and ends
        before, everything on the calling stream."""
        comp = torch.cuda.current_stream()
        n = 1 + len(self.shapes)
        if getattr(self, "_up", None) is None:
            self._up, self._down = torch.cuda.Stream(), torch.cuda.Stream()
            self._ev_in = [torch.cuda.Event() for _ in range(n)]
            self._ev_out = [torch.cuda.Event() for _ in range(n)]
        self._up.wait_stream(comp)      # device inputs are free again
        self._down.wait_stream(comp)
        launches = self.launches()
        # unit 0: the decode phase; units 1..3: the prefill shapes
        units = [([("decode", s) for s in range(len(self.shapes))], [launches[0]])]
        for s in range(len(self.shapes)):
            units.append(([("prefill", s)], launches[1 + 2 * s:3 + 2 * s]))
        for i, (tensors, kernels) in enumerate(units):
            with torch.cuda.stream(self._up):
                for p, s in tensors:
                    self.X[p][s].copy_(self.X_host[p][s], non_blocking=True)
                self._ev_in[i].record(self._up)
            comp.wait_event(self._ev_in[i])
            for k in kernels:
                k[1]()
            self._ev_out[i].record(comp)
            with torch.cuda.stream(self._down):
                self._down.wait_event(self._ev_out[i])
                for p, s in tensors:
                    self.Y_host[p][s].copy_(self.Y[p][s], non_blocking=True)
        comp.wait_stream(self._down)    # the step ends when the last output is on the host


def capture_graph(fn):
    """CUDA graph of fn (run once eagerly first so one-time setup stays outside)."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    return g


def time_steps(step_fn, steps, warmup, flush):
    """Per-step device time (s) with CUDA events, L2 flushed before each step."""
    for _ in range(warmup):
        flush()
        step_fn()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    total = 0.0
    per = []
    for _ in range(steps):
        flush()
        gpu_head_start()
        a, b = event_pair()
        a.record()
        step_fn()
        b.record()
        b.synchronize()
        dt = a.elapsed_time(b) * 1e-3
        per.append(dt)
        total += dt
    torch.cuda.synchronize()
    barrier()
    return total, per


def per_kernel_times(step, reps, flush, launches=None):
    """Average device time of every launch of a step, each bracketed by events
    on the launching stream (eager launches, L2 flushed before each step)."""
    launches = step.launches() if launches is None else launches
    acc = {name: [] for name, _, _, _ in launches}
    for _ in range(reps):
        flush()
        gpu_head_start(1500.0)
        evs = []
        for name, fn, _, _ in launches:
            a, b = event_pair()
            a.record()
            fn()
            b.record()
            evs.append((name, a, b))
        torch.cuda.synchronize()
        for name, a, b in evs:
            acc[name].append(a.elapsed_time(b) * 1e-3)
    meta = {name: (op, by) for name, _, op, by in launches}
    return {name: {"s": statistics.mean(v), "ops": meta[name][0], "bytes": meta[name][1]}
            for name, v in acc.items()}


# ------------------------------------------------------------------ oracle arm
def oracle_sample(rows_per_shape: int = 64):
    """The CPU oracle on a bounded sample of the LLaMA step: `rows_per_shape`
    prefill rows per shape plus every decode row. Returns (ops, seconds, cores).
    Weight binarization is offline on both arms and is not timed."""
    import oracle
    oracle.build()
    prepared = []
    for s, (K, N) in enumerate(workloads.LLAMA_SHAPES):
        W = workloads.llama_weights(s)
        b, alpha = oracle.binarize_weights(W, workloads.LLAMA_GROUP)
        Xp = workloads.llama_acts(s, 2048)[:rows_per_shape]
        Xd = workloads.llama_acts(s, 1)
        prepared.append((b, alpha, Xp, Xd, K, N))
    ops = 0
    t0 = time.perf_counter()
    for b, alpha, Xp, Xd, K, N in prepared:
        for X in (Xd, Xp):
            a, sc = oracle.quantize_acts(X)
            d = oracle.int_dots(a, b, workloads.LLAMA_GROUP)
            oracle.linear_out(d, alpha, sc)
            ops += 2 * X.shape[0] * N * K
    dt = time.perf_counter() - t0
    return ops, dt, oracle.num_threads()


# ------------------------------------------------------------------ main arms
def run_ours(args):
    world, rank, local = dist_init("nccl")
    torch.cuda.set_device(local)
    import binarized_transformer_b200 as bt
    from binarized_transformer_b200 import microbench as mb
    bt.load_library()
    flush = L2Flusher()

    step = LlamaStep(rank, prefill_path=args.prefill)
    ops_step = step.ops()
    n_launch_step = len(step.launches())

    graph = capture_graph(step.run)
    with ClockSampler(local) as clk:
        total, per = time_steps(graph.replay, args.steps, args.warmup, flush)
    tmax = max_over_ranks(total, device="cuda")
    value = weak_scaling_value(ops_step, args.steps, world, tmax) / 1e12

    # end to end through the public API with host buffers (copies timed)
    e2e_total, _ = time_steps(step.run_e2e, max(1, args.steps), 1, flush)
    e2e_max = max_over_ranks(e2e_total, device="cuda")
    e2e_value = weak_scaling_value(ops_step, max(1, args.steps), world, e2e_max) / 1e12

    kern = per_kernel_times(step, max(3, args.steps), flush)
    # the popcount GEMMs, each timed alone (flush, GPU head start, events): the
    # bit planes they read are packed once first
    kern_popc = {}
    for name, fn, ops, nbytes in step.popc_launches():
        if name.startswith("gemm_popc"):
            kern_popc[name] = {"s": _time_fn(fn, max(3, args.steps), flush), "ops": ops,
                               "bytes": nbytes}
        else:
            fn()

    if rank != 0:
        barrier()
        return
    peaks, peak_src = measured_peaks()
    # word-ops / s of the tiled kernel's own inner mix (per 4-word chunk: 6 LOP3,
    # 3 POPC, adds); one word-op = 32 MACs = 64 ops
    popc_peak_tops = mb.rate("popc4") * 64 / 1e12
    gemms = {k: v for k, v in kern.items() if k.startswith("gemm_")}
    g_ops = sum(v["ops"] for v in gemms.values())
    g_s = sum(v["s"] for v in gemms.values())
    achieved = g_ops / g_s / 1e12
    hbm = peaks.get("hbm_gbs", FALLBACK_HBM_GBS)
    # fp8 dense tensor peak = the measured bf16 dense GEMM rate x 2 (the nominal
    # fp8 : bf16 ratio); the burst figure, as each GEMM launch is sub-millisecond
    fp8_peak = 2.0 * peaks.get("bf16_tflops", 1590.0)
    fp8_src = ("2 x measured bf16 burst (MEASURED_PEAKS.json)" if "bf16_tflops" in peaks
               else "2 x fallback bf16 1590 TFLOP/s")
    kernels = {}
    popc_gemms = {k: v for k, v in kern_popc.items() if k.startswith("gemm_popc")}
    p_ops = sum(v["ops"] for v in popc_gemms.values())
    p_s = sum(v["s"] for v in popc_gemms.values())
    for name, v in list(kern.items()) + list(kern_popc.items()):
        e = {"us": round(v["s"] * 1e6, 3), "alg_bytes": v["bytes"],
             "gbs": round(v["bytes"] / v["s"] / 1e9, 1)}
        if v["ops"]:
            e["tops"] = round(v["ops"] / v["s"] / 1e12, 2)
        if name.startswith("gemm_tc"):
            e["frac_of_fp8_tensor_peak"] = round(v["ops"] / v["s"] / 1e12 / fp8_peak, 4)
        elif name.startswith("gemm_"):
            e["frac_of_popc_roofline"] = round(v["ops"] / v["s"] / 1e12 / popc_peak_tops, 4)
        else:
            e["frac_of_hbm"] = round(v["bytes"] / v["s"] / 1e9 / hbm, 4)
        kernels[name] = e
    cpu_ops, cpu_s, cores = oracle_sample(args.cpu_rows)
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tmax / args.steps * 1e3, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3-f32" if step.prefill_path == "tc" else "u32", "data": "synthetic",
        "config": {"workload": "llama7b_projections", "shapes_KxN": [list(s) for s in step.shapes],
                   "M_prefill": step.M["prefill"], "M_decode": step.M["decode"],
                   "group": step.group, "acts": "student-t(3), 1% x20 outliers, ternarized",
                   "l2": "flushed before every step (256 MiB write, then 256 MiB read)",
                   "parallelism": f"dp{world}" if world > 1 else "single"},
        "roofline": ({"bound": "tensor", "kernel": "k_gemm_tc (prefill, 3 shapes)",
                      "achieved": round(achieved, 3), "peak": round(fp8_peak, 1),
                      "unit": "TFLOP/s", "frac": round(achieved / fp8_peak, 4),
                      "peak_source": fp8_src, "traffic": tc_traffic(),
                      "traffic_note": "DRAM bytes per k_gemm_tc launch, mean of the 3 shapes (ncu)",
                      "popc_path_ceiling_tops": round(popc_peak_tops, 1)}
                     if step.prefill_path == "tc" else
                     {"bound": "alu", "kernel": "k_gemm_tiled (prefill, 3 shapes)",
                      "achieved": round(achieved, 3), "peak": round(popc_peak_tops, 3),
                      "unit": "TOPS", "frac": round(achieved / popc_peak_tops, 4),
                      "peak_source": "microbenchmarked rate of the kernel's inner mix per 4-word "
                                     "chunk (4+2 LOP3, 3 POPC, adds) x 64 ops per word",
                      "traffic": None}),
        "popc_roofline": {"bound": "alu", "kernel": "k_gemm_tiled (prefill, 3 shapes, timed beside the step)",
                          "achieved": round(p_ops / p_s / 1e12, 3), "peak": round(popc_peak_tops, 3),
                          "unit": "TOPS", "frac": round(p_ops / p_s / 1e12 / popc_peak_tops, 4),
                          "peak_source": "microbenchmarked rate of the kernel's inner mix per 4-word "
                                         "chunk (4+2 LOP3, 3 POPC, adds) x 64 ops per word"},
        "cpu_baseline": {"value": round(cpu_ops / cpu_s / 1e12, 6), "unit": UNIT, "cores": cores,
                         "kind": "oracle",
                         "sample": f"{args.cpu_rows} prefill rows per shape + the decode row, "
                                   f"3 LLaMA-7B shapes, {cpu_s:.2f} s"},
        "e2e": {"value": round(e2e_value, 3), "unit": UNIT, "h2d_bytes_per_step": step.h2d_bytes(),
                "d2h_bytes_per_step": step.d2h_bytes()},
        "gpu_launches": n_launch_step * args.steps,
        "clocks": clk.summary(),
        "kernels": kernels,
        "hbm_peak_gbs": hbm, "hbm_peak_source": peak_src,
        "step_ms": [round(p * 1e3, 4) for p in per],
    }
    print(json.dumps(line), flush=True)
    barrier()


def run_reference(args):
    world, rank, _ = dist_info()
    if rank != 0:
        return
    for _ in range(args.warmup):
        oracle_sample(max(2, args.cpu_rows // 8))
    ops = secs = 0.0
    cores = 1
    for _ in range(args.steps):
        o, s, cores = oracle_sample(args.cpu_rows)
        ops += o
        secs += s
    value = ops / secs / 1e12
    line = {
        "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(secs / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "i64", "data": "synthetic",
        "impl": "reference",
        "config": {"workload": "llama7b_projections", "group": workloads.LLAMA_GROUP,
                   "sample_rows_per_shape": args.cpu_rows},
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{args.cpu_rows} prefill rows per shape + the decode row per step"},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _time_fn(fn, reps, flush):
    """Mean device time of fn over reps, L2 flushed before each rep."""
    fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        flush()
        gpu_head_start()
        a, b = event_pair()
        a.record()
        fn()
        b.record()
        b.synchronize()
        ts.append(a.elapsed_time(b) * 1e-3)
    return statistics.mean(ts)


def decode_model_row(args, flush, hbm, emit, layers=32):
    """Decode of one token through the linear layers of a 32-layer LLaMA-7B:
    per layer, ternarize+pack the layer input and run the GEMV of the fused
    q/k/v (4096 -> 12288), o (4096 -> 4096), fused gate/up (4096 -> 22016) and
    down (11008 -> 4096) projections, all 128 weight matrices distinct
    (1.01 GB of packed bits and scales, far above L2). Captured in one CUDA
    graph; consecutive kernels overlap their launch through programmatic
    dependent launch. Weights come from a seeded torch generator on the GPU."""
    import binarized_transformer_b200 as bt
    shapes = [(4096, 12288), (4096, 4096), (4096, 22016), (11008, 4096)]
    g = torch.Generator(device="cuda")
    g.manual_seed(1234)
    weights = []
    for _ in range(layers):
        for K, N in shapes:
            W = torch.randn((N, K), generator=g, device="cuda", dtype=torch.float32) * 0.02
            weights.append(bt.bwta_pack_weights(W, 128))
            del W
    xs = {K: torch.from_numpy(workloads.llama_acts(0 if K == 4096 else 2, 1)).cuda()
          for K in (4096, 11008)}
    planes = {K: bt.bwta_quantize_pack_acts(xs[K]) for K in xs}
    outs = {N: torch.empty((1, N), dtype=torch.float32, device="cuda") for _, N in shapes}
    wbytes = sum(wb.numel() * 4 + ws.numel() * 4 for wb, ws in weights)

    def step():
        for li in range(layers):
            for si, (K, N) in enumerate(shapes):
                wb, ws = weights[li * len(shapes) + si]
                m, sg, sc = planes[K]
                bt.bwta_quantize_pack_acts(xs[K], out=(m, sg, sc))
                bt.bwta_gemm(m, sg, sc, wb, ws, K, 128, out=(outs[N], None), flags=ready)

    ready = 0
    graph = capture_graph(step)
    t0 = _time_fn(graph.replay, max(3, args.steps), flush)
    emit("llama7b_decode_32_layers_wait_first", t0, nbytes=wbytes, tokens_per_s=round(1.0 / t0, 1),
         launches=2 * layers * len(shapes), note="linear layers only; GEMV waits before its loads")
    ready = bt.GEMM_WEIGHTS_READY
    graph = capture_graph(step)
    t = _time_fn(graph.replay, max(3, args.steps), flush)
    emit("llama7b_decode_32_layers_weights_ready", t, nbytes=wbytes, tokens_per_s=round(1.0 / t, 1),
         launches=2 * layers * len(shapes), note="linear layers only")

    def fused_step():
        for li in range(layers):
            for si, (K, N) in enumerate(shapes):
                wb, ws = weights[li * len(shapes) + si]
                bt.bwta_linear_decode(xs[K], wb, ws, 128, out=(outs[N], None),
                                      flags=bt.GEMM_WEIGHTS_READY)

    graph = capture_graph(fused_step)
    t = _time_fn(graph.replay, max(3, args.steps), flush)
    emit("llama7b_decode_32_layers", t, nbytes=wbytes, tokens_per_s=round(1.0 / t, 1),
         launches=layers * len(shapes), kernel="k_decode (fused ternarize + GEMV)",
         note="linear layers only")


def run_rows(args):
    """One JSON line per measured row of the other workloads (1 GPU)."""
    import binarized_transformer_b200 as bt
    from binarized_transformer_b200 import microbench as mb
    torch.cuda.set_device(0)
    flush = L2Flusher()
    peaks, _ = measured_peaks()
    hbm = peaks.get("hbm_gbs", FALLBACK_HBM_GBS)
    popc_tops = mb.rate("popc4") * 64 / 1e12
    reps = max(3, args.steps)
    rows = args.workload.split(",")
    if "all" in rows:
        rows = ["tiny", "bert", "llama_decode", "llama_decode_batched", "gemv_big",
                "llama_decode_model", "attn", "billm1", "billm16", "billm512", "pack"]
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()

    def emit(name, t, ops=None, nbytes=None, **extra):
        d = {"row": name, "us": round(t * 1e6, 3)}
        if ops:
            d["tops"] = round(ops / t / 1e12, 3)
            d["frac_of_popc_roofline"] = round(ops / t / 1e12 / popc_tops, 4)
        if nbytes:
            d["alg_bytes"] = nbytes
            d["gbs"] = round(nbytes / t / 1e9, 1)
            d["frac_of_hbm"] = round(nbytes / t / 1e9 / hbm, 4)
        d.update(extra)
        print(json.dumps(d), flush=True)

    def linear_rows(tag, X, W, group):
        M, K = X.shape
        N = W.shape[0]
        wb, ws = bt.bwta_pack_weights(dev(W), group)
        Xd = dev(X)
        m, sg, sc = bt.bwta_quantize_pack_acts(Xd)
        Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
        ld = m.shape[1]
        t = _time_fn(lambda: bt.bwta_quantize_pack_acts(Xd, out=(m, sg, sc)), reps, flush)
        emit(f"{tag}_quantize_pack", t, nbytes=M * K * 2 + 2 * M * ld * 4 + M * 4)
        G = (K // group) if group else 1
        t = _time_fn(lambda: bt.bwta_gemm(m, sg, sc, wb, ws, K, group, out=(Y, None)), reps, flush)
        emit(f"{tag}_gemm", t, ops=2 * M * N * K,
             nbytes=N * ld * 4 + N * G * 4 + 2 * M * ld * 4 + M * 4 + M * N * 4)
        if M > 8:
            _, _, a8, sc8 = bt.bwta_quantize_pack_acts_ex(Xd, planes=False)
            t = _time_fn(lambda: bt.bwta_quantize_pack_acts_ex(Xd, planes=False, out=(None, None, a8, sc8)),
                         reps, flush)
            emit(f"{tag}_quantize_pack_e4m3", t, nbytes=M * K * 2 + a8.numel() + M * 4)
            t = _time_fn(lambda: bt.bwta_gemm_tc(a8, sc8, wb, ws, K, group, out=(Y, None)), reps, flush)
            emit(f"{tag}_gemm_tc", t, ops=2 * M * N * K,
                 nbytes=N * ld * 4 + N * G * 4 + a8.numel() + M * 4 + M * N * 4,
                 frac_of_fp8_tensor_peak=round(2 * M * N * K / t / 1e12 / (2.0 * peaks.get("bf16_tflops", 1590.0)), 4))

    for row in rows:
        if row in ("llama_prefill", "llama_decode"):
            M = 2048 if row == "llama_prefill" else 1
            for s in range(3):
                t = workloads.llama(s, M)
                linear_rows(f"llama{s}_{t['K']}x{t['N']}_M{M}", t["X"], t["W"], t["group"])
        elif row == "llama_decode_batched":
            jobs, nbytes, ops = [], 0, 0
            for i in range(3):
                t = workloads.llama(i, 1)
                wb, ws = bt.bwta_pack_weights(dev(t["W"]), t["group"])
                jobs.append((dev(t["X"]), wb, ws, t["group"]))
                nbytes += wb.numel() * 4 + ws.numel() * 4 + t["K"] * 2 + t["N"] * 4
                ops += 2 * t["N"] * t["K"]
            desc = bt.decode_jobs(jobs)
            t = _time_fn(lambda: bt.bwta_linear_decode_batched(
                None, flags=bt.GEMM_WEIGHTS_READY, descriptors=desc), reps, flush)
            emit("llama_decode_3_projections_one_launch", t, ops=ops, nbytes=nbytes,
                 kernel="k_decode (fused ternarize + GEMV, 3 jobs)")
        elif row == "gemv_big":
            W = workloads.billm_weights()  # 28672 x 8192 latent weights, per-128 scales
            X = workloads.billm_acts(1)
            linear_rows("gemv_28672x8192_M1", X, W, 128)
        elif row == "llama_decode_model":
            decode_model_row(args, flush, hbm, emit)
        elif row == "tiny":
            t = workloads.tiny()
            linear_rows("tiny", t["X"], t["W"], 0)
        elif row == "bert":
            for s in (0, 1):
                t = workloads.bert(s)
                linear_rows(f"bert{s}_{t['K']}x{t['N']}", t["X"], t["W"], 0)
        elif row == "attn":
            a = workloads.attn()
            B, H, L, D = workloads.ATTN_SHAPE
            Q, Kt = dev(a["Q"].reshape(-1, D)), dev(a["K"].reshape(-1, D))
            qm, qs, qsc = bt.bwta_quantize_pack_acts(Q)
            km, ks, ksc = bt.bwta_quantize_pack_acts(Kt)
            # past the scores: ternary probabilities straight from the planes, then A . V
            BH = B * H
            pm, ps, psc = bt.bwta_attn_softmax_ternarize(qm, qs, qsc, km, ks, ksc, BH, L, L, D,
                                                         1.0 / np.sqrt(D))
            t = _time_fn(lambda: bt.bwta_attn_softmax_ternarize(
                qm, qs, qsc, km, ks, ksc, BH, L, L, D, 1.0 / np.sqrt(D), out=(pm, ps, psc)),
                reps, flush)
            emit("attn_softmax_ternarize", t,
                 nbytes=2 * (qm.numel() + km.numel()) * 4 + (qsc.numel() + ksc.numel()) * 4 +
                 2 * pm.numel() * 4 + psc.numel() * 4,
                 scores_per_s=round(BH * L * L / t / 1e9, 2), unit_note="G scores/s (fp64 softmax)")
            V = workloads.attn_v()
            Vt = dev(np.ascontiguousarray(V.reshape(BH, L, D).transpose(0, 2, 1)).reshape(-1, L))
            vm, vs, vsc = bt.bwta_quantize_pack_acts(Vt)
            O = torch.empty((BH, L, D), dtype=torch.float32, device="cuda")
            t = _time_fn(lambda: bt.bwta_attn_av(pm, ps, psc, vm, vs, vsc, BH, L, D, L,
                                                 out=(None, O)), reps, flush)
            emit("attn_av", t, ops=2 * BH * L * L * D,
                 nbytes=2 * (pm.numel() + vm.numel()) * 4 + (psc.numel() + vsc.numel()) * 4 +
                 O.numel() * 4)
            t = _time_fn(lambda: bt.bwta_quantize_pack_acts(Q, out=(qm, qs, qsc)), reps, flush)
            emit("attn_quantize_pack_q", t, nbytes=Q.numel() * 2 + 2 * qm.numel() * 4 + qsc.numel() * 4)
            Si = torch.empty((B * H, L, L), dtype=torch.int32, device="cuda")
            Sf = torch.empty((B * H, L, L), dtype=torch.float32, device="cuda")
            inb = 2 * (qm.numel() + km.numel()) * 4 + (qsc.numel() + ksc.numel()) * 4
            for wi, wf, tag in ((True, True, "both"), (False, True, "f32"), (True, False, "i32")):
                fn = lambda wi=wi, wf=wf: bt.bwta_attn_scores(
                    qm, qs, qsc, km, ks, ksc, B * H, L, L, D, want_int=wi, want_float=wf,
                    out=(Si if wi else None, Sf if wf else None))
                t = _time_fn(fn, reps, flush)
                emit(f"attn_scores_{tag}", t, nbytes=inb + Si.numel() * 4 * (int(wi) + int(wf)),
                     outputs=tag)
        elif row.startswith("billm"):
            M = int(row[5:])
            if not hasattr(run_rows, "_billm"):
                run_rows._billm = bt.billm_pack_weights(dev(workloads.billm_weights()))
            Wq = run_rows._billm
            X = dev(workloads.billm_acts(M))
            Y = torch.empty((M, Wq.N), dtype=torch.float32, device="cuda")
            t = _time_fn(lambda: bt.billm_gemm(X, Wq, out=Y), reps, flush)
            wbytes = sum(x.numel() * x.element_size() for x in (Wq.sign, Wq.gmap, Wq.res, Wq.bscale))
            emit(f"billm_gemm_M{M}", t, nbytes=wbytes + X.numel() * 2 + Y.numel() * 4,
                 gflops=round(2 * M * Wq.N * Wq.K / t / 1e9, 1))
        elif row == "pack":
            for s, (K, N) in enumerate(workloads.LLAMA_SHAPES):
                W = dev(workloads.llama_weights(s))
                t = _time_fn(lambda: bt.bwta_pack_weights(W, 128), reps, flush)
                emit(f"pack_weights_{K}x{N}", t, nbytes=W.numel() * 4 + W.numel() // 8 + W.numel() // 32)
            W = dev(workloads.billm_weights())
            t = _time_fn(lambda: bt.billm_pack_weights(W), 1, flush)
            emit("billm_pack_weights", t, nbytes=W.numel() * 4, split="0.5*max")
            t = _time_fn(lambda: bt.billm_pack_weights(W, split=2), 1, flush)
            emit("billm_pack_weights_searched_split", t, nbytes=W.numel() * 4, split="searched")
        else:
            raise SystemExit(f"unknown workload row {row}")


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama")
    ap.add_argument("--cpu-rows", type=int, default=64)
    ap.add_argument("--prefill", default="tc", choices=["tc", "popc"],
                    help="prefill GEMM: tensor cores (default) or the LOP3+POPC kernel")
    args = ap.parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.workload != "llama":
        return run_rows(args)
    return run_ours(args)


if __name__ == "__main__":
    main()
