#!/usr/bin/env python
"""Benchmark of the exact, IO-aware attention forward on B200.

One step = one attention forward (the whole hot path: one kernel launch) over
the patch self-attention 3 MP workload, B=1, H=16, N=11616, d=64, non-causal,
bf16 Q/K/V/O and fp32 LSE, inputs resident in HBM.  L2 is flushed (a 256 MiB
write) before every timed step; each step is timed with CUDA events on the
stream the kernel is launched on.  Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

With N > 1 (launched by torch.distributed.run) every rank runs its own
replica of the workload on its own GPU (the path has no exchange step):
value = FLOPs of all ranks / the slowest rank's time, scaling "weak".
``--impl reference`` times the fp64 CPU oracle instead, on a bounded sample
of the same workload.  ``--pass backward`` times the backward by
recomputation (attn_bwd: dQ, dK, dV from Q, K, V, O, LSE and a seeded dO) on
the same workload instead of the forward; it is a secondary line, not the
headline metric.  ``--sweep`` prints one line per patch count of the pages'
image sweep (N = 1944, 3952, 7776, 11616, 38400; B=1, H=16, d=64): TFLOP/s
and the call's peak extra device bytes next to one materialised H x N x N
bf16 score table.  ``--pad-sweep`` times the 3 MP shape against the fraction
of trailing keys that are padded (padded key tiles are skipped).
"""
import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attn fwd TFLOP/s (% bf16 TC peak) at H16 N11616 d64; peak extra HBM bytes"
WORKLOAD = {"name": "patch self-attention 3 MP", "B": 1, "H": 16, "N": 11616, "d": 64, "causal": False}
# the other workloads of the pages (--config); the default line is WORKLOAD
CONFIGS = {
    "headline": WORKLOAD,
    "tiny": {"name": "tiny exact attention", "B": 1, "H": 2, "N": 128, "d": 64, "causal": False},
    "half_mp": {"name": "patch self-attention 0.5 MP", "B": 1, "H": 16, "N": 1944, "d": 64, "causal": False},
    "eight_mp": {"name": "patch self-attention 8 MP", "B": 1, "H": 16, "N": 38400, "d": 64, "causal": False},
    "causal_decoder": {"name": "causal decoder", "B": 8, "H": 12, "N": 1024, "d": 64, "causal": True},
    "causal_d128": {"name": "causal decoder d=128", "B": 1, "H": 16, "N": 16384, "d": 128, "causal": True},
}
DATASHEET_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
E2E_CHUNKS = 8  # head chunks of the end-to-end path (copies overlap the kernel)
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "attn_fwd_d64_h16_n11616.md")
KERNEL_SOURCES = [os.path.join(ROOT, "exact_io_aware_102_b200", "csrc", f) for f in ("attn_fwd.cu", "sm100_ptx.cuh")]


# ----------------------------------------------------------------- arithmetic
def attn_flops(B, H, N, d, causal):
    """4*B*H*N^2*d (two N x N x d products), halved with a causal mask."""
    f = 4.0 * B * H * N * N * d
    return f / 2 if causal else f


def materialised_bytes(H, N, elem_bytes):
    """One materialised H x N x N score table, H * N^2 * b bytes."""
    return H * N * N * elem_bytes


def algorithmic_bytes(B, H, N, d):
    """Q, K, V read once, O written once (bf16), LSE written (fp32)."""
    return B * H * N * (8 * d + 4)


def output_bytes(B, H, N, d):
    return B * H * N * d * 2 + B * H * N * 4


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "hbm_gbs": float(p["hbm_gbs"]), "source": "measured"}
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS, source="fallback")


def _code_only(text):
    """C++ source with comments removed and whitespace collapsed."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def source_digest():
    """Digest of the forward kernel's code (the kernel file and its PTX helper
    header, comments and whitespace excluded): a comment edit keeps the
    profiled DRAM traffic valid, any code change does not."""
    h = hashlib.sha256()
    for path in KERNEL_SOURCES:
        with open(path) as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source (else None)."""
    try:
        text = open(PROFILE_SUMMARY).read()
    except OSError:
        return None
    vals = {}
    for line in text.splitlines():
        if ":" in line and line.strip().startswith("- "):
            k, v = line.strip()[2:].split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    if vals.get("kernel_source_sha256_16") != source_digest():
        return None
    try:
        return int(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# A spin on the device, queued right before a timed loop, while which the
# host enqueues the first steps: a host stall (interpreter, the clock-sampling
# thread) then finds the device still busy instead of leaving it idle between
# a step's start event and its launch, where the stall would count as that
# step's time.  It runs before the first step's start event (~2 ms).
HOST_LEAD_CYCLES = 4_000_000


def host_lead():
    import torch
    torch.cuda._sleep(HOST_LEAD_CYCLES)


def reduce_max(value, dist=None, device=None):
    """Max of a float over all ranks (identity on one process)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------- clock sampling
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device, period_s=0.005):
        self.device, self.period, self.samples, self.reasons = device, period_s, [], set()
        self._stop = threading.Event()
        self._thread = None
        self.max_mhz = None
        self.error = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = self._handle(pynvml)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        except Exception as e:  # no NVML: report no clocks rather than guess
            self.error = repr(e)
        return self

    def _handle(self, nv):
        # match the CUDA device by UUID (CUDA_VISIBLE_DEVICES may renumber devices)
        import torch
        try:
            uuid = str(torch.cuda.get_device_properties(self.device).uuid)
            return nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.device.index or 0)

    def _run(self):
        nv = self._nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                bits = get_reasons(self._h)
                for b, name in self.REASONS.items():
                    if bits & b:
                        self.reasons.add(name)
            except Exception as e:
                self.error = repr(e)
                return
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()
        return False

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0, "error": self.error}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ---------------------------------------------------------------- CPU oracle
def time_oracle(q, k, v, scale, causal, budget_s, max_rows=None):
    """Time the fp64 oracle on a seeded row sample grown until one run takes
    at least half of budget_s (or covers every row)."""
    import oracle
    from exact_io_aware_102_b200.inputs import sample_rows
    B, H, N, d = (int(x) for x in q.shape)
    cap = min(N, max_rows) if max_rows else N
    rows = min(8, cap)
    while True:
        idx = sample_rows(B, H, N, rows).numpy()
        t0 = time.perf_counter()
        oracle.attention_rows(q, k, v, scale, causal, rows=idx)
        secs = time.perf_counter() - t0
        if secs >= 0.5 * budget_s or rows >= cap:
            break
        rows = min(cap, int(rows * min(64.0, max(2.0, budget_s / max(secs, 1e-3)))))
    # each evaluated row costs 4*visible*d FLOP (scores + weighted sum)
    if causal:
        flop = float(sum(4.0 * (int(i) + 1) * d for i in idx.reshape(-1)))
    else:
        flop = 4.0 * idx.size * N * d
    return {"seconds": secs, "flop": flop, "rows_per_head": int(idx.shape[1]), "heads": int(idx.shape[0]),
            "cores": oracle.max_threads()}


# -------------------------------------------------------------------- arms
def workload(args):
    return CONFIGS[args.config]


def metric_name(W, what="fwd"):
    if W is WORKLOAD and what == "fwd":
        return METRIC
    return "attn %s TFLOP/s at B%d H%d N%d d%d%s" % (what, W["B"], W["H"], W["N"], W["d"],
                                                     " causal" if W["causal"] else "")


def run_cuda(args, rank, world, dist):
    import torch
    import exact_io_aware_102_b200 as pkg
    from exact_io_aware_102_b200.inputs import make_qkv

    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    W = workload(args)
    B, H, N, d, causal = W["B"], W["H"], W["N"], W["d"], W["causal"]
    scale = 1.0 / math.sqrt(d)
    q_cpu, k_cpu, v_cpu = make_qkv(B, H, N, d, seed=0)
    q, k, v = (x.to(dev) for x in (q_cpu, k_cpu, v_cpu))
    flops = attn_flops(B, H, N, d, causal)
    stream = torch.cuda.current_stream()

    # peak extra device memory of one call (allocator method of the pages)
    pkg.forward(q, k, v, scale=scale, causal=causal)  # loads the module image
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    base = torch.cuda.memory_allocated()
    torch.cuda.reset_peak_memory_stats()
    o, lse = pkg.forward(q, k, v, scale=scale, causal=causal)
    torch.cuda.synchronize()
    extra = torch.cuda.max_memory_allocated() - base
    free1 = torch.cuda.mem_get_info()[0]
    st = pkg.attn_check_device_status()
    if st != pkg.ATTN_OK:
        raise RuntimeError("device status: " + pkg.attn_status_string(st))

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]

    for _ in range(args.warmup):
        flush.zero_()
        pkg.forward(q, k, v, scale=scale, causal=causal, out=o, lse=lse)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev) as clocks:
        host_lead()
        for i in range(args.steps):
            flush.zero_()
            ev[i][0].record(stream)
            pkg.forward(q, k, v, scale=scale, causal=causal, out=o, lse=lse)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    st = pkg.attn_check_device_status()
    if st != pkg.ATTN_OK:
        raise RuntimeError("device status: " + pkg.attn_status_string(st))
    step_ms = [a.elapsed_time(b) for a, b in ev]
    ms_local = sum(step_ms) / len(step_ms)
    ms = reduce_max(ms_local, dist, dev)
    value = flops * world / (ms * 1e-3) / 1e12

    peaks = load_peaks()
    achieved = flops / (ms_local * 1e-3) / 1e12
    roofline = {"bound": "tensor", "achieved": round(achieved, 2), "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4),
                "traffic": profiled_traffic() if W is WORKLOAD else None,
                "peak_kind": "burst bf16 dense, %s" % peaks["source"],
                "algorithmic_bytes": algorithmic_bytes(B, H, N, d),
                "frac_of_datasheet_2250": round(achieved / DATASHEET_BF16_TFLOPS, 4)}

    # host time of one call of the 12-argument C entry point (argument checks,
    # tensor-map lookup, launch; the kernel runs asynchronously): median over
    # calls issued back to back, next to the kernel's own time
    host_us = None
    if not args.no_host_time:
        sh = torch.cuda.current_stream().cuda_stream
        ptrs = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr())
        n_calls = 200 if ms_local < 0.5 else 50
        times = []
        for _ in range(n_calls):
            t0 = time.perf_counter()
            st = pkg.attn_fwd(*ptrs, B, H, N, d, scale, causal, sh)
            times.append(time.perf_counter() - t0)
            if st != pkg.ATTN_OK:
                raise RuntimeError("attn_fwd: " + pkg.attn_status_string(st))
        torch.cuda.synchronize()
        host_us = round(statistics.median(times) * 1e6, 2)

    # end to end through the public call: pinned host inputs -> device -> attention -> host outputs
    e2e = None
    if not args.no_e2e:
        qh, kh, vh = (x.pin_memory() for x in (q_cpu, k_cpu, v_cpu))
        oh = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        lh = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        qd, kd, vd = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        e2e_steps = max(3, min(args.steps, 50))

        workspace = (qd, kd, vd, o, lse)

        def e2e_step():
            # host inputs -> device -> attention -> host outputs, in head chunks
            # whose transfers overlap the kernel (forward_host)
            pkg.forward_host(qh, kh, vh, scale=scale, causal=causal, chunks=E2E_CHUNKS, out=oh, lse=lh,
                             workspace=workspace)

        for _ in range(max(3, args.warmup)):
            e2e_step()
        eev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(e2e_steps)]
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        host_lead()
        for i in range(e2e_steps):
            flush.zero_()
            eev[i][0].record(stream)
            e2e_step()
            eev[i][1].record(stream)
        torch.cuda.synchronize()
        e_ms = reduce_max(sum(a.elapsed_time(b) for a, b in eev) / e2e_steps, dist, dev)
        h2d = 3 * q.numel() * q.element_size()
        d2h = o.numel() * o.element_size() + lse.numel() * lse.element_size()
        e2e = {"value": round(flops * world / (e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
               "ms_per_step": round(e_ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "path": "forward_host: pinned host Q/K/V -> device -> attn_fwd -> pinned host O/LSE, "
                       "%d head chunks with copies overlapping the kernel" % E2E_CHUNKS}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r = time_oracle(q_cpu, k_cpu, v_cpu, scale, causal, budget_s=args.cpu_budget)
        cpu = {"value": r["flop"] / r["seconds"] / 1e12, "unit": "TFLOP/s", "cores": r["cores"],
               "kind": "oracle",
               "sample": "%d of %d query rows per head x %d heads of the same workload (seeded), "
                         "fp64 C oracle, %.1f s; 4*N*d FLOP per row" % (r["rows_per_head"], N, r["heads"],
                                                                        r["seconds"])}

    line = {
        "metric": metric_name(W), "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic: iid N(0,1) rounded to bf16, seed 0",
        "config": {"workload": "%s: B=%d H=%d N=%d d=%d %s, bf16 Q/K/V/O, fp32 LSE" % (
            W["name"], B, H, N, d, "causal" if causal else "non-causal"),
            "B": B, "H": H, "N": N, "d": d, "causal": causal, "scale": scale,
            "l2": "flushed before every timed step (256 MiB write, untimed)",
            "parallelism": "replicas" if world > 1 else "single GPU"},
        "pct_of_peak": round(100 * achieved / peaks["bf16_tflops"], 2),
        "peak_extra_bytes": {"measured": int(extra), "cap_1p1x_o_lse": int(1.1 * output_bytes(B, H, N, d)),
                             "o_plus_lse": output_bytes(B, H, N, d),
                             "materialised_copy_bf16": materialised_bytes(H, N, 2),
                             "device_free_delta": int(free0 - free1),
                             "method": "memory_allocated base, reset_peak_memory_stats, call, max_memory_allocated - base"},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": args.steps,
        "host_us_per_call": host_us,
        "clocks": clocks.summary(), "step_ms_min": round(min(step_ms), 4), "step_ms_max": round(max(step_ms), 4),
    }
    return line


def bwd_flops(B, H, N, d, causal):
    """10*B*H*N^2*d: five N x N x d products (S recomputed, dP, dV, dK, dQ), halved causal."""
    f = 10.0 * B * H * N * N * d
    return f / 2 if causal else f


def run_cuda_backward(args, rank, world, dist):
    import torch
    import exact_io_aware_102_b200 as pkg
    from exact_io_aware_102_b200.inputs import make_dout, make_qkv

    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    W = workload(args)
    B, H, N, d, causal = W["B"], W["H"], W["N"], W["d"], W["causal"]
    scale = 1.0 / math.sqrt(d)
    q, k, v = (x.to(dev) for x in make_qkv(B, H, N, d, seed=0))
    dout = make_dout(B, H, N, d, seed=1).to(dev)
    o, lse = pkg.forward(q, k, v, scale=scale, causal=causal)
    flops = bwd_flops(B, H, N, d, causal)
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for _ in range(args.warmup):
        flush.zero_()
        pkg.backward(q, k, v, o, lse, dout, scale=scale, causal=causal)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev) as clocks:
        host_lead()
        for i in range(args.steps):
            flush.zero_()
            ev[i][0].record(stream)
            pkg.backward(q, k, v, o, lse, dout, scale=scale, causal=causal)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    st = pkg.attn_check_device_status()
    if st != pkg.ATTN_OK:
        raise RuntimeError("device status: " + pkg.attn_status_string(st))
    step_ms = [a.elapsed_time(b) for a, b in ev]
    ms_local = sum(step_ms) / len(step_ms)
    ms = reduce_max(ms_local, dist, dev)
    peaks = load_peaks()
    achieved = flops / (ms_local * 1e-3) / 1e12
    return {
        "metric": metric_name(W, "bwd") + " (dQ, dK, dV by recomputation)",
        "value": round(flops * world / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: iid N(0,1) rounded to bf16, Q/K/V seed 0, dO seed 1",
        "config": {"workload": "%s backward: B=%d H=%d N=%d d=%d %s, bf16 Q/K/V/O/dO/dK/dV, fp32 LSE/dQ" % (
            W["name"], B, H, N, d, "causal" if causal else "non-causal"),
            "B": B, "H": H, "N": N, "d": d, "causal": causal, "scale": scale,
            "l2": "flushed before every timed step (256 MiB write, untimed)",
            "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4), "traffic": None,
                     "peak_kind": "burst bf16 dense, %s" % peaks["source"]},
        "cpu_baseline": None, "e2e": None, "gpu_launches": 2 * args.steps,
        "clocks": clocks.summary(), "step_ms_min": round(min(step_ms), 4), "step_ms_max": round(max(step_ms), 4),
    }


def run_sweep(args):
    """TFLOP/s and peak extra device bytes over the image sweep (one JSON line each)."""
    import torch
    import exact_io_aware_102_b200 as pkg
    from exact_io_aware_102_b200.inputs import make_qkv
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    peaks = load_peaks()
    lines = []
    for N in (1944, 3952, 7776, 11616, 38400):
        B, H, d = 1, 16, 64
        q, k, v = (x.to(dev) for x in make_qkv(B, H, N, d, seed=0))
        pkg.forward(q, k, v)
        torch.cuda.synchronize()
        base = torch.cuda.memory_allocated()
        torch.cuda.reset_peak_memory_stats()
        o, lse = pkg.forward(q, k, v)
        torch.cuda.synchronize()
        extra = torch.cuda.max_memory_allocated() - base
        steps = max(5, min(args.steps, 50))
        for _ in range(max(3, args.warmup)):
            flush.zero_()
            pkg.forward(q, k, v, out=o, lse=lse)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        torch.cuda.synchronize()
        host_lead()
        for i in range(steps):
            flush.zero_()
            ev[i][0].record()
            pkg.forward(q, k, v, out=o, lse=lse)
            ev[i][1].record()
        torch.cuda.synchronize()
        st = pkg.attn_check_device_status()
        if st != pkg.ATTN_OK:
            raise RuntimeError("device status: " + pkg.attn_status_string(st))
        ms = sum(a.elapsed_time(b) for a, b in ev) / steps
        tf = attn_flops(B, H, N, d, False) / (ms * 1e-3) / 1e12
        lines.append({"sweep": "patch self-attention", "B": B, "H": H, "N": N, "d": d, "causal": False,
                      "tflops": round(tf, 2), "pct_of_peak": round(100 * tf / peaks["bf16_tflops"], 2),
                      "ms": round(ms, 4), "peak_extra_bytes": int(extra),
                      "o_plus_lse_bytes": output_bytes(B, H, N, d),
                      "materialised_copy_bf16": materialised_bytes(H, N, 2)})
        del q, k, v, o, lse
    return lines


def run_pad_sweep(args):
    """Key-padding sweep on the 3 MP shape (B=1, H=16, N=11616, d=64): the last
    f*N keys padded, f in {0, 1/4, 1/2, 3/4}.  Tiles holding only padded keys
    are skipped, so the time should fall with f; TFLOP/s counts the visible
    (query, key) pairs only, 4*H*N*visible*d."""
    import torch
    import exact_io_aware_102_b200 as pkg
    from exact_io_aware_102_b200.inputs import make_qkv
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    B, H, N, d = 1, 16, 11616, 64
    q, k, v = (x.to(dev) for x in make_qkv(B, H, N, d, seed=0))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    lines = []
    for frac in (0.0, 0.25, 0.5, 0.75):
        visible = N - int(round(frac * N))
        pad = torch.zeros((B, N), dtype=torch.bool, device=dev)
        pad[:, visible:] = True
        steps = max(5, min(args.steps, 50))
        for _ in range(max(3, args.warmup)):
            flush.zero_()
            pkg.forward(q, k, v, out=o, lse=lse, key_padding_mask=pad)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        torch.cuda.synchronize()
        host_lead()
        for i in range(steps):
            flush.zero_()
            ev[i][0].record()
            pkg.forward(q, k, v, out=o, lse=lse, key_padding_mask=pad)
            ev[i][1].record()
        torch.cuda.synchronize()
        st = pkg.attn_check_device_status()
        if st != pkg.ATTN_OK:
            raise RuntimeError("device status: " + pkg.attn_status_string(st))
        ms = sum(a.elapsed_time(b) for a, b in ev) / steps
        flop = 4.0 * B * H * N * visible * d
        lines.append({"pad_sweep": "patch self-attention 3 MP, trailing keys padded", "B": B, "H": H, "N": N,
                      "d": d, "padded_fraction": frac, "visible_keys": visible, "ms": round(ms, 4),
                      "tflops_visible": round(flop / (ms * 1e-3) / 1e12, 2)})
    return lines


def run_reference(args, rank, world):
    """The fp64 CPU oracle timed on the host cores, each step a bounded sample."""
    from exact_io_aware_102_b200.inputs import make_qkv
    W = workload(args)
    B, H, N, d, causal = W["B"], W["H"], W["N"], W["d"], W["causal"]
    scale = 1.0 / math.sqrt(d)
    q, k, v = make_qkv(B, H, N, d, seed=0)
    per_step = max(0.5, args.cpu_budget / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        time_oracle(q, k, v, scale, causal, budget_s=per_step)
    secs, flop, rows, cores = 0.0, 0.0, 0, 1
    for _ in range(args.steps):
        r = time_oracle(q, k, v, scale, causal, budget_s=per_step)
        secs += r["seconds"]
        flop += r["flop"]
        rows = r["rows_per_head"]
        cores = r["cores"]
    value = flop / secs / 1e12
    sample = ("%d of %d query rows per head x %d heads per step (seeded), fp64 C oracle" % (rows, N, B * H))
    return {
        "impl": "reference", "metric": metric_name(W), "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * secs / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic: iid N(0,1) rounded to bf16, seed 0",
        "config": {"workload": "%s: B=%d H=%d N=%d d=%d %s, bf16 Q/K/V/O, fp32 LSE" % (
            W["name"], B, H, N, d, "causal" if causal else "non-causal"), "B": B, "H": H, "N": N, "d": d,
            "causal": causal, "scale": scale, "parallelism": "single process (rank 0)"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for the CPU baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-host-time", action="store_true",
                    help="skip timing the host side of one attn_fwd call")
    ap.add_argument("--pass", dest="which", choices=["forward", "backward"], default="forward",
                    help="time the forward (the headline) or the backward")
    ap.add_argument("--sweep", action="store_true", help="TFLOP/s and peak extra bytes over the image sweep")
    ap.add_argument("--pad-sweep", action="store_true",
                    help="time against the fraction of padded keys (3 MP shape, trailing padding)")
    ap.add_argument("--config", choices=sorted(CONFIGS), default="headline",
                    help="workload (default: the headline patch self-attention 3 MP)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.steps < 1:
        ap.error("--steps must be at least 1")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world != args.gpus:
        ap.error("--gpus %d but WORLD_SIZE=%d: launch N>1 with torch.distributed.run" % (args.gpus, world))

    if args.sweep:
        if world != 1:
            ap.error("--sweep runs on one GPU")
        for line in run_sweep(args):
            print(json.dumps(line), flush=True)
        return 0

    if args.pad_sweep:
        if world != 1:
            ap.error("--pad-sweep runs on one GPU")
        for line in run_pad_sweep(args):
            print(json.dumps(line), flush=True)
        return 0

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, rank, world)), flush=True)
        return 0

    dist = None
    if world > 1:
        import datetime
        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        tdist.init_process_group(backend="nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    try:
        line = (run_cuda_backward if args.which == "backward" else run_cuda)(args, rank, world, dist)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
