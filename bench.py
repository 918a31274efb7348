#!/usr/bin/env python
"""Throughput of the fused fp16 GEMM C = GELU_erf(A.B + bias) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload fused_8192]

One step is one pass of the whole path over one batch: a single
``tg_gemm`` call (fp16 A[M,K] @ B[K,N] with fp32 accumulation, bias add,
erf-GELU, fp16 store) on inputs already resident in HBM.  The metric is the
tutorial's TFLOP/s = 2*M*N*K / time (epilogue flops not counted).

Multi-GPU: one process per GPU (torchrun); each rank runs its own replica of
the workload (the GEMM needs no exchange), so per-GPU work is fixed
("weak" scaling) and the job value is the sum over ranks, timed as the max
over ranks.  ``--impl reference`` times the CPU oracle (fp64, OpenMP) on a
bounded sample of the same workload, on rank 0 only.

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import glob
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

METRIC = "fp16 GEMM(+bias+GELU) TFLOP/s at 2048^3 and 8192^3; % of B200 fp16 dense peak"
UNIT = "TFLOP/s"
NOMINAL_FP16_DENSE_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024
EPI_NAMES = {0: "none", 1: "bias", 2: "bias_gelu", 3: "bias_gelu_tanh", 4: "bias_softmax"}


# ---------------------------------------------------------------------------- helpers

GEMM_DEVICE_SOURCES = ("tg_kernels.cuh", "tg_ptx.cuh")


def kernel_source_hash(kernel_config: dict) -> str:
    """Hash of the GEMM kernel's device code and of the configuration it is
    launched with (tile shape, stages, CTA pair, rasterisation panel, work
    division, loader): ncu traffic figures hold only for that pair."""
    h = hashlib.sha256()
    files = [os.path.join(ROOT, "tensor_core_gemm_fp16_b200", "csrc", f) for f in GEMM_DEVICE_SOURCES]
    for f in files:
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode())
            h.update(fh.read())
    h.update(json.dumps(kernel_config, sort_keys=True).encode())
    return h.hexdigest()[:16]


def workload_kernel_hash(name: str, num_sms: int = 148) -> str:
    """kernel_source_hash of the configuration the library picks for a named
    GEMM workload (a host-only query: no GPU needed)."""
    from tensor_core_gemm_fp16_b200 import binding
    from tensor_core_gemm_fp16_b200 import workloads as wl
    w = wl.WORKLOADS[name]
    return kernel_source_hash(binding.tg_gemm_select_config(w.M, w.N, w.K, w.epilogue, num_sms))


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def profiled_traffic(workload: str, kernel_config: dict):
    """DRAM bytes per launch of the GEMM kernel from the committed ncu summary
    for this workload, or None when absent or taken on another kernel (device
    code or launch configuration)."""
    path = os.path.join(ROOT, "profiles", f"gemm_persistent_kernel_{workload}.md")
    try:
        with open(path) as f:
            text = f.read()
    except OSError:
        return None
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    h = re.search(r"source_hash:\s*([0-9a-f]+)", text)
    if not m or not h or h.group(1) != kernel_source_hash(kernel_config):
        return None
    return float(m.group(1))


class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML in a thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, torch, device_index: int, period_s: float = 0.002):
        self.ok = False
        self.samples = []
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            self.ok = True
        except Exception as e:  # no NVML: report it rather than guess
            self.err = f"{type(e).__name__}: {e}"
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0,
                                     int(self._reasons(self.h))))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if not self.ok:
            return {"error": getattr(self, "err", "nvml unavailable")}
        self._stop.set()
        self._t.join()
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mask = 0
        for _, _, r in self.samples:
            mask |= r
        reasons = [name for bit, name in self.REASONS.items() if mask & bit and name != "gpu_idle"]
        return {"sm_mhz": statistics.median(s[0] for s in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "power_w_max": round(max(s[1] for s in self.samples), 1),
                "samples": len(self.samples)}


def max_over_ranks(x: float, world: int, dist=None, device=None) -> float:
    """Maximum of x over all ranks (the job's time is its slowest rank's)."""
    if world <= 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(flops_per_rank: int, world: int, step_ms: float) -> float:
    """Whole-job TFLOP/s: every rank's flops over the slowest rank's step time."""
    return world * flops_per_rank / (step_ms * 1e-3) / 1e12


# ---------------------------------------------------------------------------- oracle timing

def oracle_rows_for(w, a, b, bb, target_s: float):
    """Row count whose oracle call takes at most about target_s: one probe
    call (after a warm one) at 4 rows per thread, scaled linearly.  The
    probe's fixed cost (fp16 decode of B) makes the projection conservative."""
    import oracle
    r0 = min(w.M, 4 * max(1, oracle.num_threads()))
    oracle.gemm(a, b, bb, w.epilogue, rows=list(range(min(r0, 2))))
    t0 = time.perf_counter()
    oracle.gemm(a, b, bb, w.epilogue, rows=list(range(r0)))
    dt = time.perf_counter() - t0
    return max(2, min(w.M, int(r0 * target_s / max(dt, 1e-3))))


def evenly_spaced(M: int, rows: int):
    return sorted(set(int(i * M // rows) for i in range(rows)))


def oracle_sample(w, A, B, bias, target_s: float):
    """Time the oracle (as it stands) on a row sample of workload w sized to
    about target_s seconds.  Returns (tflops, seconds, rows, cores)."""
    import oracle
    from tensor_core_gemm_fp16_b200 import workloads as wl
    a, b, bb = wl.to_bits(A), wl.to_bits(B), wl.to_bits(bias)
    sel = evenly_spaced(w.M, oracle_rows_for(w, a, b, bb, target_s))
    t0 = time.perf_counter()
    oracle.gemm(a, b, bb, w.epilogue, rows=sel)
    dt = time.perf_counter() - t0
    return 2.0 * len(sel) * w.N * w.K / dt / 1e12, dt, len(sel), oracle.num_threads()


def oracle_single_core(target_s: float = 1.0):
    """The oracle on one core for gemm_256 (whole) and gemm_2048 (a row sample
    of about target_s): GFLOP/s of each, as a per-core reference."""
    import oracle
    from tensor_core_gemm_fp16_b200 import workloads as wl
    prev = oracle.set_num_threads(1)
    try:
        out = {}
        for name in ("gemm_256", "gemm_2048"):
            w = wl.WORKLOADS[name]
            A, B, bias = wl.workload_inputs(w)
            a, b, bb = wl.to_bits(A), wl.to_bits(B), wl.to_bits(bias)
            sel = evenly_spaced(w.M, oracle_rows_for(w, a, b, bb, target_s))
            t0 = time.perf_counter()
            oracle.gemm(a, b, bb, w.epilogue, rows=sel)
            dt = time.perf_counter() - t0
            out[name] = {"gflops": 2.0 * len(sel) * w.N * w.K / dt / 1e9,
                         "rows": f"{len(sel)} of {w.M}", "seconds": dt}
        return out
    finally:
        oracle.set_num_threads(prev)


# ---------------------------------------------------------------------------- arms

def run_reference(args, w, rank, world):
    """The CPU oracle on a bounded row sample of the same workload."""
    if rank != 0:
        return 0
    import oracle
    from tensor_core_gemm_fp16_b200 import workloads as wl
    oracle.build()
    A, B, bias = wl.workload_inputs(w)
    # each step: one oracle call on a row sample; about 120 s in total
    per_step = max(1.0, min(8.0, 120.0 / max(1, args.steps + args.warmup)))
    a, b, bb = wl.to_bits(A), wl.to_bits(B), wl.to_bits(bias)
    sel = evenly_spaced(w.M, oracle_rows_for(w, a, b, bb, per_step))
    cores = oracle.num_threads()
    for _ in range(args.warmup):
        oracle.gemm(a, b, bb, w.epilogue, rows=sel)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.gemm(a, b, bb, w.epilogue, rows=sel)
        times.append(time.perf_counter() - t0)
    ms = 1e3 * statistics.mean(times)
    value = 2.0 * len(sel) * w.N * w.K / (ms * 1e-3) / 1e12
    sample = (f"{len(sel)} evenly spaced rows of the {w.M}x{w.N}x{w.K} output per step "
              f"({len(sel) * w.N} outputs, fp64, one oracle call incl. fp16 decode)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, extra=None):
    from tensor_core_gemm_fp16_b200 import workloads as wl  # noqa: F401
    dist = ("A,B,bias ~ N(0,1)" if w.dist == "normal" else "A,B,bias ~ U(-1,1)")
    if w.b_scale != 1.0 or w.a_scale != 1.0:
        dist += f"; A scaled by {w.a_scale:.6g}, B scaled by {w.b_scale:.6g} (1/sqrt(K))"
    cfg = {"workload": w.name, "M": w.M, "N": w.N, "K": w.K, "epilogue": EPI_NAMES[w.epilogue],
           "inputs": f"{dist}, torch CPU generator seed {w.seed}, rounded to fp16",
           "parallelism": "replicas"}
    if extra:
        cfg.update(extra)
    return cfg


def time_workload(torch, binding, w, steps, warmup, dev, stream, flush_buf, config_id=-1):
    """Device-resident inputs; returns dict with per-launch and per-step times."""
    from tensor_core_gemm_fp16_b200 import workloads as wl
    A, B, bias = wl.workload_inputs(w)
    a, b = A.to(dev), B.to(dev)
    bb = bias.to(dev) if bias is not None else None
    c = torch.empty(w.M, w.N, dtype=torch.float16, device=dev)
    args = (a.data_ptr(), b.data_ptr(), bb.data_ptr() if bb is not None else None, c.data_ptr(),
            w.M, w.N, w.K, w.epilogue)
    big = 2 * (w.M * w.K + w.K * w.N + w.M * w.N) > L2_BYTES

    def launch():
        if config_id < 0:
            st = binding.tg_gemm(*args, stream.cuda_stream)
        else:
            st = binding.tg_gemm_ex(*args, config_id=config_id, stream=stream.cuda_stream)
        if st != binding.TG_OK:
            raise binding.TgError(st, "tg_gemm")

    for _ in range(warmup):
        if not big:
            flush_buf.zero_()
        launch()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    return {"A": A, "B": B, "bias": bias, "a": a, "b": b, "bb": bb, "c": c, "args": args,
            "big": big, "launch": launch, "ev": ev, "t_start": t_start, "t_end": t_end}


def time_attention(torch, binding, w, steps, warmup, dev, stream, flush_buf):
    """Device-resident inputs for an attention workload; the same dict shape as
    time_workload (launch closure and per-step events)."""
    from tensor_core_gemm_fp16_b200 import workloads as wl
    Q, K, V = wl.attn_workload_inputs(w)
    q, k, v = Q.to(dev), K.to(dev), V.to(dev)
    o = torch.empty_like(q)
    big = 2 * w.B * w.H * w.D * (2 * w.Sq + 2 * w.Sk) > L2_BYTES

    def launch():
        st = binding.tg_attention_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                      w.B, w.H, w.Sq, w.Sk, w.D, int(w.causal), 0.0,
                                      stream.cuda_stream)
        if st != binding.TG_OK:
            raise binding.TgError(st, "tg_attention_fwd")

    for _ in range(warmup):
        if not big:
            flush_buf.zero_()
        launch()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    return {"q": q, "k": k, "v": v, "o": o, "big": big, "launch": launch, "ev": ev}


def run_ours(args, w, rank, world):
    import torch
    import torch.distributed as dist
    from tensor_core_gemm_fp16_b200 import binding
    from tensor_core_gemm_fp16_b200 import workloads as wl

    binding.load()
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev,
                                timeout=__import__("datetime").timedelta(seconds=120))
    stream = torch.cuda.current_stream(dev)
    flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    def reduce_max(x: float) -> float:
        return max_over_ranks(x, world, dist, dev)

    # ---------------------------------------------------------------- device-resident timing
    s = time_workload(torch, binding, w, args.steps, args.warmup, dev, stream, flush_buf,
                      args.config)
    sampler = ClockSampler(torch, local)
    barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    s["t_start"].record(stream)
    for i in range(args.steps):
        if not s["big"]:
            flush_buf.zero_()           # untimed: outside the per-launch events
        s["ev"][i][0].record(stream)
        s["launch"]()
        s["ev"][i][1].record(stream)
    s["t_end"].record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clocks = sampler.stop()
    launch_ms = [e0.elapsed_time(e1) for e0, e1 in s["ev"]]
    kernel_ms = statistics.mean(launch_ms)
    region_ms = s["t_start"].elapsed_time(s["t_end"])
    step_ms = region_ms / args.steps if s["big"] else sum(launch_ms) / args.steps
    step_ms = reduce_max(step_ms)
    value = job_value(w.flops, world, step_ms)
    launches_per_step = binding.tg_gemm_launch_count(*s["args"])
    st = binding.tg_gemm_check_error(stream.cuda_stream)
    if st != binding.TG_OK:
        raise binding.TgError(st, "device error word after the timed region")

    # ---------------------------------------------------------------- other sizes named by the metric
    also = []
    for name in args.also:
        if name == w.name:
            continue
        if name in wl.ATTN_WORKLOADS:
            w2 = wl.ATTN_WORKLOADS[name]
            s2 = time_attention(torch, binding, w2, args.steps, args.warmup, dev, stream,
                                flush_buf)
        else:
            w2 = wl.WORKLOADS[name]
            s2 = time_workload(torch, binding, w2, args.steps, args.warmup, dev, stream,
                               flush_buf)
        barrier()
        torch.cuda.synchronize(dev)
        for i in range(args.steps):
            if not s2["big"]:
                flush_buf.zero_()
            s2["ev"][i][0].record(stream)
            s2["launch"]()
            s2["ev"][i][1].record(stream)
        torch.cuda.synchronize(dev)
        ms2 = reduce_max(statistics.mean(e0.elapsed_time(e1) for e0, e1 in s2["ev"]))
        entry = {"workload": name, "value": world * w2.flops / (ms2 * 1e-3) / 1e12,
                 "unit": UNIT, "ms_per_step": ms2,
                 "kind": "attention" if name in wl.ATTN_WORKLOADS else "gemm",
                 "gbs": w2.algorithmic_bytes / (ms2 * 1e-3) / 1e9,
                 "pct_of_fp16_dense_peak_nominal":
                     100.0 * w2.flops / (ms2 * 1e-3) / 1e12 / NOMINAL_FP16_DENSE_TFLOPS,
                 "l2": "flushed between launches" if not s2["big"] else "inputs larger than L2"}
        if not s2["big"]:
            # Hot L2: the same launches back to back with no flush, so the
            # operands of each launch are still in L2 from the previous one.
            barrier()
            torch.cuda.synchronize(dev)
            for i in range(args.steps):
                s2["ev"][i][0].record(stream)
                s2["launch"]()
                s2["ev"][i][1].record(stream)
            torch.cuda.synchronize(dev)
            ms_hot = reduce_max(statistics.mean(e0.elapsed_time(e1) for e0, e1 in s2["ev"]))
            entry["hot_l2"] = {"value": world * w2.flops / (ms_hot * 1e-3) / 1e12, "unit": UNIT,
                               "ms_per_step": ms_hot,
                               "gbs": w2.algorithmic_bytes / (ms_hot * 1e-3) / 1e9,
                               "l2": "operands left in L2 by the previous launch"}
        also.append(entry)
        del s2

    # ---------------------------------------------------------------- end to end (host buffers)
    e2e = run_e2e(torch, binding, w, s, args, dev, stream, barrier, reduce_max, world) \
        if not args.no_e2e else None

    # ---------------------------------------------------------------- roofline + CPU baseline
    return finish(torch, binding, dist, w, s, args, rank, world, dev, step_ms, value, kernel_ms,
                  region_ms, launches_per_step, clocks, also, e2e)


def run_e2e(torch, binding, w, s, args, dev, stream, barrier, max_over_ranks, world):
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    A_h = s["A"].pin_memory()
    B_h = s["B"].pin_memory()
    bias_h = s["bias"].pin_memory() if s["bias"] is not None else None
    C_h = torch.empty(w.M, w.N, dtype=torch.float16, pin_memory=True)
    has_bias = bias_h is not None and w.epilogue != 0
    ws_bytes = binding.tg_gemm_host_workspace_size(w.M, w.N, w.K, has_bias)
    del s["a"], s["b"], s["c"]
    torch.cuda.empty_cache()
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

    def e2e_call():
        st = binding.tg_gemm_host(A_h.data_ptr(), B_h.data_ptr(),
                                  bias_h.data_ptr() if has_bias else None, C_h.data_ptr(),
                                  w.M, w.N, w.K, w.epilogue, ws.data_ptr(), ws_bytes,
                                  stream.cuda_stream)
        if st != binding.TG_OK:
            raise binding.TgError(st, "tg_gemm_host")

    e2e_call()
    torch.cuda.synchronize(dev)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_call()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps)
    h2d = 2 * (w.M * w.K + w.K * w.N + (w.N if has_bias else 0))
    d2h = 2 * w.M * w.N
    return {"value": world * w.flops / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
            "path": "tg_gemm_host: pinned host -> device copies, GEMM in row panels, copy back, overlapped on three streams"}


def roofline(w, kernel_ms, peaks, peak_src, peak_kind, kcfg, big):
    """Roofline entry of one GEMM workload: TFLOP/s against the tensor peak for
    shapes above about 100 flop per byte (or larger than L2), else GB/s of
    algorithmic bytes against the copy bandwidth; DRAM traffic per launch from
    the committed ncu summary of the same kernel and configuration, if any."""
    if big or w.flops / max(w.algorithmic_bytes, 1) > 100:
        tens = peaks["bf16_tflops"] if peak_kind == "burst" else peaks["bf16_tflops_sustained"]
        achieved = w.flops / (kernel_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tens, "unit": "TFLOP/s",
                "frac": achieved / tens,
                "peak_source": f"{peak_src} bf16 {peak_kind} x 1.0 (fp16:bf16 dense ratio)"}
    else:
        achieved = w.algorithmic_bytes / (kernel_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "peak_source": f"{peak_src} copy bandwidth"}
    roof["traffic"] = profiled_traffic(w.name, kcfg)
    roof["algorithmic_per_launch"] = {"flops": w.flops, "bytes": w.algorithmic_bytes}
    roof["kernel_ms"] = kernel_ms
    return roof


def finish(torch, binding, dist, w, s, args, rank, world, dev, step_ms, value, kernel_ms,
           region_ms, launches_per_step, clocks, also, e2e):
    from tensor_core_gemm_fp16_b200 import workloads as wl
    peaks, peak_src = load_peaks()
    peak_kind = "burst" if region_ms < 1000.0 else "sustained"
    num_sms = torch.cuda.get_device_properties(dev).multi_processor_count
    kcfg = binding.tg_config_info(args.config) if args.config >= 0 else \
        binding.tg_gemm_select_config(w.M, w.N, w.K, w.epilogue, num_sms)
    roof = roofline(w, kernel_ms, peaks, peak_src, peak_kind, kcfg, s["big"])
    for entry in also:
        if entry["kind"] != "gemm":
            continue
        w2 = wl.WORKLOADS[entry["workload"]]
        entry["roofline"] = roofline(
            w2, entry["ms_per_step"], peaks, peak_src, "burst",
            binding.tg_gemm_select_config(w2.M, w2.N, w2.K, w2.epilogue, num_sms), False)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tflops, secs, rows, cores = oracle_sample(w, s["A"], s["B"], s["bias"],
                                                  target_s=args.cpu_seconds)
        cpu = {"value": tflops, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{rows} evenly spaced full rows of the {w.M}x{w.N}x{w.K} output "
                         f"({rows * w.N} outputs) in {secs:.1f} s, fp64, one call incl. decode",
               "single_core": oracle_single_core()}

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": workload_config(w, {
            "kernel_config": kcfg,
            "l2": ("inputs larger than L2 (%.0f MiB vs 126 MiB), launches back to back"
                   % (2 * (w.M * w.K + w.K * w.N + w.M * w.N) / 2 ** 20))
            if s["big"] else "L2 flushed (256 MiB write) between timed launches"}),
        "pct_of_fp16_dense_peak_nominal": 100.0 * value / world / NOMINAL_FP16_DENSE_TFLOPS,
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "also": also,
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="fused_8192")
    ap.add_argument("--also", nargs="*",
                    default=["gemm_256", "gemm_2048", "fused_2048", "ragged_fused",
                             "fused_tanh_2048", "softmax_8192x256x4096",
                             "deepk_fused_1024x1024x8192", "attn_4x16x2048x128",
                             "attn_causal_4x16x2048x128"],
                    help="other workloads timed the same way and reported under 'also'")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--config", type=int, default=-1,
                    help="force a kernel configuration id for the main workload (profiling)")
    ap.add_argument("--shape", type=int, nargs=3, metavar=("M", "N", "K"),
                    help="custom fused workload (bias + GELU, N(0,1) inputs, B scaled by "
                         "1/sqrt(K), seed 7) instead of --workload; for profiling cases")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)     # at least 3 untimed warm-up steps, always
    from tensor_core_gemm_fp16_b200 import workloads as wl
    if args.shape:
        M, N, K = args.shape
        w = wl.Workload(f"fused_{M}x{N}x{K}", M, N, K, wl.EPI_BIAS_GELU, "normal", 7,
                        b_scale=1.0 / math.sqrt(max(K, 1)), has_bias=True)
    else:
        w = wl.WORKLOADS[args.workload]
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != args.gpus:
        world = max(world, 1)
    if args.impl == "reference":
        return run_reference(args, w, rank, world)
    return run_ours(args, w, rank, world)


if __name__ == "__main__":
    sys.exit(main())
