"""Benchmark of the LLM.int8() decomposed linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Prints ONE JSON line (rank 0).  Workloads (seeded synthetic inputs, int8_quantized_02_b200.synth):
  decode     (default) X [b, 4096] for b in (1, 8, 16), six outlier columns |x| in [6, 60] on
             every row; CB [16384, 4096] quantized once beforehand.  One step = the three
             llmint8_linear calls.  Metric: weight-streaming GB/s =
             sum_b (N*K + 4N + 2bK + 2bN) / time.
  ffn6.7b    X [2048, 4096] . W1^T (16384 outputs), then X2 [2048, 16384] . W2^T (4096 outputs);
             six outlier columns of U(6, 20) on 75 % of rows.  Metric: TOPS = 2MNK / time.
  proj175b   X [4096, 12288] . W^T (49152 outputs), W ~ N(0, 0.01).  TOPS.
  sweep      X [4096, 8192] . W^T (8192 outputs); one step = K' in {0, 6, 64, 512} at
             threshold 6, plus threshold=inf and threshold=0.  TOPS.
Multi-GPU (torchrun): replicas only - every rank runs the same workload on its own GPU with no
data-path collective; value = units of all ranks / max-over-ranks time ("scaling": "weak").
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from int8_quantized_02_b200 import synth  # noqa: E402

DECODE_BATCHES = (1, 8, 16)
L2_BYTES = 126 * 1024 * 1024


# ---------------------------------------------------------------------------- helpers ----

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=p["hbm_gbs"], bf16_tflops=p["bf16_tflops"],
                    bf16_tflops_sustained=p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                source="fallback")


class ClockSampler:
    """SM clock and throttle reasons sampled (NVML, read-only) while the timed region runs."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, device_index: int):
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._nvml = None
        self._handle = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            handle = None
            uuid = getattr(props, "uuid", None)
            if uuid is not None:
                try:
                    handle = pynvml.nvmlDeviceGetHandleByUUID(f"GPU-{uuid}")
                except Exception:  # noqa: BLE001
                    handle = None
            if handle is None:
                handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self._nvml, self._handle = pynvml, handle
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001 - clocks are reported as unavailable
            self._nvml = None

    def _sample(self):
        nv, h = self._nvml, self._handle
        try:
            sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
            reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
            self.samples.append((sm, reasons))
        except Exception:  # noqa: BLE001
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(0.005)

    def __enter__(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=10)
            self._sample()              # the clocks as the region ends

    def summary(self):
        if self._nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "NVML unavailable"}
        active = set()
        for _, r in self.samples:
            for name, const in self.REASONS:
                if r & getattr(self._nvml, const, 0):
                    active.add(name)
        sm = [s for s, _ in self.samples]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(active), "samples": len(sm)}


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "int8_quantized_02_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per launch of the product kernel from the committed ncu summary of this
    workload, when it was taken on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", f"traffic_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_hash = re.search(r"kernel_source_hash:\s*(\w+)", text)
    m_val = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not m_hash or not m_val or m_hash.group(1) != kernel_source_hash():
        return None
    return float(m_val.group(1))


# -------------------------------------------------------------------------- workloads ----

class Call:
    """One llmint8_linear call with its resident inputs (and rotating weight copies)."""

    def __init__(self, L, torch, X, CBs, SCBs, threshold, name, units, kernel_bytes,
                 h2d_bytes, d2h_bytes, cap, rotation):
        self.L, self.torch = L, torch
        self.X, self.CBs, self.SCBs = X, CBs, SCBs
        self.t, self.name = threshold, name
        self.units, self.kernel_bytes = units, kernel_bytes
        self.h2d_bytes, self.d2h_bytes = h2d_bytes, d2h_bytes
        M, K = X.shape
        N = CBs[0].shape[0]
        self.M, self.K, self.N = M, K, N
        self.cap = cap
        self.ws = torch.empty((L.llmint8_linear_workspace_size(M, N, K, cap),),
                              dtype=torch.uint8, device="cuda")
        self.Y = torch.empty((M, N), dtype=torch.float16, device="cuda")
        self.rotation = rotation          # shared by all calls on the same weight copies
        self.plans = self.plan()

    def plan(self, X=None):
        """Prepared calls on X (default: the resident input), one per weight copy."""
        X = self.X if X is None else X
        return [self.L.LinearPlan(X, self.CBs[i], self.SCBs[i], threshold=self.t,
                                  max_outliers=self.cap, Y=self.Y, workspace=self.ws)
                for i in range(len(self.CBs))]

    def host_plan(self, X_host, Y_host, X_dev, stream):
        """Prepared host-buffer calls (llmint8_linear_host) on `stream`, one per weight copy."""
        return [self.L.LinearHostPlan(X_host, self.CBs[i], self.SCBs[i], Y_host=Y_host,
                                      threshold=self.t, max_outliers=self.cap, X_dev=X_dev,
                                      Y_dev=self.Y, workspace=self.ws, stream=stream)
                for i in range(len(self.CBs))]

    def run(self, plans=None):
        plans = self.plans if plans is None else plans
        i = self.rotation[0] % len(plans)
        self.rotation[0] += 1
        plans[i]()


def _weights(L, torch, N, K, std, copies):
    W = torch.from_numpy(synth.weight(N, K, std, seed=0)).cuda()
    CB, SCB = L.llmint8_quantize_weight_colwise(W)
    del W
    CBs, SCBs = [CB], [SCB]
    for _ in range(copies - 1):
        CBs.append(CB.clone())
        SCBs.append(SCB.clone())
    return CBs, SCBs


def build_workload(name, L, torch):
    calls = []
    if name == "decode":
        N, K = 16384, 4096
        copies = max(2, -(-3 * L2_BYTES // (N * K)) + 1)   # > 3 x L2 of weights in rotation
        CBs, SCBs = _weights(L, torch, N, K, 0.02, copies)
        rotation = [0]
        for b in DECODE_BATCHES:
            wl = synth.decode(b)
            X = torch.from_numpy(wl.make_x()[0]).cuda()
            nbytes = N * K + 4 * N + 2 * b * K + 2 * b * N
            calls.append(Call(L, torch, X, CBs, SCBs, 6.0, wl.name, nbytes,
                              N * K + 4 * N + b * K + 4 * b + 2 * b * N, 2 * b * K, 2 * b * N, 64,
                              rotation))
        unit, metric_bound = "GB/s", "hbm"
    elif name in ("ffn6.7b", "proj175b", "sweep"):
        if name == "ffn6.7b":
            specs = [(synth.FFN_W1, 6.0), (synth.FFN_W2, 6.0)]
        elif name == "proj175b":
            specs = [(synth.PROJ_175B, 6.0)]
        else:
            specs = [(synth.sweep(k), 6.0) for k in (0, 6, 64, 512)] + \
                [(synth.sweep(6, float("inf")), float("inf")), (synth.sweep(0, 0.0), 0.0)]
        cache = {}
        for wl, t in specs:
            key = (wl.N, wl.K, wl.w_std)
            if key not in cache:
                cache[key] = _weights(L, torch, wl.N, wl.K, wl.w_std, 1)
            CBs, SCBs = cache[key]
            X = torch.from_numpy(wl.make_x()[0]).cuda()
            cap = wl.K if t <= 0 else 512
            calls.append(Call(L, torch, X, CBs, SCBs, t, wl.name, wl.int8_ops,
                              wl.M * wl.K * 2 + wl.N * wl.K + 2 * wl.M * wl.N,
                              2 * wl.M * wl.K, 2 * wl.M * wl.N, cap, [0]))
        unit, metric_bound = "TOPS", "tensor"
    else:
        raise SystemExit(f"unknown workload {name}")
    return calls, unit, metric_bound


def unit_value(units, seconds, unit):
    return units / seconds / 1e9 if unit == "GB/s" else units / seconds / 1e12


def max_over_ranks(seconds: float, world: int, device=None) -> float:
    """The slowest rank's time (every rank calls this at the same point)."""
    if world <= 1:
        return float(seconds)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(seconds)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(units_per_step: float, steps: int, world: int, seconds: float,
                    unit: str) -> float:
    """Units all ranks processed (replicas: the same per rank) / the max-over-ranks time."""
    return unit_value(units_per_step * steps * world, seconds, unit)


# ------------------------------------------------------------------------ our arm ----

def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from int8_quantized_02_b200 import llmint8 as L

    torch.cuda.set_device(local_rank)
    L.load()
    calls, unit, bound = build_workload(args.workload, L, torch)
    step_units = sum(c.units for c in calls)

    def step():
        for c in calls:
            c.run()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    for c in calls:
        st = L.llmint8_device_status(c.ws)
        if st != L.OK:
            raise SystemExit(f"{c.name}: device status {L.status_string(st)}")

    # ---- timed region: whole steps, inputs resident, CUDA events on the launching stream.
    # Prefill calls run for a tenth of a millisecond or more, so a pair of profile events
    # around each GEMM launch costs little (the GEMM then starts after its quantize kernel
    # instead of overlapping its tail) and gives the dominant kernel's own duration.  A decode call
    # lasts about 20 us and an event pair adds about 5 us, so decode records no per-call
    # events: its weight-streaming kernel spans the whole call (the quantize kernel runs under
    # it as a programmatic dependent), and the call's duration is region time / calls.
    stream = torch.cuda.current_stream()
    per_call_events = bound != "hbm"
    kev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in calls] for _ in range(args.steps if per_call_events else 0)]
    # torch creates an event's CUDA handle on its first record(): record each once here so
    # the library can re-record the same handles around the product kernel
    for row in kev:
        for ev_a, ev_b in row:
            ev_a.record(stream)
            ev_b.record(stream)
    torch.cuda.synchronize()
    launches0 = L.llmint8_kernel_launch_count()
    barrier()
    with ClockSampler(local_rank) as clk:
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for s in range(args.steps):
            for j, c in enumerate(calls):
                if per_call_events:
                    L.llmint8_set_profile_events(*kev[s][j])
                c.run()
        e1.record(stream)
        if per_call_events:
            L.llmint8_set_profile_events(None, None)
        torch.cuda.synchronize()
    barrier()
    launches = L.llmint8_kernel_launch_count() - launches0
    elapsed = max_over_ranks(e0.elapsed_time(e1) / 1e3, world, device="cuda")
    if per_call_events:
        call_s = [sum(kev[s][j][0].elapsed_time(kev[s][j][1]) for s in range(args.steps))
                  / 1e3 / args.steps for j in range(len(calls))]
    else:
        # no per-call split inside the region: each call gets its share of the step by units
        call_s = [elapsed / args.steps * c.units / step_units for c in calls]
    kern_s = sum(call_s) * args.steps
    for c in calls:
        st = L.llmint8_device_status(c.ws)
        if st != L.OK:
            raise SystemExit(f"{c.name}: device status {L.status_string(st)}")

    # ---- per-call figures, after the timed region: each decode call alone, back to back on
    # rotating weights, between one pair of events (the headline above does not use these)
    alone_s = None
    if not per_call_events:
        alone_s = []
        for c in calls:
            b0 = torch.cuda.Event(enable_timing=True)
            b1 = torch.cuda.Event(enable_timing=True)
            b0.record(stream)
            for _ in range(args.steps):
                c.run()
            b1.record(stream)
            torch.cuda.synchronize()
            alone_s.append(max_over_ranks(b0.elapsed_time(b1) / 1e3 / args.steps, world,
                                          device="cuda"))

    # ---- end to end through the C ABI's host-buffer call: every call copies its X from pinned
    # host memory, runs the layer and copies Y back into pinned host memory.  The calls of a
    # step share no buffer (own X, Y and workspace), so each runs on a stream of its own and
    # one call's copies overlap the others' kernels; a call's steps stay in order.
    hosts = [(c.X.cpu().pin_memory(),
              torch.empty((c.M, c.N), dtype=torch.float16).pin_memory()) for c in calls]
    xd = [torch.empty_like(c.X) for c in calls]
    e2e_streams = [torch.cuda.Stream() for _ in calls]
    e2e_plans = [c.host_plan(hosts[j][0], hosts[j][1], xd[j], e2e_streams[j])
                 for j, c in enumerate(calls)]
    e2e_steps = max(1, min(args.steps, 50))

    def e2e_run(n):
        start = torch.cuda.Event()
        start.record(stream)
        for st in e2e_streams:
            st.wait_event(start)
        for _ in range(n):
            for j, c in enumerate(calls):
                c.run(e2e_plans[j])
        for st in e2e_streams:
            done = torch.cuda.Event()
            done.record(st)
            stream.wait_event(done)

    e2e_run(2)
    barrier()
    a0 = torch.cuda.Event(enable_timing=True)
    a1 = torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    e2e_run(e2e_steps)
    a1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_s = max_over_ranks(a0.elapsed_time(a1) / 1e3, world, device="cuda")
    for j, c in enumerate(calls):
        st = L.llmint8_device_status(c.ws)
        if st != L.OK:
            raise SystemExit(f"{c.name} (end to end): device status {L.status_string(st)}")
        if not torch.equal(hosts[j][1], c.Y.cpu()):
            raise SystemExit(f"{c.name} (end to end): host Y differs from the device Y")

    peaks = measured_peaks()
    traffic = profiled_traffic(args.workload)
    if bound == "hbm":
        # algorithmic bytes of a call: N*K + 4N + 2MK + 2MN (weights, scales, X in, Y out)
        achieved = step_units * args.steps / kern_s / 1e9
        peak = peaks["hbm_gbs"]
        roof_unit = "GB/s"
        kernel_name = "llmint8_decode_kernel (+ llmint8_decode_quantize_kernel under it)"
        timing = "device time of the timed region / calls (no per-call events)"
    else:
        achieved = step_units * args.steps / kern_s / 1e12
        peak = 2.0 * peaks["bf16_tflops"]           # int8 dense = 2 x bf16 dense (nominal ratio)
        roof_unit = "TOPS"
        kernel_name = ("llmint8_gemm_pair_kernel" if all(c.M > 128 for c in calls)
                       else "llmint8_gemm_kernel")
        timing = "CUDA events around each GEMM launch, averaged over the timed region"
    result = {
        "metric": "LLM.int8 linear TOPS (prefill) / weight GB/s (decode); fraction of roofline",
        "value": whole_job_value(step_units, args.steps, world, elapsed, unit),
        "unit": unit,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": elapsed / args.steps * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "i8",
        "dtype_note": "int8 x int8 -> int32 product; fp16 in/out; fp16 x fp16 -> fp32 outlier part",
        "data": "synthetic (seeded, int8_quantized_02_b200.synth)",
        "config": workload_config(args.workload, calls),
        "roofline": {"bound": bound, "achieved": achieved, "peak": peak, "unit": roof_unit,
                     "frac": achieved / peak,
                     "peak_source": f"{peaks['source']} "
                                    + ("hbm_gbs" if bound == "hbm" else "2 x bf16_tflops (burst)"),
                     "kernel": kernel_name, "timing": timing,
                     "traffic": traffic},
        "e2e": {"value": whole_job_value(step_units, e2e_steps, world, e2e_s, unit), "unit": unit,
                "h2d_bytes_per_step": sum(c.h2d_bytes for c in calls),
                "d2h_bytes_per_step": sum(c.d2h_bytes for c in calls)},
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
        "per_call": {c.name: None for c in calls},
    }
    # per-call figure: the GEMM's own events (prefill) or the call run alone (decode)
    for j, c in enumerate(calls):
        sec = call_s[j] if alone_s is None else alone_s[j]
        v = c.units / sec / (1e9 if bound == "hbm" else 1e12)
        result["per_call"][c.name] = {("call_us" if bound == "hbm" else "kernel_us"):
                                      sec * 1e6, unit: v}
        if alone_s is not None:
            result["per_call"][c.name]["timing"] = "this call alone, steps back-to-back calls"
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(args.workload)
    return result


def workload_config(name, calls):
    cfg = {"workload": name,
           "calls": [{"name": c.name, "M": c.M, "K": c.K, "N": c.N, "threshold": c.t,
                      "max_outliers": c.cap} for c in calls],
           "parallelism": "replicas"}
    if name == "decode":
        cfg["l2"] = (f"{len(calls[0].CBs)} rotating int8 weight copies "
                     f"({len(calls[0].CBs) * calls[0].N * calls[0].K / 2**20:.0f} MiB > 126 MiB L2)")
    else:
        cfg["l2"] = "inputs larger than L2 (weights and activations)"
    return cfg


# ------------------------------------------------------------------- oracle (CPU) ----

def _oracle_sample(name):
    """A bounded sample of every call of the workload for the CPU oracle, and its metric units:
    the same X rows and shapes, against a slice of the output channels (and, for prefill,
    of the token rows)."""
    from oracle import oracle
    pieces, units = [], 0
    if name == "decode":
        N, K = 16384, 4096
        rows = 2048                                   # 1/8 of the output channels
        CB, SCB = oracle.quantize_weight_colwise(synth.weight(rows, K, 0.02, seed=0))
        for b in DECODE_BATCHES:
            pieces.append((synth.decode(b).make_x()[0], CB, SCB, 6.0))
            units += rows * K + 4 * rows + 2 * b * K + 2 * b * rows
        desc = (f"decode b=1,8,16: X [b, {K}] against {rows} of the {N} output channels")
        return pieces, units, desc
    specs = {"ffn6.7b": [(synth.FFN_W1, 6.0), (synth.FFN_W2, 6.0)],
             "proj175b": [(synth.PROJ_175B, 6.0)],
             "sweep": [(synth.sweep(k), 6.0) for k in (0, 6, 64, 512)]
             + [(synth.sweep(6, float("inf")), float("inf")), (synth.sweep(0, 0.0), 0.0)]}[name]
    rows_x, rows_w = 128, 256
    for wl, t in specs:
        X = wl.make_x()[0][:rows_x].copy()
        CB, SCB = oracle.quantize_weight_colwise(synth.weight(rows_w, wl.K, wl.w_std, seed=0))
        pieces.append((X, CB, SCB, t))
        units += 2 * rows_x * rows_w * wl.K
    desc = (f"{name}: every call on the first {rows_x} rows of X against {rows_w} "
            f"output channels")
    return pieces, units, desc


def _oracle_step(pieces):
    from oracle import oracle
    for X, CB, SCB, t in pieces:
        oracle.linear(X, CB, SCB, threshold=t)


def _cores():
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count()))


def cpu_baseline(name, budget_s=15.0):
    pieces, units, desc = _oracle_sample(name)
    _oracle_step(pieces[:1])                                  # load + warm
    times = []
    deadline = time.perf_counter() + budget_s
    while not times or time.perf_counter() < deadline:
        t0 = time.perf_counter()
        _oracle_step(pieces)
        times.append(time.perf_counter() - t0)
    unit = "GB/s" if name == "decode" else "TOPS"
    sec = statistics.median(times)
    return {"value": unit_value(units, sec, unit), "unit": unit, "cores": _cores(),
            "kind": "oracle", "sample": f"{desc}; median of {len(times)} runs of {sec:.3f} s"}


def run_reference(args, rank, world):
    """The oracle timed on the host cores, each step a bounded sample of the same workload."""
    if rank != 0:
        return None
    pieces, units, desc = _oracle_sample(args.workload)
    for _ in range(min(args.warmup, 1)):
        _oracle_step(pieces)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_step(pieces)
    sec = time.perf_counter() - t0
    unit = "GB/s" if args.workload == "decode" else "TOPS"
    value = unit_value(units * args.steps, sec, unit)
    return {
        "impl": "reference",
        "metric": "LLM.int8 linear TOPS (prefill) / weight GB/s (decode); fraction of roofline",
        "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": sec / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, int8_quantized_02_b200.synth)",
        "config": {"workload": args.workload, "sample": desc, "parallelism": "replicas"},
        "cpu_baseline": {"value": value, "unit": unit, "cores": _cores(), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: 1000 for decode, 20 otherwise; 20 for the "
                         "reference arm)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="decode",
                    choices=("decode", "ffn6.7b", "proj175b", "sweep"))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.steps is None:
        # a decode step lasts about 65 us: 1000 of them keep the clock sampler in the region
        args.steps = 1000 if args.workload == "decode" and args.impl == "ours" else 20
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        out = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
