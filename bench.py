"""Benchmark of the LLM.int8() decomposed linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Prints ONE JSON line (rank 0).  By default every workload runs: decode is the headline (the
line's value, roofline, e2e, ...), and the prefill workloads follow under "workloads", each
with the same keys.  Workloads (seeded synthetic inputs, int8_quantized_02_b200.synth):
  decode     X [b, 4096] for b in (1, 8, 16), six outlier columns |x| in [6, 60] on every row;
             CB [16384, 4096] quantized once beforehand.  One step = the three llmint8_linear
             calls.  Metric: weight-streaming GB/s = sum_b (N*K + 4N + 2bK + 2bN) / time.
  decode175b the same three calls at the 175B-class projection shape: X [b, 12288] against
             CB [49152, 12288] (604 MB).  GB/s as for decode.
  ffn6.7b    X [2048, 4096] . W1^T (16384 outputs), then X2 [2048, 16384] . W2^T (4096 outputs);
             six outlier columns of U(6, 20) on 75 % of rows.  Metric: TOPS = 2MNK / time.
  ffn6.7b_chain  the FFN pair chained: W2 takes W1's output Y1 as its X.  The W1 call
             (llmint8_linear_next_bitmaps) also writes the outlier bitmaps of Y1, and the W2
             call (llmint8_linear_with_bitmaps) uses them, so it makes no outlier scan of its
             own.  Y1 of these random weights has about 700 columns reaching 6.0 (capacity
             1024).  TOPS.
  proj175b   X [4096, 12288] . W^T (49152 outputs), W ~ N(0, 0.01).  TOPS.
  sweep      X [4096, 8192] . W^T (8192 outputs); one step = K' in {0, 6, 64, 512} at
             threshold 6, plus threshold=inf and threshold=0.  TOPS.
Timing: each workload's region of K whole steps (inputs resident in HBM, larger than L2 or
rotated through more than 3 x L2) is bracketed by a barrier and a synchronize on both sides and
timed with CUDA events on the launching stream (the slowest rank's time); the region is
repeated until the repeats add up to about a second (half a second per prefill workload) and
the value is the median over the repeats, reported with its spread.
Multi-GPU (torchrun): replicas only - every rank runs the same workload on its own GPU with no
data-path collective; value = units of all ranks / max-over-ranks time ("scaling": "weak").
"""
from __future__ import annotations

import argparse
import json
import os
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


class ChainHead(Call):
    """The first layer of a chained pair: llmint8_linear_next_bitmaps, which also writes the
    outlier bitmaps of its Y (`bits`) for the second layer."""

    def __init__(self, *args, next_threshold=6.0, **kw):
        self.next_t = next_threshold
        super().__init__(*args, **kw)

    def _call(self, X):
        L, torch = self.L, self.torch
        if not hasattr(self, "bits"):
            self.bits = torch.empty(((self.M + 31) // 32, (self.N + 31) // 32),
                                    dtype=torch.int32, device="cuda")
        fn = L.load().llmint8_linear_next_bitmaps
        args = (L._ptr(X), self.M, self.K, L._ptr(self.CBs[0]), L._ptr(self.SCBs[0]), self.N,
                None, None, L.ctypes.c_float(self.t), self.cap, L._ptr(self.Y), L._ptr(self.ws),
                self.ws.numel(), L._stream(None), None, L.ctypes.c_float(self.next_t),
                L._ptr(self.bits))

        def call():
            code = fn(*args)
            if code != L.OK:
                raise L.LLMInt8Error(code, "llmint8_linear_next_bitmaps")
        return call

    def plan(self, X=None):
        return [self._call(self.X if X is None else X)]

    def host_plan(self, X_host, Y_host, X_dev, stream):
        run = self._call(X_dev)

        def call():
            X_dev.copy_(X_host, non_blocking=True)
            run()
        return [call]


class ChainTail(Call):
    """The second layer of a chained pair: llmint8_linear_with_bitmaps on the head's Y with
    the head's bitmaps (no outlier scan of its own)."""

    def __init__(self, L, torch, head, CBs, SCBs, name, units, kernel_bytes, d2h_bytes, cap):
        self.head = head
        super().__init__(L, torch, head.Y, CBs, SCBs, head.next_t, name, units, kernel_bytes,
                         0, d2h_bytes, cap, [0])

    def _call(self):
        L = self.L
        fn = L.load().llmint8_linear_with_bitmaps
        bits = self.head.bits
        args = (L._ptr(self.head.Y), self.M, self.K, L._ptr(self.CBs[0]), L._ptr(self.SCBs[0]),
                self.N, None, None, L._ptr(bits), bits.shape[0], self.cap, L._ptr(self.Y),
                L._ptr(self.ws), self.ws.numel(), L._stream(None), None)

        def call():
            code = fn(*args)
            if code != L.OK:
                raise L.LLMInt8Error(code, "llmint8_linear_with_bitmaps")
        return call

    def plan(self, X=None):
        return [self._call()]

    def host_plan(self, X_host, Y_host, X_dev, stream):
        run = self._call()

        def call():
            run()
            Y_host.copy_(self.Y, non_blocking=True)
        return [call]


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
    if name in DECODE_WORKLOADS:
        make = synth.decode if name == "decode" else synth.decode175b
        N, K, std = make(1).N, make(1).K, make(1).w_std
        copies = max(2, -(-3 * L2_BYTES // (N * K)) + 1)   # > 3 x L2 of weights in rotation
        CBs, SCBs = _weights(L, torch, N, K, std, copies)
        rotation = [0]
        for b in DECODE_BATCHES:
            wl = make(b)
            X = torch.from_numpy(wl.make_x()[0]).cuda()
            nbytes = N * K + 4 * N + 2 * b * K + 2 * b * N
            calls.append(Call(L, torch, X, CBs, SCBs, 6.0, wl.name, nbytes,
                              N * K + 4 * N + b * K + 4 * b + 2 * b * N, 2 * b * K, 2 * b * N, 64,
                              rotation))
        unit, metric_bound = "GB/s", "hbm"
    elif name == "ffn6.7b_chain":
        w1, w2 = synth.FFN_W1, synth.FFN_W2
        CB1, SCB1 = _weights(L, torch, w1.N, w1.K, w1.w_std, 1)
        CB2, SCB2 = _weights(L, torch, w2.N, w2.K, w2.w_std, 1)
        X = torch.from_numpy(w1.make_x()[0]).cuda()
        head = ChainHead(L, torch, X, CB1, SCB1, 6.0, "ffn6.7b_w1_next_bitmaps", w1.int8_ops,
                         w1.M * w1.K * 2 + w1.N * w1.K + 2 * w1.M * w1.N,
                         2 * w1.M * w1.K, 0, 512, [0], next_threshold=6.0)
        tail = ChainTail(L, torch, head, CB2, SCB2, "ffn6.7b_w2_with_bitmaps", w2.int8_ops,
                         w2.M * w2.K * 2 + w2.N * w2.K + 2 * w2.M * w2.N, 2 * w2.M * w2.N, 1024)
        calls = [head, tail]
        unit, metric_bound = "TOPS", "tensor"
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


def int8_peak_kind(clocks):
    """Which measured bf16 figure a prefill line is judged against: its repeated regions keep
    the tensor cores busy for about half a second, and when their clock record shows the
    power cap (or SM clocks below 95 % of the maximum) the kernels ran in the sustained
    regime; otherwise the burst figure.  Returns (peaks key, capped)."""
    capped = "sw_power_cap" in clocks.get("reasons", []) or bool(
        clocks.get("sm_mhz") and clocks.get("sm_max_mhz")
        and clocks["sm_mhz"] < 0.95 * clocks["sm_max_mhz"])
    return ("bf16_tflops_sustained" if capped else "bf16_tflops"), capped


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


def repeat_count(region_s: float, target_s: float, lo: int = 3, hi: int = 200) -> int:
    """How many times to repeat a timed region of `region_s` seconds so that the repeats
    together last about `target_s` (at least `lo`, at most `hi`)."""
    if region_s <= 0:
        return hi
    return int(max(lo, min(hi, -(-target_s // region_s))))


def spread(values):
    """Median and spread of the per-repeat values of a metric."""
    v = sorted(values)
    q = lambda f: v[min(len(v) - 1, int(round(f * (len(v) - 1))))]  # noqa: E731
    return {"n": len(v), "median": statistics.median(v), "min": v[0], "max": v[-1],
            "p10": q(0.1), "p90": q(0.9)}


# ------------------------------------------------------------------------ our arm ----

# Seconds of timed work the repeats of each workload's region add up to.
TARGET_S = {"decode": 1.0, "decode175b": 0.5, "ffn6.7b": 0.5, "ffn6.7b_chain": 0.5,
            "proj175b": 0.5, "sweep": 0.5}
ALL_WORKLOADS = ("decode", "decode175b", "ffn6.7b", "ffn6.7b_chain", "proj175b", "sweep")
DECODE_WORKLOADS = ("decode", "decode175b")


def run_workload(name, args, rank, world, local_rank):
    """Every figure of one workload: the repeated timed region (value), the dominant kernel's
    roofline, the per-call figures, end to end through the host-buffer call, clocks, and
    (rank 0, one GPU) the oracle on the host cores."""
    import torch
    import torch.distributed as dist

    from int8_quantized_02_b200 import llmint8 as L

    calls, unit, bound = build_workload(name, L, torch)
    step_units = sum(c.units for c in calls)
    stream = torch.cuda.current_stream()

    def step():
        for c in calls:
            c.run()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def check_status(what):
        for c in calls:
            st = L.llmint8_device_status(c.ws)
            if st != L.OK:
                raise SystemExit(f"{c.name}{what}: device status {L.status_string(st)}")

    def region(n_steps, run=step):
        """One timed region of n_steps whole steps: barrier + synchronize on both sides,
        CUDA events on the launching stream, the slowest rank's time."""
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n_steps):
            run()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        return max_over_ranks(e0.elapsed_time(e1) / 1e3, world, device="cuda")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    check_status("")

    # ---- the timed region, K whole steps with inputs resident, repeated; an untimed region
    # of the same length first sets the repeat count (the same on every rank)
    reps = repeat_count(region(args.steps), TARGET_S.get(name, 0.5),
                        hi=1000 if bound == "hbm" else 200)
    launches0 = L.llmint8_kernel_launch_count()
    with ClockSampler(local_rank) as clk:
        times = [region(args.steps) for _ in range(reps)]
    launches = L.llmint8_kernel_launch_count() - launches0
    check_status("")
    vals = [whole_job_value(step_units, args.steps, world, t, unit) for t in times]
    rep = spread(vals)
    t_med = statistics.median(times)

    # ---- the dominant kernel.  Decode: one kernel per call, so its duration is the region's
    # time per call (per-call events would add several microseconds to a ~15 us call).
    # Prefill: CUDA events around each GEMM launch in one extra region of K steps (the events
    # keep the GEMM from overlapping the tail of its row-quantization kernel, which costs
    # little at these sizes).
    peaks = measured_peaks()
    per_call = {}
    if bound == "hbm":
        achieved = step_units * args.steps / t_med / 1e9
        peak, roof_unit = peaks["hbm_gbs"], "GB/s"
        kernel_name = "llmint8_decode_kernel"
        timing = "median region time / calls (one kernel per call, no per-call events)"
        # each call alone, steps calls back to back (not used by the headline)
        for c in calls:
            t = region(args.steps, c.run)
            per_call[c.name] = {"call_us": t / args.steps * 1e6,
                                "GB/s": c.units / (t / args.steps) / 1e9,
                                "timing": "this call alone, steps back-to-back calls"}
        whole = None
    else:
        kev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in calls] for _ in range(args.steps)]
        # torch creates an event's CUDA handle on its first record(): record each once here
        # so the library can re-record the same handles around the product kernel
        for row in kev:
            for ev_a, ev_b in row:
                ev_a.record(stream)
                ev_b.record(stream)
        torch.cuda.synchronize()
        barrier()
        for s_ in range(args.steps):
            for j, c in enumerate(calls):
                L.llmint8_set_profile_events(*kev[s_][j])
                c.run()
        L.llmint8_set_profile_events(None, None)
        torch.cuda.synchronize()
        barrier()
        call_s = [max_over_ranks(sum(kev[s_][j][0].elapsed_time(kev[s_][j][1])
                                     for s_ in range(args.steps)) / 1e3 / args.steps,
                                 world, device="cuda") for j in range(len(calls))]
        achieved = step_units / sum(call_s) / 1e12
        peak_kind, capped = int8_peak_kind(clk.summary())
        peak, roof_unit = 2.0 * peaks[peak_kind], "TOPS"   # int8 = 2 x bf16 (nominal ratio)
        burst_peak = 2.0 * peaks["bf16_tflops"]
        kernel_name = ", ".join(dict.fromkeys(
            ("llmint8_gemm_pair" if c.M > 128 else "llmint8_gemm")
            + ("_bits" if isinstance(c, ChainHead) else "") + "_kernel" for c in calls))
        timing = "CUDA events around each GEMM launch, one region of K steps"
        for j, c in enumerate(calls):
            per_call[c.name] = {"kernel_us": call_s[j] * 1e6,
                                "TOPS": c.units / call_s[j] / 1e12}
        w = rep["median"] / world
        whole = {"achieved": w, "frac": w / peak, "frac_of_burst_peak": w / burst_peak,
                 "timing": "whole llmint8_linear calls (every kernel of the layer): median "
                           "region time"}

    # ---- end to end through the C ABI's host-buffer call, on the same single stream as the
    # timed region: every call copies its X in from pinned host memory, runs the layer and
    # copies Y out into pinned host memory
    hosts = [(c.X.cpu().pin_memory(),
              torch.empty((c.M, c.N), dtype=torch.float16).pin_memory()) for c in calls]
    xd = [torch.empty_like(c.X) for c in calls]
    e2e_plans = [c.host_plan(hosts[j][0], hosts[j][1], xd[j], stream)
                 for j, c in enumerate(calls)]

    def e2e_step():
        for j, c in enumerate(calls):
            c.run(e2e_plans[j])

    for _ in range(2):
        e2e_step()
    e2e_reps = repeat_count(region(args.steps, e2e_step), TARGET_S.get(name, 0.5) / 2, lo=3,
                            hi=50)
    e2e_times = [region(args.steps, e2e_step) for _ in range(e2e_reps)]
    e2e_vals = [whole_job_value(step_units, args.steps, world, t, unit) for t in e2e_times]
    check_status(" (end to end)")
    for j, c in enumerate(calls):
        if c.d2h_bytes and not torch.equal(hosts[j][1], c.Y.cpu()):
            raise SystemExit(f"{c.name} (end to end): host Y differs from the device Y")

    out = {
        "value": rep["median"],
        "unit": unit,
        "ms_per_step": t_med / args.steps * 1e3,
        "repeats": {**rep, "steps_per_repeat": args.steps,
                    "note": "value = median over repeats of the K-step timed region"},
        "config": workload_config(name, calls),
        "roofline": {"bound": bound, "achieved": achieved, "peak": peak, "unit": roof_unit,
                     "frac": achieved / peak,
                     "peak_source": f"{peaks['source']} "
                                    + ("hbm_gbs" if bound == "hbm" else
                                       (f"2 x {peak_kind} (sustained: the regions ran under "
                                        f"the power cap)" if capped else
                                        f"2 x {peak_kind} (burst)")),
                     "kernel": kernel_name, "timing": timing,
                     "traffic": None,
                     "traffic_note": "DRAM bytes are not measurable inside this run (no "
                                     "profiler); the per-launch ncu counters are in profiles/"},
        "e2e": {"value": statistics.median(e2e_vals), "unit": unit,
                "h2d_bytes_per_step": sum(c.h2d_bytes for c in calls),
                "d2h_bytes_per_step": sum(c.d2h_bytes for c in calls),
                "repeats": len(e2e_vals), "min": min(e2e_vals), "max": max(e2e_vals),
                "arrangement": "llmint8_linear_host per call, one stream (as the timed region)"},
        "gpu_launches": int(launches),
        "gpu_launches_note": f"library kernels launched in the {reps} timed repeats",
        "clocks": clk.summary(),
        "per_call": per_call,
    }
    if whole is not None:
        out["roofline"]["whole_call"] = whole
        out["roofline"]["frac_of_burst_peak"] = achieved / burst_peak
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(name, budget_s=15.0 if name == "decode" else 8.0)
    del calls, hosts, xd, e2e_plans
    torch.cuda.empty_cache()
    return out


def run_ours(args, rank, world, local_rank):
    import torch

    from int8_quantized_02_b200 import llmint8 as L

    torch.cuda.set_device(local_rank)
    L.load()
    names = ALL_WORKLOADS if args.workload == "all" else (args.workload,)
    results = {n: run_workload(n, args, rank, world, local_rank) for n in names}
    head_name = names[0]
    head = results[head_name]
    result = {
        "metric": "LLM.int8 linear TOPS (prefill) / weight GB/s (decode); fraction of roofline",
        "value": head["value"],
        "unit": head["unit"],
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "i8",
        "dtype_note": "int8 x int8 -> int32 product; fp16 in/out; fp16 x fp16 -> fp32 outlier part",
        "data": "synthetic (seeded, int8_quantized_02_b200.synth)",
    }
    for k in ("config", "repeats", "roofline", "e2e", "gpu_launches", "gpu_launches_note",
              "clocks", "per_call", "cpu_baseline"):
        if k in head:
            result[k] = head[k]
    if len(names) > 1:
        result["workloads"] = {n: results[n] for n in names[1:]}
    return result


def workload_config(name, calls):
    cfg = {"workload": name,
           "calls": [{"name": c.name, "M": c.M, "K": c.K, "N": c.N, "threshold": c.t,
                      "max_outliers": c.cap} for c in calls],
           "parallelism": "replicas"}
    if name in DECODE_WORKLOADS:
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
    if name in DECODE_WORKLOADS:
        make = synth.decode if name == "decode" else synth.decode175b
        N, K, std = make(1).N, make(1).K, make(1).w_std
        rows = 2048 if name == "decode" else 512       # a slice of the output channels
        CB, SCB = oracle.quantize_weight_colwise(synth.weight(rows, K, std, seed=0))
        for b in DECODE_BATCHES:
            pieces.append((make(b).make_x()[0], CB, SCB, 6.0))
            units += rows * K + 4 * rows + 2 * b * K + 2 * b * rows
        desc = (f"{name} b=1,8,16: X [b, {K}] against {rows} of the {N} output channels")
        return pieces, units, desc
    specs = {"ffn6.7b": [(synth.FFN_W1, 6.0), (synth.FFN_W2, 6.0)],
             # the chain's arithmetic is the layer's (its bitmaps are the outlier detection the
             # oracle's layer makes): the same sample as the FFN pair
             "ffn6.7b_chain": [(synth.FFN_W1, 6.0), (synth.FFN_W2, 6.0)],
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
    unit = "GB/s" if name in DECODE_WORKLOADS else "TOPS"
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
    unit = "GB/s" if args.workload in DECODE_WORKLOADS else "TOPS"
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
                    help="steps per timed region (default 20); the region is repeated until "
                         "the repeats add up to about a second, and the value is their median")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="all", choices=("all",) + ALL_WORKLOADS,
                    help="all (default): decode is the headline, the prefill workloads are "
                         "reported under 'workloads' in the same line")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.steps is None:
        args.steps = 20
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        if args.workload == "all":
            args.workload = "decode"      # the headline's workload
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
