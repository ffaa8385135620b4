"""Benchmark of the FP8 block-scaled GEMM library on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
for the default workload ("decode"), the six decode-shaped dense GEMMs of the
DeepGEMM pages' DeepSeek-V3/R1 inference shapes, M in {64, 128} x (N, K) in
{(2112, 7168), (32768, 512), (7168, 2048)}, each with its own E4M3 operands and
power-of-two block scales, every step through the library's public call.
The metric for M <= 128 is HBM bandwidth: algorithmic bytes (A, B, their
scales, and D) per second.  The same run then times the other configurations
of the metric -- "smoke" (dense 64 x 512 x 1024), "prefill" (four dense
M = 4096 GEMMs, TFLOPS), "contiguous" and "masked" (the two MoE grouped
layouts, TFLOPS) -- the same way and reports each, with its own roofline and
CPU-oracle baseline, under ``workloads`` in the same JSON line; the headline
``value`` stays the decode step.  ``--workload`` makes any of them (or
"bf16-decode" / "bf16-prefill": the same dense shapes on BF16 operands,
against the BF16 tensor peak) the headline instead.  The tensor peak of the
E4M3 roofline is the vendor library's measured dense E4M3 GEMM rate
(``profiles/fp8_peak.md``, written from ``--measure-fp8-peak``).

Timing: inputs sit in HBM, R copies of them at different addresses are rotated
so that the bytes touched between two visits of one copy exceed the 126 MB L2;
the steps of one rotation cycle are one captured CUDA graph; a barrier and a device
synchronisation bracket exactly K timed steps, timed with CUDA events; the
result is the maximum over ranks.  The library's kernel is the only kernel in
the timed region, so the roofline's achieved rate is the step's algorithmic
units over that time; a second timed pass replays, per GEMM of the step, a
graph of back-to-back launches of that GEMM alone (``per_gemm_us``).

Under torchrun every rank runs the same per-rank workload on its own GPU (no
data-path collective: the GEMMs of a step are independent problems), so the
scaling is weak and ``value`` counts the bytes of all ranks.

``--impl reference`` times the CPU oracle instead, on the host cores: whole
steps when they fit the time budget (decode: about half a second a step),
else a bounded row sample of each step (the oracle is test infrastructure;
this leg and the ``cpu_baseline`` objects are the only product uses of it).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------- workloads --

def build_workload(name: str, seed: int = 0):
    """List of (kind, problem) making up one step."""
    if name == "decode":
        return [("dense", workloads.dense_problem(m, n, k, seed=seed + i))
                for i, (m, n, k) in enumerate(workloads.DECODE_SHAPES)]
    if name == "smoke":
        m, n, k = workloads.SMOKE_SHAPE
        return [("dense", workloads.dense_problem(m, n, k, seed=seed))]
    if name == "prefill":
        return [("dense", workloads.dense_problem(m, n, k, seed=seed + i))
                for i, (m, n, k) in enumerate(workloads.PREFILL_SHAPES)]
    if name == "contiguous":
        return [("contiguous", workloads.contiguous_problem(**workloads.CONTIGUOUS_MOE, seed=seed))]
    if name == "masked":
        return [("masked", workloads.masked_problem(**workloads.MASKED_MOE, seed=seed))]
    if name == "masked-decode":
        return [("masked", workloads.masked_problem(**workloads.MASKED_DECODE_MOE, seed=seed))]
    if name == "k-grouped":
        return [("k_grouped", workloads.k_grouped_problem(**workloads.K_GROUPED_MOE, seed=seed))]
    if name == "bf16-decode":
        return [("bf16_dense", workloads.bf16_dense_problem(m, n, k, seed=seed + i))
                for i, (m, n, k) in enumerate(workloads.DECODE_SHAPES)]
    if name == "bf16-prefill":
        return [("bf16_dense", workloads.bf16_dense_problem(m, n, k, seed=seed + i))
                for i, (m, n, k) in enumerate(workloads.PREFILL_SHAPES)]
    raise ValueError(name)


def is_bf16(name: str) -> bool:
    return name.startswith("bf16-")


def workload_meta(name: str):
    """(metric, unit, bound) for a workload."""
    if name in ("decode", "smoke"):
        return "FP8 GEMM HBM bandwidth (M<=128)", "GB/s", "hbm"
    if name == "bf16-decode":
        return "BF16 GEMM HBM bandwidth (M<=128)", "GB/s", "hbm"
    if name == "bf16-prefill":
        return "BF16 GEMM TFLOPS", "TFLOP/s", "tensor"
    return "FP8 GEMM TFLOPS", "TFLOP/s", "tensor"


def step_units(items, unit: str) -> float:
    """Algorithmic bytes (GB/s metric) or FLOPs (TFLOP/s metric) of one step."""
    if unit == "GB/s":
        return float(sum(p.bytes() for _, p in items))
    return float(sum(p.flops() for _, p in items))


def scale_units(x: float, unit: str, seconds: float) -> float:
    return x / seconds / (1e9 if unit == "GB/s" else 1e12)


SPEC_HBM_GBS = 8000.0     # B200 HBM3e, vendor figure
SPEC_FP8_TFLOPS = 4500.0  # B200 dense E4M3, vendor figure
SPEC_BF16_TFLOPS = 2250.0  # B200 dense BF16, vendor figure


def roofline_terms(items, ms: float, hbm_gbs: float, fp8_tflops: float,
                   spec_tflops: float = SPEC_FP8_TFLOPS) -> dict:
    """Roofline of one step: every GEMM's time bound is the larger of its
    FLOPs at the tensor peak of its operand type (``fp8_tflops``; the BF16
    peak for BF16 operands) and its algorithmic bytes at the HBM bandwidth;
    the step's bound is the sum.  ``bound`` names the term that dominates."""
    def t_roof(hbm, fp8):
        return sum(max(p.flops() / (fp8 * 1e12), p.bytes() / (hbm * 1e9)) for _, p in items)
    t_flop = sum(p.flops() for _, p in items) / (fp8_tflops * 1e12)
    t_byte = sum(p.bytes() for _, p in items) / (hbm_gbs * 1e9)
    t = t_roof(hbm_gbs, fp8_tflops)
    return {"bound": "tensor" if t_flop >= t_byte else "hbm", "t_roof_s": t,
            "frac_time": t / (ms / 1e3),
            "frac_time_spec": t_roof(SPEC_HBM_GBS, spec_tflops) / (ms / 1e3)}


# --------------------------------------------------------------- helpers --

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except OSError:
        return dict(PEAKS_FALLBACK), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "moe_grouped_gemm_09_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def profile_name(workload: str) -> str:
    """Stem of a workload's ncu summaries under ``profiles/``."""
    if is_bf16(workload):
        return "bf16_gemm_" + workload[len("bf16-"):]
    return "fp8_gemm_" + workload


def profiled_traffic(workload: str):
    """DRAM bytes per launch of the dominant kernel, from the committed ncu
    summary ``profiles/<stem>_traffic.md`` (its lines
    ``traffic_bytes_per_launch:`` and ``kernel_source_hash:``), or None if the
    summary is absent or was taken on other kernel sources."""
    path = os.path.join(ROOT, "profiles", f"{profile_name(workload)}_traffic.md")
    rec = {}
    try:
        with open(path) as f:
            for line in f:
                if ":" in line and not line.startswith((" ", "#", "|")):
                    k, v = line.split(":", 1)
                    rec[k.strip().strip("`")] = v.strip().strip("`")
    except OSError:
        return None
    if rec.get("kernel_source_hash") != kernel_source_hash():
        return None
    try:
        return int(float(rec["traffic_bytes_per_launch"]))
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except OSError:
            self.proc = None
        time.sleep(0.2)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        idle = 0
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                active = int(parts[3], 16)
            except ValueError:
                active = 0
            if active & 0x1:  # the GPU was idle at this sample (before the work started)
                idle += 1
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for name, val in zip(names, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0,
                    "idle_samples": idle}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "idle_samples": idle}


# ------------------------------------------------------------ rank logic --

def reduce_max(x: float, world: int, device) -> float:
    """Maximum of a per-rank value over all ranks (the slowest rank's time)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(units_per_step: float, world: int, ms_per_step: float, unit: str) -> float:
    """Throughput of the whole job: every rank processes units_per_step per
    step (weak scaling), all ranks finish within the slowest rank's time."""
    return scale_units(units_per_step * world, unit, ms_per_step / 1e3)


# ---------------------------------------------------------------- GPU arm --

def fp8_peak(peaks: dict, sustained: bool = False):
    """Dense E4M3 tensor peak (TFLOP/s) and where it comes from: the measured
    figure of ``profiles/fp8_peak.md`` (a large FP8 library GEMM timed on this
    pool's B200s, as a burst or back to back for seconds under the power cap;
    ``--measure-fp8-peak`` writes both), else 2 x the measured BF16 figure
    (the nominal 4.5 : 2.25 FP8 : BF16 ratio)."""
    path = os.path.join(ROOT, "profiles", "fp8_peak.md")
    key = "fp8_tflops_sustained:" if sustained else "fp8_tflops:"
    try:
        with open(path) as f:
            for line in f:
                if line.startswith(key):
                    return (float(line.split(":", 1)[1].strip()),
                            f"measured (fp8_peak.md, cuBLASLt E4M3{', sustained' if sustained else ''})")
    except (OSError, ValueError):
        pass
    bf16 = float(peaks.get("bf16_tflops_sustained" if sustained else "bf16_tflops",
                           PEAKS_FALLBACK["bf16_tflops"]))
    return 2.0 * bf16, "2 x bf16_tflops (nominal FP8:BF16 ratio)"


class GpuContext:
    """Device, stream and rank plumbing shared by the timed workloads."""

    def __init__(self):
        import torch
        import torch.distributed as dist
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        if self.world > 1:
            torch.cuda.set_device(local_rank)
            dist.init_process_group("nccl", device_id=torch.device("cuda", local_rank),
                                    timeout=__import__("datetime").timedelta(seconds=120))
        self.dev = torch.device("cuda", local_rank if self.world > 1 else torch.cuda.current_device())
        torch.cuda.set_device(self.dev)
        self.stream = torch.cuda.Stream(device=self.dev)

    def barrier(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()

    def max_over_ranks(self, x: float) -> float:
        return reduce_max(x, self.world, self.dev)


def _host_tensor(x):
    import torch
    # BF16 operands arrive as uint16 bit patterns
    if x.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x))


def _operands(p):
    names = ("a", "sfa", "b", "sfb") if hasattr(p, "sfa") else ("a", "b")
    return {k: getattr(p, k) for k in names}


def gemm_launches(kind: str, p) -> int:
    """Kernel launches one GEMM call makes: 1, plus the tail launches of a
    dense call whose last wave of tiles is split off (the library's own plan,
    read through dg_query_config)."""
    if kind not in ("dense", "bf16_dense"):
        return 1
    import moe_grouped_gemm_09_b200 as dg
    k_bytes = p.K * (2 if kind == "bf16_dense" else 1)
    return 1 + dg.query_config(dg.KIND_DENSE, p.M, p.N, k_bytes)["tail_launches"]


def step_launches(items) -> int:
    return sum(gemm_launches(k, p) for k, p in items)


def _launcher(dg, items, sets, outs):
    def launch_one(j, r):
        (kind, p), t, d = items[j], sets[r][j], outs[j]
        if kind == "dense":
            dg.fp8_gemm_nt(t["a"], t["sfa"], t["b"], t["sfb"], d)
        elif kind == "bf16_dense":
            dg.bf16_gemm_nt(t["a"], t["b"], d)
        elif kind == "contiguous":
            dg.m_grouped_fp8_gemm_nt_contiguous(t["a"], t["sfa"], t["b"], t["sfb"],
                                                t["m_indices"], d)
        elif kind == "k_grouped":
            dg.k_grouped_fp8_gemm_tn_contiguous(t["a"], t["sfa"], t["b"], t["sfb"], t["ks"], d=d)
        else:
            dg.m_grouped_fp8_gemm_nt_masked(t["a"], t["sfa"], t["b"], t["sfb"],
                                            t["masked_m"], p.expected_m, d)
    return launch_one


def time_workload(ctx: GpuContext, name: str, args, steps: int, per_gemm: bool, e2e: bool,
                  rotations: int = 0) -> dict:
    """Times ``steps`` steps of one workload (inputs resident in HBM, rotated
    over more than 3 x L2, one CUDA graph per rotation cycle, CUDA events on
    the launching stream, max over ranks); optionally the per-GEMM graphs and
    the end-to-end pass through the public call with host buffers."""
    import torch
    import moe_grouped_gemm_09_b200 as dg

    dev, stream = ctx.dev, ctx.stream
    items = build_workload(name, seed=args.seed)
    # dense workloads: B is the weights, so the weight preload applies
    dense = all(k in ("dense", "bf16_dense") for k, _ in items)
    preload = args.weight_preload == "on" and dense
    dg.set_weight_preload(preload)
    metric, unit, _ = workload_meta(name)
    set_bytes = sum(p.a.nbytes + p.b.nbytes + getattr(p, "sfa", p.a[:0]).nbytes
                    + getattr(p, "sfb", p.a[:0]).nbytes for _, p in items)
    R = max(2, math.ceil(3 * L2_BYTES / max(set_bytes, 1)))
    if name in ("prefill", "contiguous", "masked", "masked-decode", "k-grouped", "bf16-prefill"):
        R = max(2, min(R, 4))
    if rotations > 0:
        R = rotations
    flush_note = f"inputs rotated over {R} copies ({R * set_bytes / 2**20:.0f} MiB"
    flush_note += " > 3x L2)" if R * set_bytes > 3 * L2_BYTES else ", not above 3x L2)"

    sets = []
    for r in range(R):
        one = []
        for kind, p in items:
            t = {k: _host_tensor(v).to(dev) for k, v in _operands(p).items()}
            if kind == "contiguous":
                t["m_indices"] = _host_tensor(p.m_indices).to(dev)
            if kind == "masked":
                t["masked_m"] = _host_tensor(p.masked_m).to(dev)
            if kind == "k_grouped":
                t["ks"] = _host_tensor(p.ks).to(dev)
            one.append(t)
        sets.append(one)
    outs = []
    for kind, p in items:
        if kind in ("dense", "bf16_dense"):
            outs.append(torch.empty((p.M, p.N), dtype=torch.bfloat16, device=dev))
        elif kind == "contiguous":
            outs.append(torch.empty((p.M_sum, p.N), dtype=torch.bfloat16, device=dev))
        elif kind == "k_grouped":
            outs.append(torch.empty((p.G, p.M, p.N), dtype=torch.float32, device=dev))
        else:
            outs.append(torch.empty((p.G, p.max_m, p.N), dtype=torch.bfloat16, device=dev))
    launch_one = _launcher(dg, items, sets, outs)

    def launch_step(r):
        for j in range(len(items)):
            launch_one(j, r)

    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        for i in range(args.warmup):          # eager warm-up (also the device set-up)
            launch_step(i % R)
    torch.cuda.synchronize(dev)
    if dg.get_last_device_error() != 0:
        raise RuntimeError(f"{name}: device error during warm-up")

    # One graph holds a whole rotation cycle (steps on sets 0..R-1, so that
    # consecutive launches overlap through programmatic dependent launch
    # across step boundaries too), one the first `steps mod R` steps of a cycle.
    def capture(n_steps):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for r in range(n_steps):
                launch_step(r)
        return g

    cycle = capture(R)
    rem = steps % R
    tail = capture(rem) if rem else None
    with torch.cuda.stream(stream):
        cycle.replay()
        cycle.replay()
    torch.cuda.synchronize(dev)

    # ---- timed region: exactly `steps` steps ----
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ctx.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clocks:
        with torch.cuda.stream(stream):
            start.record(stream)
            for _ in range(steps // R):
                cycle.replay()
            if tail is not None:
                tail.replay()
            end.record(stream)
        torch.cuda.synchronize(dev)
    ctx.barrier()
    ms = ctx.max_over_ranks(start.elapsed_time(end) / steps)
    if dg.get_last_device_error() != 0:
        raise RuntimeError(f"{name}: device error during the timed steps")

    # the dense workloads: the same steps with the weight preload switched the
    # other way, for comparison (B is the weights, written by no kernel)
    ms_alt = None
    if dense:
        dg.set_weight_preload(not preload)
        plain = capture(R)
        plain_tail = capture(rem) if rem else None
        with torch.cuda.stream(stream):
            plain.replay()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ctx.barrier()
        torch.cuda.synchronize(dev)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(steps // R):
                plain.replay()
            if plain_tail is not None:
                plain_tail.replay()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        ctx.barrier()
        ms_alt = ctx.max_over_ranks(e0.elapsed_time(e1) / steps)
        dg.set_weight_preload(preload)
        del plain, plain_tail


    # ---- per GEMM (second timed pass): R back-to-back launches of one shape ----
    kernel_ms = []
    if per_gemm:
        for j in range(len(items)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for r in range(R):
                    launch_one(j, r)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                g.replay()
                e0.record(stream)
                for _ in range(args.per_gemm_reps):
                    g.replay()
                e1.record(stream)
            torch.cuda.synchronize(dev)
            kernel_ms.append(e0.elapsed_time(e1) / (args.per_gemm_reps * R))
            del g

    # ---- end to end: host buffers, copies inside the timed region ----
    e2e_res = None
    if e2e:
        pinned = []
        for kind, p in items:
            t = {k: _host_tensor(v).pin_memory() for k, v in _operands(p).items()}
            if kind == "contiguous":
                t["m_indices"] = torch.from_numpy(p.m_indices).pin_memory()
            if kind == "masked":
                t["masked_m"] = torch.from_numpy(p.masked_m).pin_memory()
            if kind == "k_grouped":
                t["ks"] = torch.from_numpy(p.ks).pin_memory()
            pinned.append(t)
        host_out = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
        h2d = sum(v.numel() * v.element_size() for t in pinned for v in t.values())
        d2h = sum(o.numel() * o.element_size() for o in outs)
        e2e_steps = max(3, min(steps, args.e2e_steps))

        def e2e_step():
            for t_h, t_d in zip(pinned, sets[0]):
                for k in t_h:
                    t_d[k].copy_(t_h[k], non_blocking=True)
            launch_step(0)
            for o_h, o_d in zip(host_out, outs):
                o_h.copy_(o_d, non_blocking=True)

        with torch.cuda.stream(stream):
            for _ in range(2):
                e2e_step()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ctx.barrier()
        torch.cuda.synchronize(dev)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(e2e_steps):
                e2e_step()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        ctx.barrier()
        e2e_ms = ctx.max_over_ranks(e0.elapsed_time(e1) / e2e_steps)
        e2e_res = {"value": round(whole_job_value(step_units(items, unit), ctx.world, e2e_ms, unit), 3),
                   "unit": unit, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}

    # ---- sustained pass: the same graphs back to back for `sustained_s`,
    # long enough for the power cap to act; its own clock samples ----
    sustained = None
    if args.sustained_s > 0:
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            c0.record(stream)
            cycle.replay()
            c1.record(stream)
        torch.cuda.synchronize(dev)
        cycle_s = max(c0.elapsed_time(c1) / 1e3, 1e-6)
        batch = max(1, int(0.05 / cycle_s))                    # ~50 ms per host sync
        n_batches = max(1, int(math.ceil(args.sustained_s / (batch * cycle_s))))
        ctx.barrier()
        torch.cuda.synchronize(dev)
        with ClockSampler(dev.index) as s_clocks:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                e0.record(stream)
            for _ in range(n_batches):
                with torch.cuda.stream(stream):
                    for _ in range(batch):
                        cycle.replay()
                torch.cuda.synchronize(dev)
            with torch.cuda.stream(stream):
                e1.record(stream)
            torch.cuda.synchronize(dev)
        ctx.barrier()
        n_steps = n_batches * batch * R
        sustained = {"ms": ctx.max_over_ranks(e0.elapsed_time(e1) / n_steps), "steps": n_steps,
                     "clocks": s_clocks.summary()}
        if dg.get_last_device_error() != 0:
            raise RuntimeError(f"{name}: device error during the sustained pass")
    del cycle, tail

    dg.set_weight_preload(False)
    return {"items": items, "ms": ms, "R": R, "flush_note": flush_note, "kernel_ms": kernel_ms,
            "clocks": clocks.summary(), "e2e": e2e_res, "metric": metric, "unit": unit,
            "preload": preload, "ms_alt": ms_alt, "sustained": sustained}


# seconds of timed steps beyond which the sustained tensor peak applies
LONG_REGION_S = 0.2


def sustained_record(name: str, t: dict, world: int, unit: str, bound: str, hbm_peak: float,
                     peaks: dict) -> dict:
    """The sustained pass: the same graphs back to back for seconds (the power
    cap acts), its rate, clocks, and fraction of the sustained peak (HBM: the
    same copy bandwidth; tensor: the sustained library GEMM rate)."""
    items, su = t["items"], t["sustained"]
    if bound == "hbm":
        peak, src, r_unit = hbm_peak, "measured (hbm_gbs copy)", "GB/s"
    elif is_bf16(name):
        peak = float(peaks.get("bf16_tflops_sustained", PEAKS_FALLBACK["bf16_tflops"]))
        src, r_unit = "measured (bf16_tflops_sustained)", "TFLOP/s"
    else:
        (peak, src), r_unit = fp8_peak(peaks, sustained=True), "TFLOP/s"
    achieved = scale_units(step_units(items, r_unit), r_unit, su["ms"] / 1e3)
    return {"value": round(whole_job_value(step_units(items, unit), world, su["ms"], unit), 3),
            "ms_per_step": round(su["ms"], 6), "steps": su["steps"],
            "roofline": {"achieved": round(achieved, 3), "peak": round(peak, 1), "unit": r_unit,
                         "frac": round(achieved / peak, 4), "peak_source": src},
            "clocks": su["clocks"]}


def workload_record(name: str, t: dict, world: int, steps: int, warmup: int) -> dict:
    """The JSON record of one timed workload: metric, value, roofline."""
    items, ms, unit = t["items"], t["ms"], t["unit"]
    peaks, peak_kind = load_peaks()
    hbm_peak = float(peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"]))
    bf16 = is_bf16(name)
    # A timed region long enough for the power cap to act (the default 2000
    # steps of a compute-bound workload last seconds) is held against the
    # sustained tensor peak; a short one (the usual 20 steps) against the burst.
    long_region = ms * steps / 1e3 > LONG_REGION_S
    if bf16:
        key = "bf16_tflops_sustained" if long_region else "bf16_tflops"
        tensor_peak = float(peaks.get(key, PEAKS_FALLBACK["bf16_tflops"]))
        tensor_src = f"{peak_kind} ({key})"
    else:
        tensor_peak, tensor_src = fp8_peak(peaks, sustained=long_region)
    roof = roofline_terms(items, ms, hbm_peak, tensor_peak,
                          SPEC_BF16_TFLOPS if bf16 else SPEC_FP8_TFLOPS)
    bound = roof["bound"]
    r_unit = "GB/s" if bound == "hbm" else "TFLOP/s"
    peak = hbm_peak if bound == "hbm" else tensor_peak
    achieved = scale_units(step_units(items, r_unit), r_unit, ms / 1e3)
    launches_per_step = step_launches(items)
    return {
        "metric": t["metric"],
        "value": round(whole_job_value(step_units(items, unit), world, ms, unit), 3),
        "unit": unit,
        "ms_per_step": round(ms, 6),
        "steps": steps,
        "warmup": warmup,
        "dtype": "bf16" if bf16 else "e4m3",
        "config": {
            "workload": name,
            "gemms": [dict(kind=k, **_shape(p)) for k, p in items],
            "l2": t["flush_note"],
            "graph": f"one CUDA graph per rotation cycle of {t['R']} steps",
            "weight_preload": t["preload"],
        },
        "gpu_launches": int(steps * launches_per_step),
        "roofline": {
            "bound": bound,
            "achieved": round(achieved, 3),
            "peak": round(peak, 1),
            "unit": r_unit,
            "frac": round(achieved / peak, 4),
            "traffic": profiled_traffic(name),
            "peak_source": f"{peak_kind} (hbm_gbs copy)" if bound == "hbm" else tensor_src,
            "tensor_peak_tflops": round(tensor_peak, 1),
            "roofline_time_us": round(roof["t_roof_s"] * 1e6, 3),
            "frac_time": round(roof["frac_time"], 4),
            "frac_time_spec": round(roof["frac_time_spec"], 4),
            "launch_avg_us": round(ms * 1e3 / launches_per_step, 3),
            "per_gemm_us": [round(x * 1e3, 3) for x in t["kernel_ms"]],
        },
        "clocks": t["clocks"],
        **({"sustained": sustained_record(name, t, world, unit, bound, hbm_peak, peaks)}
           if t.get("sustained") else {}),
        **({("value_without_weight_preload" if t["preload"] else "value_with_weight_preload"):
            round(whole_job_value(step_units(items, unit), world, t["ms_alt"], unit), 3)}
           if t["ms_alt"] else {}),
    }


EXTRA_WORKLOADS = ("smoke", "prefill", "contiguous", "masked", "masked-decode", "k-grouped",
                   "bf16-decode", "bf16-prefill")


def run_gpu(args):
    import torch

    ctx = GpuContext()
    main = time_workload(ctx, args.workload, args, args.steps, per_gemm=True, e2e=True,
                         rotations=args.rotations)
    rec = workload_record(args.workload, main, ctx.world, args.steps, args.warmup)
    res = {
        "metric": rec["metric"],
        "value": rec["value"],
        "unit": rec["unit"],
        "n_gpus": ctx.world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": rec["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": rec["dtype"],
        "data": "synthetic",
        "config": dict(rec["config"], parallelism=(f"replicas x{ctx.world}" if ctx.world > 1
                                                   else "single GPU")),
        "e2e": main["e2e"],
        "gpu_launches": rec["gpu_launches"],
        "roofline": rec["roofline"],
        "clocks": rec["clocks"],
    }
    for key in ("value_without_weight_preload", "value_with_weight_preload", "sustained"):
        if key in rec:
            res[key] = rec[key]
    cpu_ok = ctx.rank == 0 and ctx.world == 1 and not args.no_cpu_baseline
    if cpu_ok:
        res["cpu_baseline"] = run_oracle_sample(main["items"], main["unit"],
                                                budget_s=args.cpu_budget_s)
    del main
    torch.cuda.empty_cache()

    # The other configurations of the same metric, timed the same way in the
    # same process (the headline `value` stays the workload above).
    extras = [w for w in (args.extra_workloads.split(",") if args.extra_workloads else [])
              if w and w != args.workload]
    if extras:
        res["workloads"] = {}
        for w in extras:
            t = time_workload(ctx, w, args, args.steps, per_gemm=(w == "prefill"), e2e=False,
                              rotations=args.rotations)
            r = workload_record(w, t, ctx.world, args.steps, args.warmup)
            if cpu_ok:
                r["cpu_baseline"] = run_oracle_sample(t["items"], t["unit"],
                                                      budget_s=args.extra_cpu_budget_s)
            res["workloads"][w] = r
            del t
            torch.cuda.empty_cache()
    if ctx.rank == 0:
        print(json.dumps(res), flush=True)
    if ctx.world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def measure_fp8_peak(args):
    """Dense E4M3 peak of this GPU from the vendor library: torch._scaled_mm
    (cuBLASLt) on an 8192^3 E4M3 x E4M3 GEMM with FP32 per-tensor scales and
    BF16 output, best of 20 CUDA-event-timed launches (burst) and the mean
    over a 4 s back-to-back loop (sustained)."""
    import torch
    dev = torch.device("cuda", 0)
    n = args.peak_size
    a = torch.randn((n, n), device=dev).to(torch.float8_e4m3fn)
    b = torch.randn((n, n), device=dev).to(torch.float8_e4m3fn)
    one = torch.ones((), device=dev)

    def mm():
        return torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)

    for _ in range(5):
        mm()
    torch.cuda.synchronize()
    best = 1e30
    for _ in range(20):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        mm()
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    flop = 2.0 * n ** 3
    with ClockSampler(0) as clocks:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        iters = 0
        t_end = time.perf_counter() + 4.0
        while time.perf_counter() < t_end:
            for _ in range(20):
                mm()
            iters += 20
            torch.cuda.synchronize()
        e1.record()
        torch.cuda.synchronize()
    sustained_ms = e0.elapsed_time(e1) / iters
    print(json.dumps({"fp8_tflops": round(flop / best / 1e9, 1),
                      "fp8_tflops_sustained": round(flop / sustained_ms / 1e9, 1),
                      "shape": [n, n, n], "how": "torch._scaled_mm E4M3 x E4M3 -> BF16, "
                      "per-tensor FP32 scales; best of 20 launches / mean of a 4 s loop",
                      "clocks": clocks.summary(), "gpu": torch.cuda.get_device_name(0)}),
          flush=True)


def _shape(p):
    if isinstance(p, (workloads.DenseProblem, workloads.Bf16DenseProblem)):
        return {"M": p.M, "N": p.N, "K": p.K}
    if isinstance(p, workloads.ContiguousProblem):
        return {"M_sum": p.M_sum, "N": p.N, "K": p.K, "G": p.G, "valid_rows": p.valid_rows()}
    if isinstance(p, workloads.KGroupedProblem):
        return {"G": p.G, "M": p.M, "N": p.N, "K_sum": p.K_sum, "valid_tokens": p.valid_rows(),
                "out": "fp32"}
    return {"G": p.G, "max_m": p.max_m, "N": p.N, "K": p.K, "valid_rows": p.valid_rows(),
            "expected_m": p.expected_m}


# ------------------------------------------------------ CPU oracle timing --

def _row_units(items, unit):
    """Total rows per GEMM, for scaling a row sample up to the full step."""
    out = []
    for kind, p in items:
        if kind in ("dense", "bf16_dense", "k_grouped"):
            out.append(p.M)
        else:
            out.append(p.valid_rows())
    return out


def _oracle_rows(o, kind, p, rows: np.ndarray):
    if kind == "dense":
        o.gemm_nt(p.a[rows], p.sfa[rows], p.b, p.sfb, want_acc=False)
    elif kind == "bf16_dense":
        o.bf16_gemm_nt(p.a[rows], p.b, want_acc=False)
    elif kind == "contiguous":
        valid = np.nonzero(p.m_indices >= 0)[0][rows]
        o.grouped_contiguous(p.a[valid], p.sfa[valid], p.b, p.sfb, p.m_indices[valid])
    elif kind == "k_grouped":
        # output rows m of every group: the columns m of A and their scales
        o.k_grouped_tn(p.a[:, rows], p.sfa[rows], p.b, p.sfb, p.ks)
    else:
        pairs = [(g, m) for g in range(p.G) for m in range(min(max(int(p.masked_m[g]), 0), p.max_m))]
        sel = sorted(pairs[i] for i in rows)
        # one oracle call per run of consecutive rows of one group (the oracle
        # spreads the rows of a call over its threads)
        i = 0
        while i < len(sel):
            g, m0 = sel[i]
            j = i + 1
            while j < len(sel) and sel[j] == (g, m0 + (j - i)):
                j += 1
            o.gemm_nt(p.a[g, m0:m0 + (j - i)], p.sfa[g, m0:m0 + (j - i)], p.b[g], p.sfb[g],
                      want_acc=False)
            i = j


def run_oracle_sample(items, unit, budget_s: float):
    """Time the oracle on a bounded row sample of the step and scale to the
    full step by rows (its cost is linear in output rows)."""
    import oracle
    o = oracle.default()
    rows_total = _row_units(items, unit)
    units = step_units(items, unit)
    # rows per GEMM: grow until the sample takes about budget_s
    frac = 1.0 / 64
    while True:
        t0 = time.perf_counter()
        done_frac = []
        for (kind, p), tot in zip(items, rows_total):
            n = max(1, int(round(tot * frac)))
            _oracle_rows(o, kind, p, np.arange(n))
            done_frac.append(n / tot)
        dt = time.perf_counter() - t0
        if dt > budget_s / 4 or frac >= 1.0:
            break
        frac = min(1.0, frac * max(2.0, budget_s / 2 / max(dt, 1e-3)))
    if frac >= 1.0 and dt < budget_s / 2:
        # the whole step is cheap: time whole steps back to back instead
        reps = max(2, int(budget_s / 2 / max(dt, 1e-3)))
        t0 = time.perf_counter()
        for _ in range(reps):
            for kind, p in items:
                _oracle_rows(o, kind, p, np.arange(_row_units([(kind, p)], unit)[0]))
        dt = time.perf_counter() - t0
        full_s = dt / reps
        sample = f"{reps} whole steps back to back ({dt:.1f} s)"
    else:
        full_s = dt / (sum(done_frac) / len(done_frac))
        lo, hi = 100 * min(done_frac), 100 * max(done_frac)
        share = f"{lo:.2f}%" if f"{lo:.2f}" == f"{hi:.2f}" else f"{lo:.2f}%..{hi:.2f}%"
        sample = (f"first {share} of the output rows of every GEMM of one step ({dt:.1f} s), "
                  f"scaled to the full step by rows")
    return {"value": round(scale_units(units, unit, full_s), 4), "unit": unit,
            "cores": o.num_threads(), "kind": "oracle", "sample": sample}


def run_reference(args):
    """The oracle as the reference arm: K timed steps on the host cores.  A
    step is one whole step of the workload when the oracle finishes one in a
    few seconds (decode: about half a second on 16 threads), else a bounded
    row sample of it (one output row per host thread of one GEMM, round robin
    over the GEMMs) scaled to the full step by rows."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    o = oracle.default()
    items = build_workload(args.workload, seed=args.seed)
    metric, unit, _ = workload_meta(args.workload)
    units = step_units(items, unit)
    rows_total = _row_units(items, unit)

    def whole_step():
        for (kind, p), n in zip(items, rows_total):
            _oracle_rows(o, kind, p, np.arange(n))

    # one probe step decides whole steps or a row sample
    t0 = time.perf_counter()
    whole_step()
    probe_s = time.perf_counter() - t0
    whole = probe_s * (args.steps + args.warmup) <= args.reference_budget_s
    if whole:
        for _ in range(max(0, args.warmup - 1)):
            whole_step()
        t0 = time.perf_counter()
        for _ in range(args.steps):
            whole_step()
        dt = time.perf_counter() - t0
        full_s = dt / args.steps
        sample = f"{args.steps} whole steps back to back ({dt:.1f} s)"
    else:
        per = max(1, o.num_threads())
        cursor = [0] * len(items)

        def one_step(i):
            j = i % len(items)
            n = min(per, rows_total[j])
            rows = (cursor[j] + np.arange(n)) % rows_total[j]
            cursor[j] = int((cursor[j] + n) % rows_total[j])
            _oracle_rows(o, items[j][0], items[j][1], rows)
            return n / rows_total[j] / len(items)

        for i in range(args.warmup):
            one_step(i)
        full_equiv = 0.0
        t0 = time.perf_counter()
        for i in range(args.steps):
            full_equiv += one_step(i)
        dt = time.perf_counter() - t0
        full_s = dt / full_equiv
        sample = (f"{args.steps} timed steps of {per} output rows each (one GEMM per step, "
                  f"round robin), {dt:.1f} s, scaled to full steps by rows")
    value = scale_units(units, unit, full_s)
    res = {
        "impl": "reference",
        "metric": metric, "value": round(value, 4), "unit": unit, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * full_s, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "gemms": [dict(kind=k, **_shape(p)) for k, p in items]},
        "cpu_baseline": {"value": round(value, 4), "unit": unit, "cores": o.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": unit, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(res), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="decode",
                    choices=("decode", "smoke", "prefill", "contiguous", "masked", "masked-decode",
                             "k-grouped", "bf16-decode", "bf16-prefill"))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--per-gemm-reps", type=int, default=20,
                    help="replays of each single-GEMM graph behind per_gemm_us")
    ap.add_argument("--cpu-budget-s", type=float, default=20.0)
    ap.add_argument("--extra-cpu-budget-s", type=float, default=4.0,
                    help="oracle time per extra workload's cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--extra-workloads", default=",".join(EXTRA_WORKLOADS),
                    help="comma-separated workloads timed after the main one and reported "
                         "under 'workloads' ('' for none)")
    ap.add_argument("--rotations", type=int, default=0,
                    help="input copies rotated between steps (0: enough to exceed 3x L2)")
    ap.add_argument("--reference-budget-s", type=float, default=120.0,
                    help="reference arm: whole oracle steps if they fit in this time")
    ap.add_argument("--sustained-s", type=float, default=2.0,
                    help="after the timed steps, replay the same graphs back to back for this "
                         "long and report the sustained rate and its clocks (0: skip)")
    ap.add_argument("--weight-preload", choices=("on", "off"), default="off",
                    help="dense workloads: let each GEMM load B (the weights) before waiting "
                         "on the previous kernel; the line also reports the value with the "
                         "other setting")
    ap.add_argument("--measure-fp8-peak", action="store_true",
                    help="time the vendor library's dense E4M3 GEMM and print its TFLOP/s")
    ap.add_argument("--peak-size", type=int, default=8192)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.measure_fp8_peak:
        measure_fp8_peak(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
