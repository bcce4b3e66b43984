#!/usr/bin/env python
"""Benchmark of the FastVim SSM layer (pooled selective scan) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config NAME]

One step = one fastvim_ssm_forward call over the whole batch of the workload (pool ->
projections -> scans -> repeat/skip/gate), inputs resident in HBM.  The default workload is the
FastVim-T layer at 2048 px: B = 128, a 128 x 128 token grid, E = 384, N = 16, R = 12, column
pooling, forward + backward scans, fp32.  Its x, z and y take 9.7 GB, far above the 126 MB L2,
so no L2 flush is needed between steps (workloads under twice the L2 size get one before every
step, outside the step's timed span).

Under torchrun (N > 1) every rank runs its own batch of B distinct images on its own GPU
(images rank*B .. rank*B + B - 1 of the seeded stream; the images are independent, so there is
no data-path collective: weak scaling); the step time is the maximum over ranks of each rank's
CUDA-event time.  Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle on the host cores instead (rank 0 only), on a bounded
sample of images of the same workload per step.

--grad times a training step of the layer instead: the forward call (keeping the scan states,
FV_FLAG_KEEP_STATES, unless --recompute-states) and then the gradient call (fastvim_ssm_backward:
dx, dz and the parameter gradients for a seeded upstream gradient dy) over the same batch, and
prints its own line for that.
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

METRIC = "SSM-layer grid tokens/s at 2048² FastVim-T (fp32, B=128); HBM GB/s vs peak"
UNIT = "grid tokens/s"
FALLBACK_HBM_GBS = 6650.0
REFERENCE_BUDGET_S = 150.0
HEADLINE_NAME = "fastvim_t_2048"

L2_BYTES = 126 * 1024 * 1024
# Special-function (MUFU) lanes per SM per clock on sm_100: 4 per SM sub-partition.
MUFU_PER_SM_CLK = 16
# fp32 FMA lanes per SM per clock on sm_100 (4 sub-partitions x 32); 2 flops each.
FFMA_PER_SM_CLK = 128


def kernel_work(name: str, cfg, pool_axis: int):
    """(bound, algorithmic amount per step) of kernel `name` on workload `cfg` (all its launches in
    one step; a staged layer launches a kernel once per chunk of images):
    bytes for the streaming kernels (what the step must move at minimum), exp2 evaluations for
    the scans (one per state, step, channel and direction), fp32 flops for the x_proj GEMM, the
    step sizes written for dt_proj (a K = R tensor-core GEMM whose output is the cost), None for the
    rest."""
    tok = cfg.tokens_per_call()                       # grid tokens, or kept tokens when masked
    row = 4 * cfg.E                                   # one fp32 token row
    T = cfg.h if pool_axis == 0 else cfg.w
    if name in ("pool_dense_kernel", "mask_pool_kernel", "pool_conv_kernel"):
        return "hbm", row * tok                       # read x (with the Conv1D: its input)
    if name in ("epilogue_dense_kernel", "mask_epilogue_kernel", "ln_epilogue_kernel", "ln_epilogue_reg_kernel",
                "fused_layer_kernel", "epilogue_conv_kernel"):
        return "hbm", 3 * row * tok                   # read x and z, write y (the fused launch: the layer)
    if name == "scan_seq_kernel":
        return "alu", cfg.B * T * cfg.E * cfg.N * cfg.nd
    if name == "proj_gemm_kernel":
        return "fma", 2 * cfg.B * T * cfg.E * cfg.nd * (cfg.R + 2 * cfg.N)
    if name == "dt_proj_kernel":
        return "hbm", 4 * cfg.B * T * cfg.E * cfg.nd          # Delta written (tensor-core GEMM, K = R)
    # the gradient's kernels
    if name in ("bwd_gate_dense_kernel", "bwd_gate_masked_kernel", "bwd_ln_gate_kernel", "bwd_ln_gate_reg_kernel"):
        return "hbm", 5 * row * tok                   # read x, z, dy; write dz and dx
    if name == "bwd_pool_dense_kernel":
        return "hbm", 2 * row * tok                   # dx read and written back (+ the pooled share)
    if name == "bwd_pool_masked_kernel":
        return "hbm", 2 * row * tok
    if name == "bwd_scan_kernel":
        return "alu", cfg.B * T * cfg.E * cfg.N * cfg.nd   # one exp2 per state and step (the minimum)
    if name == "bwd_reduce_kernel:du":                # the 64-channel tiles' du shares read, du written
        return "hbm", 4 * (-(-cfg.E // 64) + 1) * cfg.nd * cfg.B * T * (cfg.R + 2 * cfg.N)
    if name == "bwd_reduce_kernel:params":            # per-image partials of dA_log, dW_dt, db_dt read
        return "hbm", 4 * cfg.B * cfg.nd * cfg.E * (cfg.N + cfg.R + 1)
    if name in ("bwd_dwx_kernel", "bwd_dxbar_kernel"):   # dW_x = du^T xbar, dxbar = du W_x
        return "fma", 2 * cfg.B * T * cfg.E * (cfg.R + 2 * cfg.N) * cfg.nd
    return None, 0


def ffma_peak_tflops(device_index: int, sm_max_mhz) -> float:
    import torch
    sms = torch.cuda.get_device_properties(device_index).multi_processor_count
    return sms * FFMA_PER_SM_CLK * 2 * float(sm_max_mhz or 1965) * 1e6 / 1e12


def mufu_peak_gops(device_index: int, sm_max_mhz) -> float:
    import torch
    sms = torch.cuda.get_device_properties(device_index).multi_processor_count
    return sms * MUFU_PER_SM_CLK * float(sm_max_mhz or 1965) * 1e6 / 1e9


def parse(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="fastvim_t_2048")
    ap.add_argument("--pool-axis", type=int, default=None, help="override the workload's pool axis")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the batch (small cases for profiler captures; not a benchmark line)")
    ap.add_argument("--path", choices=["auto", "staged", "fused"], default="auto",
                    help="implementation of the layer (auto picks the fused launch for this workload)")
    ap.add_argument("--ln", action="store_true",
                    help="add the post-SSM LayerNorm before the gate (gamma = 1, beta = 0: the usual init)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end (host buffer) leg")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--conv", type=int, default=0, choices=range(0, 5), metavar="TAPS",
                    help="put the block's Conv1D (TAPS taps per direction, SiLU after it) in front of the layer")
    ap.add_argument("--no-configs", action="store_true",
                    help="time only the chosen workload (by default the headline run also times the other "
                         "workloads and reports them under 'configs')")
    ap.add_argument("--grad", action="store_true",
                    help="time a training step: the forward call, then the gradient call on its workspace")
    ap.add_argument("--recompute-states", action="store_true",
                    help="--grad without FV_FLAG_KEEP_STATES: the gradient reruns the recurrences for their "
                         "states instead of reading the ones the forward kept")
    a = ap.parse_args(argv)
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    if a.steps < 1:
        ap.error("--steps must be >= 1")
    return a


def workload_desc(cfg, pool_axis):
    axis = "w (column pooling, T = h)" if pool_axis == 0 else "h (row pooling, T = w)"
    dirs = {1: "forward", 2: "backward", 3: "forward+backward"}[cfg.dir_flags]
    d = {
        "workload": f"{cfg.name}: {cfg.note}",
        "B": cfg.B, "grid": [cfg.h, cfg.w], "E": cfg.E, "N": cfg.N, "R": cfg.R,
        "pool": axis, "scan": dirs,
    }
    if cfg.masked:
        d["kept_tokens_per_sample"] = cfg.K
    return d


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, copy)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (6.65 TB/s earlier pool measurement)"


# Sources each recorded kernel is built from (the traffic record is void once any of them changes).
KERNEL_SOURCES = {
    "fused_layer_kernel": ("fastvim_ssm.cu", "fv_common.cuh", "fv_fused.cuh", "fv_scan.cuh"),
    "bwd_gate_dense_kernel": ("fastvim_ssm.cu", "fv_common.cuh", "fv_kernels.cuh", "fv_backward.cuh"),
    "bwd_pool_dense_kernel": ("fastvim_ssm.cu", "fv_common.cuh", "fv_kernels.cuh", "fv_backward.cuh"),
}


def kernel_source_hash(kernel=None):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "pooled_selective_scan_b200", "csrc")
    names = KERNEL_SOURCES.get(kernel) or [n for n in os.listdir(csrc) if n.endswith((".cu", ".cuh"))]
    for name in sorted(names):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, cfg_name):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if it was taken on the
    current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(p) as f:
            j = json.load(f)
    except Exception:
        return None
    ent = j.get("kernels", {}).get(f"{cfg_name}/{kernel}")
    if not ent or ent.get("kernel_source_hash") != kernel_source_hash(kernel):
        return None
    return ent.get("dram_bytes_per_full_launch")


# ------------------------------------------------------------------------------------------------
# Clock sampling (NVML, read-only) during the timed region.
# ------------------------------------------------------------------------------------------------
class ClockSampler:
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
               0x1: "gpu_idle", 0x10: "sync_boost", 0x100: "display_clock_setting"}

    def __init__(self, torch_device_index, period_s=0.02):
        self.ok = False
        self.samples = []
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml as nv
            import torch
            nv.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(torch_device_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.h = nv.nvmlDeviceGetHandleByUUID(uuid)
            self.nv = nv
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self._reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            self.ok = True
        except Exception as e:  # sampling is best effort; the JSON says when it was unavailable
            self.err = f"{type(e).__name__}: {e}"

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = self._reasons(self.h)
                self.samples.append((mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": getattr(self, "err", "unavailable")}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [m for m, _ in self.samples]
        mask = 0
        for _, r in self.samples:
            mask |= int(r)
        reasons = sorted(n for bit, n in self.REASONS.items() if mask & bit and n != "gpu_idle")
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(mhz), "sm_mhz_min": min(mhz)}


# ------------------------------------------------------------------------------------------------
# Multi-rank plumbing
# ------------------------------------------------------------------------------------------------
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(value: float, device=None) -> float:
    """Max of a per-rank float over the process group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank: int, world: int, max_seconds: float) -> float:
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return units_per_rank * world / max_seconds


# ------------------------------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline of our arm, and the reference arm)
# ------------------------------------------------------------------------------------------------
def oracle_sample(cfg, pool_axis, n_images):
    import oracle
    from pooled_selective_scan_b200 import inputs
    which = list(range(min(n_images, cfg.B)))
    d = inputs.layer_inputs(cfg, which=which)
    oracle.build()

    def step(nthreads):
        oracle.forward(d["x"], d["z"], d["A_log"], d["D"], d["W_x"], d["W_dt"], d["b_dt"], pool_axis,
                       cfg.dir_flags, keep_idx=d.get("keep_idx"), h=cfg.h, w=cfg.w, nthreads=nthreads)
    return which, step


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(cfg, pool_axis, min_seconds=10.0):
    cores = host_cores()
    n_img = min(cfg.B, max(1, cores), 32)
    which, step = oracle_sample(cfg, pool_axis, n_img)
    threads = min(cores, len(which))
    step(threads)  # warm
    t0 = time.perf_counter()
    reps = 0
    while True:
        step(threads)
        reps += 1
        el = time.perf_counter() - t0
        if el * threads >= min_seconds or el >= min_seconds:
            break
    tok = len(which) * (cfg.K if cfg.masked else cfg.h * cfg.w)
    return {"value": tok * reps / el, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{len(which)} images of {cfg.name} x {reps} passes, fp64 C oracle, OpenMP over images "
                      f"({el:.1f} s wall, {el * threads:.1f} core-s)"}


def run_reference(a, cfg, pool_axis):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    cores = host_cores()
    n_img = min(cfg.B, max(1, cores), 16)
    which, step = oracle_sample(cfg, pool_axis, n_img)
    threads = min(cores, len(which))
    # keep the whole run within a few minutes: halve the per-step sample while the first warm-up
    # step says that steps + warm-up would take longer than REFERENCE_BUDGET_S
    while True:
        t0 = time.perf_counter()
        step(threads)
        per_step = time.perf_counter() - t0
        if per_step * (a.steps + a.warmup) <= REFERENCE_BUDGET_S or len(which) == 1:
            break
        which, step = oracle_sample(cfg, pool_axis, max(1, len(which) // 2))
        threads = min(cores, len(which))
    for _ in range(a.warmup - 1):
        step(threads)
    t0 = time.perf_counter()
    for _ in range(a.steps):
        step(threads)
    el = time.perf_counter() - t0
    tok = len(which) * (cfg.K if cfg.masked else cfg.h * cfg.w)
    value = tok * a.steps / el
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": a.gpus,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": 1e3 * el / a.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(workload_desc(cfg, pool_axis), sample_per_step=f"{len(which)} of {cfg.B} images"),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{len(which)} images of {cfg.name} per step, fp64 C oracle, OpenMP over images"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------------------------
# Our arm
# ------------------------------------------------------------------------------------------------
# The other workloads of the method's efficiency study, timed in the same default run after the
# headline (one GPU): (config name, pool axis).  The 224 px layer runs both axes (alternating
# blocks); its inputs fit in L2, so each of its steps starts after an L2 flush.
SECONDARY = (("fastvim_t_224_tiny", 0), ("fastvim_t_224", 0), ("fastvim_t_224", 1), ("fastvim_s_1024", 1),
             ("fastmaskvim_b_1024_mask75", 0))
# Variants timed beside them: (config, pool axis, Conv1D taps, path).  The headline layer with the
# block's Conv1D in front (4 taps per direction, SiLU after it: x is the Conv1D's input, so the
# layer's algorithmic bytes are unchanged), and the small 224 px layer on the single persistent
# launch (the automatic choice takes the staged kernels there).
SECONDARY_VARIANTS = (("fastvim_t_2048", 0, 4, "auto"), ("fastvim_t_224", 0, 0, "fused"))


def summarize_kernels(per_kernel, names, cfg, pool_axis, peak, mufu_peak, fma_peak):
    """Per kernel: launches per step, mean device time per step, share of the step's kernel time,
    and achieved work rate against the bound of kernel_work."""
    total_k = sum(sum(v) for v in per_kernel.values())
    kern = {}
    for n, v in per_kernel.items():
        avg_s = statistics.mean(v) / 1e3
        bound, amount = kernel_work(n, cfg, pool_axis)
        ent = {"launches_per_step": names.count(n), "us_per_step": avg_s * 1e6,
               "share": sum(v) / total_k if total_k > 0 else 0.0, "bound": bound}
        if bound == "hbm":
            ent.update(achieved=amount / avg_s / 1e9, unit="GB/s", frac=amount / avg_s / 1e9 / peak)
        elif bound == "alu":
            ent.update(achieved=amount / avg_s / 1e9, unit="G exp2/s", frac=amount / avg_s / 1e9 / mufu_peak)
        elif bound == "fma":
            ent.update(achieved=amount / avg_s / 1e12, unit="TFLOP/s fp32", frac=amount / avg_s / 1e12 / fma_peak)
        kern[n] = ent
    return kern


def roofline_of(kern, dom, cfg, pool_axis, peak, peak_src, mufu_peak, fma_peak):
    """The roofline object of the dominant kernel `dom` (algorithmic amount per launch over the mean
    CUDA-event duration of its launches)."""
    bound, amount = kernel_work(dom, cfg, pool_axis)
    dk = kern[dom]
    amount //= max(1, dk["launches_per_step"])
    if bound == "alu":
        return {"bound": "alu", "kernel": dom, "achieved": dk["achieved"], "peak": mufu_peak,
                "unit": "G exp2/s", "frac": dk["frac"], "traffic": recorded_traffic(dom, cfg.name),
                "algorithmic_exp2_per_launch": amount,
                "peak_source": f"derived: SMs x {MUFU_PER_SM_CLK} MUFU lanes/clk x max SM clock",
                "note": "achieved = exp2 evaluations per launch / mean CUDA-event duration of the launch"}
    if bound == "fma":
        return {"bound": "alu", "kernel": dom, "achieved": dk["achieved"], "peak": fma_peak,
                "unit": "TFLOP/s fp32", "frac": dk["frac"], "traffic": recorded_traffic(dom, cfg.name),
                "algorithmic_flop_per_launch": amount,
                "peak_source": f"derived: SMs x {FFMA_PER_SM_CLK} FMA lanes/clk x 2 flop x max SM clock",
                "note": "achieved = flops per launch / mean CUDA-event duration of the launch"}
    return {"bound": "hbm", "kernel": dom, "achieved": dk.get("achieved"), "peak": peak, "unit": "GB/s",
            "frac": dk.get("frac"), "traffic": recorded_traffic(dom, cfg.name),
            "algorithmic_bytes_per_launch": amount, "peak_source": peak_src,
            "note": "achieved = algorithmic bytes per launch / mean CUDA-event duration of the launch"}


def time_layer(a, cfg, pool_axis, dev, world=1, first_image=0, clocks=None, conv=None, path=None):
    """Device-timed forward calls of one workload (inputs resident in HBM): `a.warmup` untimed calls,
    then `a.steps` timed ones between CUDA events on the launching stream, each launch bracketed by
    its own pair of events.  Returns the step time (max over ranks), the per-kernel table and the
    roofline of the dominant kernel, plus the shape (for the end-to-end leg)."""
    import torch
    import torch.distributed as dist

    from pooled_selective_scan_b200 import ssm, workload

    conv = a.conv if conv is None else conv
    path = a.path if path is None else path
    t = workload.layer_tensors(cfg, dev, first_image=first_image)
    if a.ln:
        t.update(workload.ln_tensors(cfg, dev))
    if conv:
        t.update(workload.conv_tensors(cfg, dev, conv))
    keep = t.get("keep_idx")
    shape = ssm.infer_shape(t["x"], t["A_log"], t["W_dt"], pool_axis, cfg.dir_flags, keep, cfg.h, cfg.w, path=path,
                            ln=a.ln, d_conv=conv, conv_silu=bool(conv))
    y = torch.empty_like(t["x"])
    ws = ssm.alloc_workspace(shape, dev)
    stream = torch.cuda.current_stream(dev)
    fwd = ssm.BoundForward(shape, t, y, ws, stream)
    names = ssm.launch_names(shape)
    nl = len(names)

    for _ in range(a.warmup):
        fwd.run()
    torch.cuda.synchronize(dev)
    if ssm.device_status(ws) != 0:
        raise SystemExit(f"{cfg.name}: device status reported an error during warm-up")

    # events[2j], events[2j+1] bracket launch j on the stream it runs on
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * nl)] for _ in range(a.steps)]
    for evs in events:  # materialise the event handles outside the timed region
        for e in evs:
            e.record(stream)
    torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    # Workloads whose inputs fit in L2 get an L2 flush (a write of 2x the L2 size) before every
    # step; the step time is then the span of the step's own launches (first to last event).
    alg_bytes_call = cfg.algorithmic_bytes_per_call()
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev) if alg_bytes_call < 2 * L2_BYTES else None

    own_clocks = clocks is None
    if own_clocks:
        clocks = ClockSampler(dev.index or 0)
        clocks.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    start.record(stream)
    for i in range(a.steps):
        if flush is not None:
            flush.fill_(float(i))
        fwd.run_events(events[i])
    end.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    if own_clocks:
        clocks.stop()
    if flush is None:
        local_ms = start.elapsed_time(end)
    else:
        local_ms = sum(evs[0].elapsed_time(evs[2 * nl - 1]) for evs in events)  # first to last launch
    max_ms = reduce_max(local_ms, dev)
    # per kernel: its launches' device time in each step
    per_kernel = {n: [] for n in dict.fromkeys(names)}
    for evs in events:
        step = {n: 0.0 for n in per_kernel}
        for j, n in enumerate(names):
            step[n] += evs[2 * j].elapsed_time(evs[2 * j + 1])
        for n, v in step.items():
            per_kernel[n].append(v)
    if ssm.device_status(ws) != 0:
        raise SystemExit(f"{cfg.name}: device status reported an error in the timed region")

    tokens = cfg.tokens_per_call()
    ms_step = max_ms / a.steps
    peak, peak_src = load_peaks()
    summ = clocks.summary()
    mufu_peak = mufu_peak_gops(dev.index or 0, summ.get("sm_max_mhz"))
    fma_peak = ffma_peak_tflops(dev.index or 0, summ.get("sm_max_mhz"))
    kern = summarize_kernels(per_kernel, names, cfg, pool_axis, peak, mufu_peak, fma_peak)
    dom = max(kern, key=lambda n: kern[n]["share"])
    res = {
        "ms_per_step": ms_step,
        "value": weak_scaling_value(tokens * a.steps, world, max_ms / 1e3),
        "layer_hbm": {"achieved_gbs": alg_bytes_call / (ms_step / 1e3) / 1e9, "peak_gbs": peak,
                      "frac": alg_bytes_call / (ms_step / 1e3) / 1e9 / peak,
                      "algorithmic_bytes_per_step": alg_bytes_call},
        "roofline": roofline_of(kern, dom, cfg, pool_axis, peak, peak_src, mufu_peak, fma_peak),
        "kernels": kern,
        "gpu_launches": nl * a.steps,
        "l2": (f"inputs {alg_bytes_call / 1e9:.2f} GB per step > 126 MB L2; no flush" if flush is None
               else f"inputs {alg_bytes_call / 1e6:.1f} MB per step < 2 x L2: L2 flushed (256 MB write) "
                    f"before every step, step time = span of the step's launches"),
        "shape": shape,
    }
    if own_clocks:
        res["clocks"] = summ
    del fwd, t, y, ws, events, flush
    torch.cuda.empty_cache()
    return res


def link_copy_rates(dev, nbytes=1 << 30, reps=3):
    """Measured pinned-host <-> device copy rates (GB/s) over one direction at a time: the host
    link's own ceiling for the end-to-end leg."""
    import torch
    h = torch.empty(nbytes // 4, dtype=torch.float32).pin_memory()
    d = torch.empty(nbytes // 4, dtype=torch.float32, device=dev)
    rates = {}
    for name, (dst, src) in (("h2d", (d, h)), ("d2h", (h, d))):
        best = float("inf")
        for _ in range(reps):
            torch.cuda.synchronize(dev)
            t0 = time.perf_counter()
            dst.copy_(src, non_blocking=True)
            torch.cuda.synchronize(dev)
            best = min(best, time.perf_counter() - t0)
        rates[name] = nbytes / best / 1e9
    del h, d
    return rates


def time_e2e(a, cfg, shape, dev, world=1, first_image=0):
    """End-to-end calls through fastvim_ssm_forward_host on pinned host buffers (every rank; max
    over ranks), with the host link's measured copy rates as its ceiling."""
    import torch
    import torch.distributed as dist

    from pooled_selective_scan_b200 import ssm, workload

    host = workload.layer_tensors(cfg, dev, pinned_host=True, first_image=first_image)
    if a.ln:
        host.update({k: v.pin_memory() for k, v in workload.ln_tensors(cfg, "cpu").items()})
    if a.conv:
        host.update({k: v.pin_memory() for k, v in workload.conv_tensors(cfg, "cpu", a.conv).items()})
    run = ssm.HostForward(shape, dev)
    y_host = torch.empty(host["x"].shape, dtype=torch.float32).pin_memory()
    run(host, y_host)  # warm
    if world > 1:
        dist.barrier()
    t0 = time.perf_counter()
    for _ in range(a.e2e_steps):
        run(host, y_host)
    el = reduce_max(time.perf_counter() - t0, dev)
    tokens = cfg.tokens_per_call()
    bi, bo = run.h2d_bytes(), run.d2h_bytes()
    del run, host, y_host
    torch.cuda.empty_cache()
    rates = link_copy_rates(dev)
    step_s = el / a.e2e_steps
    # the two directions run on separate copy engines: the slower one bounds a step
    bound_s = max(bi / (rates["h2d"] * 1e9), bo / (rates["d2h"] * 1e9))
    return {"value": weak_scaling_value(tokens * a.e2e_steps, world, el), "unit": UNIT,
            "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "steps": a.e2e_steps,
            "link": {"h2d_gbs": bi / step_s / 1e9, "d2h_gbs": bo / step_s / 1e9,
                     "h2d_copy_gbs_measured": rates["h2d"], "d2h_copy_gbs_measured": rates["d2h"],
                     "bound_ms": bound_s * 1e3, "frac": bound_s / step_s,
                     "note": "frac = the step time that one-way pinned copies at the measured rates would take, "
                             "over the measured step time"},
            "note": "pinned host x, z, params -> device, layer, y -> pinned host; per-step wall time"}


def run_ours(a, cfg, pool_axis):
    import torch
    import torch.distributed as dist

    from pooled_selective_scan_b200 import build as fvbuild
    from pooled_selective_scan_b200 import workload
    from pooled_selective_scan_b200.configs import by_name

    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the layer has no CPU path)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    if not os.path.exists(os.path.join(ROOT, "pooled_selective_scan_b200", "libfastvim_ssm.so")):
        if rank == 0:
            fvbuild.build()
        if world > 1:
            dist.barrier()

    mine = workload.shard_images(cfg, rank, world)
    r = time_layer(a, cfg, pool_axis, dev, world, first_image=mine.start)
    line = {
        "metric": METRIC, "value": r["value"], "unit": UNIT, "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
        "ms_per_step": r["ms_per_step"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic (seeded N(0,1) x, z; Mamba-style parameter init)",
        "config": dict(workload_desc(cfg, pool_axis),
                       **({"post_ssm_layernorm": "gamma = 1, beta = 0, eps = 1e-5"} if a.ln else {}),
                       **({"conv1d": f"{a.conv} taps per direction + SiLU in front; x is its input"} if a.conv else {}),
                       l2=r["l2"], global_batch=cfg.B * world,
                       parallelism=f"data parallel, no collective: each of {world} GPU(s) runs its own "
                                   f"{cfg.B} distinct images"),
        "layer_hbm": r["layer_hbm"],
        "roofline": r["roofline"],
        "kernels": r["kernels"],
        "gpu_launches": r["gpu_launches"],
        "clocks": r["clocks"],
    }
    line["e2e"] = None if a.no_e2e else time_e2e(a, cfg, r["shape"], dev, world, first_image=mine.start)

    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, pool_axis)

    # the other workloads of the efficiency study, one GPU, default run only
    if world == 1 and not a.no_configs and a.batch is None and cfg.name == HEADLINE_NAME and not a.conv and not a.ln:
        configs = {}
        for name, axis in SECONDARY:
            c = by_name(name)
            sub = time_layer(a, c, axis, dev)
            ent = {"workload": workload_desc(c, axis), "ms_per_step": sub["ms_per_step"], "value": sub["value"],
                   "unit": UNIT + (" (kept tokens)" if c.masked else ""), "steps": a.steps, "warmup": a.warmup,
                   "l2": sub["l2"], "layer_hbm": sub["layer_hbm"], "roofline": sub["roofline"],
                   "kernels": sub["kernels"], "gpu_launches": sub["gpu_launches"], "clocks": sub["clocks"]}
            if not a.no_cpu_baseline:
                ent["cpu_baseline"] = cpu_baseline(c, axis, min_seconds=5.0)
            configs[f"{name}/{'pool_w' if axis == 0 else 'pool_h'}"] = ent
        for name, axis, taps, path in SECONDARY_VARIANTS:
            c = by_name(name)
            sub = time_layer(a, c, axis, dev, conv=taps, path=path)
            desc = workload_desc(c, axis)
            if taps:
                desc["conv1d"] = f"{taps} taps per direction + SiLU in front; x is its input"
            if path != "auto":
                desc["path"] = path
            ent = {"workload": desc, "ms_per_step": sub["ms_per_step"], "value": sub["value"], "unit": UNIT,
                   "steps": a.steps, "warmup": a.warmup, "l2": sub["l2"], "layer_hbm": sub["layer_hbm"],
                   "roofline": sub["roofline"], "kernels": sub["kernels"], "gpu_launches": sub["gpu_launches"],
                   "clocks": sub["clocks"]}
            key = name + (f"+conv{taps}" if taps else "") + ("" if path == "auto" else f"+{path}")
            configs[f"{key}/{'pool_w' if axis == 0 else 'pool_h'}"] = ent
        line["configs"] = configs
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_grad(a, cfg, pool_axis):
    """One step = the forward call + the gradient call over the batch (a training step of the
    layer), inputs and dy resident in HBM; 1 GPU."""
    import torch

    from pooled_selective_scan_b200 import build as fvbuild
    from pooled_selective_scan_b200 import ssm, workload

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the layer has no CPU path)")
    world, rank, local = dist_env()
    if world > 1:
        raise SystemExit("--grad runs on one GPU")
    if a.conv:
        raise SystemExit("--grad: the gradient through the Conv1D is not built")
    if not os.path.exists(os.path.join(ROOT, "pooled_selective_scan_b200", "libfastvim_ssm.so")):
        fvbuild.build()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    t = workload.layer_tensors(cfg, dev)
    if a.ln:
        t.update(workload.ln_tensors(cfg, dev))
    dy = workload.upstream_grad(cfg, dev)
    keep = t.get("keep_idx")
    shape = ssm.infer_shape(t["x"], t["A_log"], t["W_dt"], pool_axis, cfg.dir_flags, keep, cfg.h, cfg.w, path=a.path,
                            ln=a.ln, keep_states=not a.recompute_states)
    y = torch.empty_like(t["x"])
    fws = ssm.alloc_workspace(shape, dev)
    bws = torch.empty(max(ssm.backward_workspace_size(shape), 256), dtype=torch.uint8, device=dev)
    grads = {"dx": torch.empty_like(t["x"]), "dz": torch.empty_like(t["z"])}
    for n in ("A_log", "D", "W_x", "W_dt", "b_dt") + (("ln_gamma", "ln_beta") if a.ln else ()):
        grads["d" + n] = torch.empty_like(t[n])
    stream = torch.cuda.current_stream(dev)
    fwd = ssm.BoundForward(shape, t, y, fws, stream)
    bwd = ssm.BoundBackward(shape, t, dy, grads, fws, bws, stream)
    names = ssm.launch_names(shape) + bwd.names
    nf, nl = fwd.n_launch, len(names)
    for _ in range(a.warmup):
        fwd.run()
        bwd.run()
    torch.cuda.synchronize(dev)
    if ssm.device_status(fws) != 0:
        raise SystemExit("device status reported an error during warm-up")
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * nl)] for _ in range(a.steps)]
    for evs in events:
        for e in evs:
            e.record(stream)
    torch.cuda.synchronize(dev)
    alg_bytes = cfg.algorithmic_bytes_per_call()
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev) if alg_bytes < 2 * L2_BYTES else None
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    torch.cuda.synchronize(dev)
    start.record(stream)
    for i in range(a.steps):
        if flush is not None:
            flush.fill_(float(i))
        fwd.run_events(events[i][:2 * nf])
        bwd.run_events(events[i][2 * nf:])
    end.record(stream)
    torch.cuda.synchronize(dev)
    clocks.stop()
    if flush is None:
        ms = start.elapsed_time(end)
    else:
        ms = sum(evs[0].elapsed_time(evs[2 * nl - 1]) for evs in events)
    per_kernel = {n: [] for n in dict.fromkeys(names)}
    for evs in events:
        step = {n: 0.0 for n in per_kernel}
        for j, n in enumerate(names):
            step[n] += evs[2 * j].elapsed_time(evs[2 * j + 1])
        for n, v in step.items():
            per_kernel[n].append(v)
    tokens = cfg.tokens_per_call()
    peak, peak_src = load_peaks()
    mufu_peak = mufu_peak_gops(local, clocks.summary().get("sm_max_mhz"))
    fma_peak = ffma_peak_tflops(local, clocks.summary().get("sm_max_mhz"))
    kern = summarize_kernels(per_kernel, names, cfg, pool_axis, peak, mufu_peak, fma_peak)
    dom = max((n for n in kern if n.startswith("bwd_")), key=lambda n: kern[n]["share"])
    dk = kern[dom]
    bound, amount = kernel_work(dom, cfg, pool_axis)
    roofline = {"bound": bound if bound == "hbm" else "alu", "kernel": dom, "achieved": dk.get("achieved"),
                "peak": peak if bound == "hbm" else (mufu_peak if bound == "alu" else fma_peak), "unit": dk.get("unit"),
                "frac": dk.get("frac"), "traffic": recorded_traffic(dom, cfg.name) if cfg.B == 128 else None,
                "algorithmic_per_launch": amount, "peak_source": peak_src if bound == "hbm" else "derived",
                "note": "dominant kernel of the gradient; achieved = algorithmic amount per launch / mean "
                        "CUDA-event duration of the launch"}
    # the gradient's own HBM floor: read x, z, dy, write dx, dz (5 rows per token)
    bwd_ms = sum(statistics.mean(per_kernel[n]) for n in dict.fromkeys(bwd.names))
    line = {
        "metric": "SSM-layer training step (forward + gradient) grid tokens/s at " + cfg.name +
                  (" with the post-SSM LayerNorm" if a.ln else "") + " (fp32)",
        "value": tokens * a.steps / (ms / 1e3), "unit": UNIT, "n_gpus": 1, "steps": a.steps, "warmup": a.warmup,
        "ms_per_step": ms / a.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic (seeded N(0,1) x, z, dy; Mamba-style parameter init)",
        "config": dict(workload_desc(cfg, pool_axis), step="forward call + gradient call",
                       scan_states="kept by the forward (FV_FLAG_KEEP_STATES)" if shape.keep_states
                       else "recomputed by the gradient",
                       l2=("no flush (inputs > 2 x L2)" if flush is None else "L2 flushed before every step")),
        "gradient": {"ms": bwd_ms, "hbm_floor_ms": 5 * 4 * cfg.E * tokens / (peak * 1e9) * 1e3,
                     "floor_note": "x, z, dy read once, dx, dz written once at the measured copy rate"},
        "roofline": roofline,
        "kernels": kern,
        "gpu_launches": nl * a.steps,
        "clocks": clocks.summary(),
        "e2e": None,
    }
    if not a.no_cpu_baseline:
        import numpy as np

        import oracle
        from pooled_selective_scan_b200 import inputs
        cores = host_cores()
        which = list(range(min(cfg.B, max(1, cores), 16)))
        d = inputs.layer_inputs(cfg, which=which)
        shp = inputs.token_shape(cfg)
        dyh = np.stack([inputs.image_dy(cfg.seed, b, shp) for b in which])
        oracle.build()
        lnkw = {}
        if a.ln:
            lnkw = dict(ln_gamma=np.ones(cfg.E, np.float32), ln_beta=np.zeros(cfg.E, np.float32), ln_eps=1e-5)
        t0 = time.perf_counter()
        oracle.forward(d["x"], d["z"], d["A_log"], d["D"], d["W_x"], d["W_dt"], d["b_dt"], pool_axis, cfg.dir_flags,
                       keep_idx=d.get("keep_idx"), h=cfg.h, w=cfg.w, nthreads=len(which), **lnkw)
        oracle.backward(d["x"], d["z"], d["A_log"], d["D"], d["W_x"], d["W_dt"], d["b_dt"], dyh, pool_axis,
                        cfg.dir_flags, keep_idx=d.get("keep_idx"), h=cfg.h, w=cfg.w, nthreads=len(which), **lnkw)
        el = time.perf_counter() - t0
        tok = len(which) * (cfg.K if cfg.masked else cfg.h * cfg.w)
        line["cpu_baseline"] = {"value": tok / el, "unit": UNIT, "cores": len(which), "kind": "oracle",
                                "sample": f"{len(which)} images of {cfg.name}: fp64 oracle forward + gradient, "
                                          f"OpenMP over images ({el:.1f} s wall)"}
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    a = parse(argv)
    from pooled_selective_scan_b200.configs import by_name
    cfg = by_name(a.config)
    if a.batch is not None:
        import dataclasses
        cfg = dataclasses.replace(cfg, B=a.batch)
    pool_axis = cfg.pool_axes[0] if a.pool_axis is None else a.pool_axis
    if a.impl == "reference":
        return run_reference(a, cfg, pool_axis)
    if a.grad:
        return run_grad(a, cfg, pool_axis)
    return run_ours(a, cfg, pool_axis)


if __name__ == "__main__":
    sys.exit(main())
