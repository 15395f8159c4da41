#!/usr/bin/env python
"""Throughput of the R2L sidecar forward on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config 2]

A step is one full sidecar forward (in_proj → conv+SiLU → x_proj → dt_proj →
reverse scan → out_proj → LayerNorm + gated residual) over one batch of the
serving workload of "Bifocal Diffusion Language Models" (arXiv 2606.27732v1,
§4.3 / Table 3: batch 8, prompt 4096; d_model 2048 per §4.1), with seeded
synthetic hidden states and weights.  Every rank (one per GPU, launched by
torchrun for N > 1) runs its own contiguous slice of one global batch of
N × B sequences: sequences are independent, so the batch shards with no
data-path collective (weak scaling).

`value` is device time (CUDA events on the launching stream, max over ranks)
with inputs resident in HBM; the per-step working set (~1.5 GB of activations
and workspace) is far larger than the 126 MB L2, so no flush is needed.
`e2e` is the same call with the hidden states copied from pinned host memory
and the result copied back inside the timed region.
"""
from __future__ import annotations

import argparse
import hashlib
import glob
import json
import os
import statistics
import subprocess
import sys
import time
from datetime import timedelta

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "R2L sidecar tokens/sec at B=8,L=4096,d=2048; scan HBM GB/s % of peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--config", type=int, default=2, help="workload 1..4 (2 = the headline)")
    ap.add_argument("--batch", type=int, default=None, help="override the workload's batch size (profiling)")
    ap.add_argument("--seq", type=int, default=None, help="override the workload's sequence length (profiling)")
    ap.add_argument("--general-a", action="store_true", help="force the general-A scan path")
    ap.add_argument("--graph", action="store_true",
                    help="capture one step in a CUDA graph and time its replays (no per-stage times)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--scan-backward", action="store_true",
                    help="time the fp32 reverse-scan gradient (r2l_reverse_scan_backward) at B=8, L=4096, "
                         "d_inner=4096 instead of the forward")
    ap.add_argument("--hook-backward", action="store_true",
                    help="time the whole hook's gradient (r2l_sidecar_backward: dh, ds and every parameter) on "
                         "the workload instead of the forward")
    return ap.parse_args(argv)


# ---------------------------------------------------------------- helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# The sources each stage's kernel is built from (a profile of that kernel stays
# valid while these files are unchanged).
_COMMON = ["common.cuh", "sm100_primitives.cuh", "tmap.cu", "tmap.h"]
STAGE_SOURCES = {
    "gemm": ["gemm_tc.cuh", "tc_gemm.cu", "tc_gemm.h"] + _COMMON,
    "in_proj": ["gemm_tc.cuh", "tc_gemm.cu", "tc_gemm.h"] + _COMMON,
    "x_proj": ["gemm_convx.cuh", "gemm_tc.cuh", "tc_gemm.cu", "tc_gemm.h"] + _COMMON,
    "conv": ["conv_fast.cuh", "gemm_convx.cuh"] + _COMMON,
    "dt_proj": ["gemm_tc.cuh", "tc_gemm.cu", "tc_gemm.h"] + _COMMON,
    "out_proj": ["gemm_tc.cuh", "tc_gemm.cu", "tc_gemm.h"] + _COMMON,
    "scan": ["scan_fast.cuh", "scan_fast.h", "scan_launch.cu", "scan_pair.cuh", "scan_split.cuh"] + _COMMON,
    "ln_residual": ["simt_kernels.cuh"] + _COMMON,
    "scan_bwd": ["scan_bwd.cu", "scan_bwd.h", "scan_bwd_seq.cuh"] + _COMMON,
    "scan_general": ["scan_fast.cuh", "scan_fast.h", "scan_launch.cu", "scan_pair.cuh", "scan_split.cuh"] + _COMMON,
}


def source_sha(stage=None):
    """Hash of the kernel sources: of one stage's files, or of all of them."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "reverse_selective_ssm_b200", "csrc")
    files = sorted(glob.glob(os.path.join(csrc, "*"))) if stage is None else \
        [os.path.join(csrc, f) for f in sorted(STAGE_SOURCES[stage])]
    for f in files:
        h.update(open(f, "rb").read())
    return h.hexdigest()[:16]


def read_traffic(stage, workload_tag):
    """dram bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    for f in glob.glob(os.path.join(ROOT, "profiles", "*.txt")):
        kv = {}
        for line in open(f):
            if ":" in line:
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
        if kv.get("stage") == stage and kv.get("workload") == workload_tag and \
                kv.get("source_sha") == source_sha(stage) and "dram_bytes_per_launch" in kv:
            try:
                return float(kv["dram_bytes_per_launch"])
            except ValueError:
                return None
    return None


def read_profile_value(stage, workload_tag, key):
    """A numeric field of the committed ncu summary of one stage, if it was
    taken on the current kernel sources (else None)."""
    for f in glob.glob(os.path.join(ROOT, "profiles", "*.txt")):
        kv = {}
        for line in open(f):
            if ":" in line:
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
        if kv.get("stage") == stage and kv.get("workload") == workload_tag and \
                kv.get("source_sha") == source_sha(stage) and key in kv:
            try:
                return float(kv[key].split()[0])
            except ValueError:
                return None
    return None


# FP32 operations per (token, channel) that the scan's arithmetic needs, on the
# FMA pipe: the 16 decays r, r², …, r¹⁶ (15 products), Δu·B (16), the state
# update (16 FMAs) and ⟨C, H⟩ (16 FMAs and a final add) for the 16 states, plus
# softplus (4), Δu and D·u (2), SiLU(z) (3) and the gate (2).
SCAN_FP32_OPS_PER_TOKEN_CHANNEL = 15 + 16 + 16 + 17 + 4 + 2 + 3 + 2
B200_SMS = 148


def scan_ceilings(case, ms, clocks, workload_tag):
    """The scan against the two ceilings that bind before HBM does: the FP32
    pipe (128 lane-operations per clock per SM, all 148 SMs) on the
    arithmetic the recurrence needs, and instruction issue (one warp
    instruction per clock per scheduler) on the instructions the kernel
    executes (ncu, committed summary).  Both at the median SM clock sampled
    during the timed region (the maximum if none was sampled)."""
    T, E = case.valid_tokens, case.dims.d_inner
    mhz = (clocks or {}).get("sm_mhz") or (clocks or {}).get("sm_max_mhz") or 1965.0
    f = mhz * 1e6
    sec = ms * 1e-3
    ops = SCAN_FP32_OPS_PER_TOKEN_CHANNEL * float(T) * E
    fp32_peak = B200_SMS * 128 * f
    out = {"clock_mhz": mhz,
           "fp32_pipe": {"ops_per_token_channel": SCAN_FP32_OPS_PER_TOKEN_CHANNEL,
                         "achieved_tops": round(ops / sec / 1e12, 3), "peak_tops": round(fp32_peak / 1e12, 3),
                         "frac": round(ops / sec / fp32_peak, 4),
                         "ceiling_ms": round(ops / fp32_peak * 1e3, 4)}}
    inst = read_profile_value("scan", workload_tag, "inst_per_token_channel")
    if inst is not None:
        warp_inst = inst * T * E / 32.0
        ceiling = warp_inst / (B200_SMS * 4 * f)
        out["issue"] = {"inst_per_token_channel": inst, "ceiling_ms": round(ceiling * 1e3, 4),
                        "frac": round(ceiling / sec, 4),
                        "source": "smsp__inst_executed of the committed ncu summary (profiles/)"}
    fma = read_profile_value("scan", workload_tag, "fma_pipe_active_frac")
    if fma is not None:
        out["fp32_pipe"]["ncu_fma_pipe_active_frac"] = fma
    return out


class ClockSampler:
    """SM clock and clock-event reasons of this rank's GPU, read (never set)
    every few milliseconds between start() and stop(): through NVML on a
    thread when pynvml imports, else from an ``nvidia-smi -lms`` child."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits (nvml.h): SwPowerCap, HwSlowdown, SwThermal, HwThermal
    REASON_BITS = (("sw_power_cap", 0x4), ("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20),
                   ("hw_thermal_slowdown", 0x40))
    PERIOD_S = 0.005

    def __init__(self, local_rank):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        self.gpu = vis.split(",")[local_rank].strip() if vis else str(local_rank)
        self.proc = None
        self.thread = None
        self.samples = []

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        if self.gpu.startswith("GPU-") or self.gpu.startswith("MIG-"):
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(self.gpu)
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(int(self.gpu))

    def start(self):
        import threading
        try:
            nv, hnd = self._nvml_handle()
        except Exception:
            nv = None
        if nv is not None:
            self.stop_event = threading.Event()
            smax = nv.nvmlDeviceGetMaxClockInfo(hnd, nv.NVML_CLOCK_SM)

            def loop():
                while not self.stop_event.is_set():
                    try:
                        sm = nv.nvmlDeviceGetClockInfo(hnd, nv.NVML_CLOCK_SM)
                        rs = nv.nvmlDeviceGetCurrentClocksEventReasons(hnd) \
                            if hasattr(nv, "nvmlDeviceGetCurrentClocksEventReasons") \
                            else nv.nvmlDeviceGetCurrentClocksThrottleReasons(hnd)
                        self.samples.append((float(sm), float(smax), int(rs)))
                    except Exception:
                        pass
                    self.stop_event.wait(self.PERIOD_S)

            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", self.gpu],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_event.set()
            self.thread.join(timeout=5)
            sm = [x[0] for x in self.samples]
            smax = [x[1] for x in self.samples]
            reasons = {n for _, _, r in self.samples for n, bit in self.REASON_BITS if r & bit}
            return {"sm_mhz": statistics.median(sm) if sm else None,
                    "sm_max_mhz": max(smax) if smax else None,
                    "reasons": sorted(reasons), "samples": len(sm), "source": "nvml"}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvidia-smi"}


def algorithmic(case, stage):
    """(bound, amount per launch, unit) for one stage on ``case`` (valid tokens only)."""
    d, E, R, N = case.dims.d_model, case.dims.d_inner, case.dims.dt_rank, case.dims.d_state
    T = case.valid_tokens
    a = 2 if case.dtype.itemsize == 2 else 4
    if stage == "in_proj":
        return "tensor", 2.0 * T * d * 2 * E, "flop"
    if stage == "x_proj":
        return "tensor", 2.0 * T * E * (R + 2 * N), "flop"
    if stage == "dt_proj":
        return "tensor", 2.0 * T * R * E, "flop"
    if stage == "out_proj":
        return "tensor", 2.0 * T * E * d, "flop"
    if stage == "conv":
        return "hbm", float(T) * E * (a + a), "byte"
    if stage == "scan":
        # the step's bytes per token as the scope table counts them: u, z and
        # dt_raw read, y written (activation dtype) + B, C read (fp32)
        return "hbm", float(T) * (E * 4 * a + 2 * N * 4), "byte"
    if stage == "ln_residual":  # o read, h read, h written
        return "hbm", float(T) * d * 3 * a, "byte"
    raise KeyError(stage)


def scan_kernel_bytes(case):
    """Bytes the scan kernel itself moves per launch: with dt_proj inside it
    (bf16, dt_rank 128) it reads the dt_rank-wide Δr row instead of dt_raw."""
    E, R, N = case.dims.d_inner, case.dims.dt_rank, case.dims.d_state
    a = 2 if case.dtype.itemsize == 2 else 4
    dt_bytes = R * 2 if (a == 2 and R == 128) else E * a
    return float(case.valid_tokens) * (E * 3 * a + dt_bytes + 2 * N * 4)


# Stages that run as launches of one kernel function (the bf16 path): in_proj and
# out_proj are the same tcgen05 GEMM; the rest are one kernel each.
KERNEL_STAGES = {"gemm": ("in_proj", "out_proj"), "scan": ("scan",), "x_proj": ("conv", "x_proj"),
                 "ln_residual": ("ln_residual",)}


def dominant_kernel(per_launch):
    """The kernel function with the most time per step (its stages summed)."""
    tot = {k: sum(per_launch.get(s, 0.0) for s in st) for k, st in KERNEL_STAGES.items()}
    return max(tot, key=tot.get)


def tensor_peak(peaks, peak_kind, clocks, timed_ms):
    """The dense bf16 peak that applies to GEMMs timed in this run: the burst
    cuBLAS figure when the timed region is short (under a second) and the
    clock record shows no power cap with the median SM clock near its maximum;
    otherwise the sustained, power-capped figure.  Returns (peak, note)."""
    c = clocks or {}
    sm, smax = c.get("sm_mhz"), c.get("sm_max_mhz")
    capped = "sw_power_cap" in (c.get("reasons") or [])
    near_max = bool(sm and smax and sm >= 0.95 * smax)
    if timed_ms < 1000.0 and near_max and not capped:
        return peaks["bf16_tflops"], (f"{peak_kind} cuBLAS bf16 burst: timed region {timed_ms:.0f} ms, "
                                      f"median SM clock {sm:.0f} of {smax:.0f} MHz, no power cap")
    why = "power cap seen" if capped else (f"timed region {timed_ms:.0f} ms" if timed_ms >= 1000.0
                                          else "SM clock below 95 % of max or not sampled")
    return peaks["bf16_tflops_sustained"], f"{peak_kind} cuBLAS bf16 sustained ({why})"


def roofline_kernel(case, kernel, per_launch, peaks, peak_kind, workload_tag, tpeak):
    """roofline of one kernel function: algorithmic work over its launches per
    step ÷ their total time (= per launch ÷ average launch duration).
    tpeak: (dense bf16 peak, note) from tensor_peak()."""
    if kernel != "gemm":
        stage = "x_proj" if kernel == "x_proj" else kernel
        return roofline_obj(case, stage, per_launch[stage] + (per_launch.get("conv", 0.0) if kernel == "x_proj" else 0.0),
                            peaks, peak_kind, workload_tag, tpeak)
    st = KERNEL_STAGES["gemm"]
    flops = sum(algorithmic(case, s)[1] for s in st)
    ms = sum(per_launch[s] for s in st)
    achieved = flops / (ms * 1e-3) / 1e12
    peak, note = tpeak
    return {"kernel": "gemm_tc (in_proj + out_proj launches)", "bound": "tensor", "achieved": round(achieved, 2),
            "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
            "frac_of_burst": round(achieved / peaks["bf16_tflops"], 4),
            "frac_of_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4),
            "peak_source": note,
            "algorithmic_per_launch": flops / len(st), "ms_per_launch": round(ms / len(st), 5),
            "traffic": read_traffic("gemm", workload_tag)}


def roofline_obj(case, stage, ms, peaks, peak_kind, workload_tag, tpeak=None):
    bound, amount, _ = algorithmic(case, stage)
    if bound == "tensor":
        achieved = amount / (ms * 1e-3) / 1e12
        peak, peak_note = tpeak or (peaks["bf16_tflops_sustained"], f"{peak_kind} cuBLAS bf16 sustained")
        unit = "TFLOP/s"
    else:
        achieved = amount / (ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        unit = "GB/s"
        peak_note = f"{peak_kind} HBM copy"
    obj = {"kernel": stage, "bound": bound, "achieved": round(achieved, 2), "peak": peak, "unit": unit,
           "frac": round(achieved / peak, 4), "peak_source": peak_note,
           "algorithmic_per_launch": amount, "ms_per_launch": round(ms, 5),
           "traffic": read_traffic(stage, workload_tag)}
    if stage == "scan":
        kb = scan_kernel_bytes(case)
        obj["kernel_bytes_per_launch"] = kb
        obj["frac_of_kernel_bytes"] = round(kb / (ms * 1e-3) / 1e9 / peak, 4)
    return obj


# ---------------------------------------------------------------- ranks

def max_over_ranks(ms: float, world: int, device=None) -> float:
    """The slowest rank's time (every rank must call this, in the same order)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(tokens_per_rank: int, world: int, steps: int, ms_max: float) -> float:
    """Tokens per second over all ranks: every rank runs its own batch (weak
    scaling), and the job takes as long as its slowest rank."""
    return tokens_per_rank * world * steps / (ms_max * 1e-3)


# ---------------------------------------------------------------- our arm

def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from reverse_selective_ssm_b200 import binding as bd
    from reverse_selective_ssm_b200 import synthetic as S

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    bd.load()
    # rank r runs sequences [r·B, (r+1)·B) of one global batch of N·B sequences
    case = S.make_case(args.config, B=args.batch, L=args.seq, shard=(rank, world))
    if args.batch or args.seq:
        case.name += f" (resized to B={case.B} L={case.L})"
    flags = bd.R2L_FLAG_GENERAL_A if args.general_a else 0
    dims = bd.dims_of(case.dims, case.dtype, flags)
    h = case.h.to(dev)
    wdev = [bd.weights_to_device(w, dev) for w in case.weights]
    lengths = None if case.lengths is None else case.lengths.to(dev)
    ws = bd.alloc_workspace(dims, case.B, case.L, dev)
    stream = torch.cuda.current_stream()
    hooks = len(wdev)
    nst = len(bd.STAGES)

    def step(events=None):
        # always the stream current at call time (the capture stream under a graph)
        st = torch.cuda.current_stream()
        launches = 0
        if events is None and hooks > 1:
            # a stack of hooks is one r2l_sidecar_stack call: one length check and
            # one A_log check for all hooks
            bd.sidecar_stack(h, wdev, dims, case.s, lengths, ws, st)
            return launches
        for k in range(hooks):
            if events is not None:
                launches += bd.sidecar_forward_profiled(h, wdev[k], dims, case.s[k], events[k], lengths, ws, st)
            else:
                bd.sidecar_forward(h, wdev[k], dims, case.s[k], lengths, ws, st)
        return launches

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st, fl = bd.get_device_status(ws, stream)
    if st != 0:
        raise RuntimeError(f"device status {st} flags {fl}")

    K = args.steps
    if args.graph:
        return run_graph(args, case, step, barrier, rank, world, local_rank, dev)
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)] for _ in range(hooks)]
           for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    # touch the events once so their handles exist before the timed region
    for per_step in evs:
        for per_hook in per_step:
            for e in per_hook:
                e.record(stream)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    if rank == 0:
        clocks.start()
        time.sleep(0.3)
    t0.record(stream)
    launches = 0
    for k in range(K):
        launches += step(evs[k])
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop() if rank == 0 else None
    ms_total = t0.elapsed_time(t1)
    stage_ms = {s: 0.0 for s in bd.STAGES}
    for k in range(K):
        for hk in range(hooks):
            e = evs[k][hk]
            for i, s in enumerate(bd.STAGES):
                stage_ms[s] += e[i].elapsed_time(e[i + 1])
    per_launch = {s: v / (K * hooks) for s, v in stage_ms.items()}

    ms_total = max_over_ranks(ms_total, world, dev)

    # ---- the general-A path: the same step with R2L_FLAG_GENERAL_A, timed on
    # its own (A_log of a trained model is not the S4D-real initialisation)
    general = None
    if not args.general_a:
        gdims = bd.dims_of(case.dims, case.dtype, bd.R2L_FLAG_GENERAL_A)
        gev = [[[torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)] for _ in range(hooks)]
               for _ in range(K)]
        for k in range(max(2, args.warmup // 2)):
            for hk in range(hooks):
                bd.sidecar_forward(h, wdev[hk], gdims, case.s[hk], lengths, ws, stream)
        torch.cuda.synchronize()
        barrier()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for k in range(K):
            for hk in range(hooks):
                bd.sidecar_forward_profiled(h, wdev[hk], gdims, case.s[hk], gev[k][hk], lengths, ws, stream)
        g1.record(stream)
        torch.cuda.synchronize()
        barrier()
        g_total = max_over_ranks(g0.elapsed_time(g1), world, dev)
        si = bd.STAGES.index("scan")
        g_scan = sum(gev[k][hk][si].elapsed_time(gev[k][hk][si + 1]) for k in range(K) for hk in range(hooks))
        general = {"ms_per_step": g_total / K, "scan_ms_per_launch": g_scan / (K * hooks)}

    # ---- end to end through host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, case, h, wdev, dims, lengths, ws, stream, barrier, world, dev)

    if rank != 0:
        return None

    peaks, peak_kind = load_peaks()
    workload_tag = f"config{args.config}-B{case.B}-L{case.L}"
    dom = dominant_kernel(per_launch)
    line = {
        "metric": METRIC if args.config == 2 else f"R2L sidecar tokens/sec, {case.name}",
        "value": round(whole_job_rate(case.valid_tokens, world, K, ms_total), 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(ms_total / K, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if case.dtype.itemsize == 2 else "f32",
        "data": "synthetic (seeded N(0,1) hidden states, N(0,0.02) weights, A=-(1..16), D=1)",
        "config": {"workload": case.name, "B": case.B, "L": case.L, "hooks": hooks,
                   "d_model": case.dims.d_model, "d_inner": case.dims.d_inner,
                   "d_state": case.dims.d_state, "dt_rank": case.dims.dt_rank,
                   "valid_tokens_per_gpu": case.valid_tokens, "s": case.s if hooks > 1 else case.s[0],
                   "l2": "inputs larger than L2 (~1.5 GB working set per step), no flush",
                   "global_batch": case.meta["global_batch"],
                   "parallelism": f"dp{world}: rank r runs sequences [r*{case.B}, (r+1)*{case.B}) of the global "
                                  f"batch of {case.meta['global_batch']}, seeded per global sequence; no collective",
                   "scan_path": "general-A" if args.general_a else "auto (power fast path when A=-(1..16))"},
        "roofline": roofline_kernel(case, dom, per_launch, peaks, peak_kind, workload_tag,
                                    tensor_peak(peaks, peak_kind, clk, ms_total)),
        "roofline_scan": dict(roofline_obj(case, "scan", per_launch["scan"], peaks, peak_kind, workload_tag),
                              path="general-A" if args.general_a else "power (A = -(1..16), exact per-call check)",
                              ceilings=scan_ceilings(case, per_launch["scan"], clk, workload_tag)),
        "stage_ms": {s: round(v, 5) for s, v in per_launch.items()},
        "roofline_scan_general": None if general is None else dict(
            roofline_obj(case, "scan", general["scan_ms_per_launch"], peaks, peak_kind, workload_tag),
            path="general-A (R2L_FLAG_GENERAL_A: one exponential per state)",
            ms_per_step=round(general["ms_per_step"], 4), traffic=None,
            tokens_per_s=round(whole_job_rate(case.valid_tokens, world, 1, general["ms_per_step"]), 1)),
        "gpu_launches": launches,
        "clocks": clk,
        "e2e": e2e,
        "source_sha": source_sha(),
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(case)
    return line


def run_graph(args, case, step, barrier, rank, world, local_rank, dev):
    """Time K replays of one step captured as a CUDA graph (launch overhead out
    of the loop); the denoise-step workload is launch-bound without it."""
    import torch
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()                      # one eager call on the capture stream first
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    with torch.cuda.graph(graph):
        step()
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    barrier()
    torch.cuda.synchronize()
    if rank == 0:
        clocks.start()
        time.sleep(0.3)
    t0.record()
    for _ in range(K):
        graph.replay()
    t1.record()
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop() if rank == 0 else None
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    del graph
    if rank != 0:
        return None
    hooks = len(case.weights)
    return {
        "metric": METRIC if args.config == 2 else f"R2L sidecar tokens/sec, {case.name}",
        "value": round(whole_job_rate(case.valid_tokens, world, K, ms), 1), "unit": "tokens/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": round(ms / K, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": {"workload": case.name, "B": case.B, "L": case.L, "hooks": hooks,
                                         "cuda_graph": True, "per_hook_us": round(ms / K / hooks * 1e3, 2),
                                         "api": "r2l_sidecar_stack" if hooks > 1 else "r2l_sidecar_forward"},
        "clocks": clk, "source_sha": source_sha(),
    }


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(case, sample_seqs=None):
    """The float64 oracle, as it stands, on a bounded sample of the workload:
    its first two sequences (one when the batch has one)."""
    import oracle as O
    from reverse_selective_ssm_b200 import synthetic as S
    if sample_seqs is None:
        sample_seqs = tuple(range(min(2, case.B)))
    h = S.to_f64(case.h)
    ws = [S.weights_f64(w) for w in case.weights]
    t = time.perf_counter()
    if len(ws) == 1:
        O.sidecar_forward(h, ws[0], case.s[0], None, "bf16", list(sample_seqs))
    else:
        O.sidecar_stack(h, ws, case.s, None, "bf16", list(sample_seqs))
    dt = time.perf_counter() - t
    tokens = case.L * len(sample_seqs)
    return {"value": round(tokens * len(ws) / dt / max(1, len(ws)), 2), "unit": "tokens/s",
            "cores": _blas_threads(), "kind": "oracle",
            "sample": f"sequences {list(sample_seqs)} of the workload in full ({tokens} tokens), "
                      f"numpy float64 oracle, {dt:.1f} s"}


E2E_BUFFERS = 3  # device buffers of the pipelined host-to-host loop


def run_e2e(args, case, h, wdev, dims, lengths, ws, stream, barrier, world, dev):
    """Tokens/s through r2l_sidecar_forward with the hidden states coming from
    and going back to pinned host memory every step.

    value: a pipelined serving loop. Step k's host-to-device copy runs on one
    stream, its forward on another and its device-to-host copy on a third, over
    E2E_BUFFERS device buffers. So the inbound copy of step k+1 and the outbound
    copy of step k-1 overlap the forward of step k. With three buffers the
    inbound copy of step k+1 does not wait for the outbound copy of step k-2,
    so the two directions of the link run at once (with two they alternate).
    The forward calls stay ordered on one stream, so they share one workspace.
    serial_value: copy in, forward, copy out, one after the other on one stream."""
    import torch
    from reverse_selective_ssm_b200 import binding as bd
    K = args.steps
    hooks = len(wdev)
    h_host = case.h.pin_memory()
    out_host = torch.empty_like(h_host).pin_memory()
    nbytes = h_host.numel() * h_host.element_size()

    def forward(buf, st):
        for k in range(hooks):
            bd.sidecar_forward(buf, wdev[k], dims, case.s[k], lengths, ws, st)

    # serial
    for _ in range(max(1, args.warmup // 2)):
        h.copy_(h_host, non_blocking=True)
        forward(h, stream)
        out_host.copy_(h, non_blocking=True)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(K):
        h.copy_(h_host, non_blocking=True)
        forward(h, stream)
        out_host.copy_(h, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_serial = max_over_ranks(e0.elapsed_time(e1), world, dev)

    # pipelined
    nb = E2E_BUFFERS
    bufs = [h] + [torch.empty_like(h) for _ in range(nb - 1)]
    s_in, s_fw, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(nb)]
    ev_fw = [torch.cuda.Event() for _ in range(nb)]
    ev_out = [torch.cuda.Event() for _ in range(nb)]

    def pipelined(n, t_start=None, t_end=None):
        if t_start is not None:
            t_start.record(s_in)
            s_fw.wait_event(t_start)
            s_out.wait_event(t_start)
        for k in range(n):
            i = k % nb
            if k >= nb:
                s_in.wait_event(ev_out[i])          # buffer i is free once step k-nb is copied out
            with torch.cuda.stream(s_in):
                bufs[i].copy_(h_host, non_blocking=True)
            ev_in[i].record(s_in)
            s_fw.wait_event(ev_in[i])
            forward(bufs[i], s_fw)
            ev_fw[i].record(s_fw)
            s_out.wait_event(ev_fw[i])
            with torch.cuda.stream(s_out):
                out_host.copy_(bufs[i], non_blocking=True)
            ev_out[i].record(s_out)
        if t_end is not None:
            s_out.wait_stream(s_in)
            s_out.wait_stream(s_fw)
            t_end.record(s_out)

    pipelined(max(nb, args.warmup))
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pipelined(K, p0, p1)
    torch.cuda.synchronize()
    barrier()
    ms_pipe = max_over_ranks(p0.elapsed_time(p1), world, dev)
    return {"value": round(whole_job_rate(case.valid_tokens, world, K, ms_pipe), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes,
            "serial_value": round(whole_job_rate(case.valid_tokens, world, K, ms_serial), 1),
            "api": "r2l_sidecar_forward via binding, pinned host hidden in/out",
            "device_buffers": nb,
            "schedule": f"pipelined: copy-in, forward and copy-out of successive steps on three streams over "
                        f"{nb} device buffers (serial_value: one stream, no overlap)"}


# ---------------------------------------------------------------- scan gradient

BWD_METRIC = "R2L reverse-scan backward tokens/sec at B=8,L=4096,E=4096 (fp32)"
B200_SCAN_BWD_BLOCK = 32  # channels per block of the walk along each sequence


def bwd_walks_sequences(B, E):
    """The library's path choice for chunk_tokens = 0: one 32-channel block
    walks each sequence when that gives at least 4 blocks per SM."""
    return B * (E // B200_SCAN_BWD_BLOCK) >= 4 * B200_SMS


def bwd_launches(B, E):
    """Kernels one r2l_reverse_scan_backward call launches: checkpoints,
    gradient, two reductions on the walk; state, carry, gradient and three
    reductions on the chunked path."""
    return 4 if bwd_walks_sequences(B, E) else 6


def bwd_bytes_per_token(E):
    """Bytes the gradient must move per position: u, z, dt_raw, dy read and du,
    dz, ddt_raw written (fp32, E channels each), B | C read and dB | dC written
    (32 fp32 each)."""
    return E * 7 * 4 + 2 * 32 * 4


def run_scan_backward(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from reverse_selective_ssm_b200 import binding as bd
    from reverse_selective_ssm_b200 import synthetic as S

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    bd.load()
    B, L, E = args.batch or 8, args.seq or 4096, 4096
    host = S.make_scan_bwd_case(B, L, E, seed=64 + rank)
    d = {k: v.to(dev) for k, v in host.items()}
    M = B * L
    out = {k: torch.empty((M, E), device=dev) for k in ("du", "dz", "ddt_raw")}
    out["dbc"] = torch.empty((M, 32), device=dev)
    out["dA_log"] = torch.empty((E, 16), device=dev)
    out["dD"] = torch.empty(E, device=dev)
    out["ddt_b"] = torch.empty(E, device=dev)
    dims = bd.make_dims(64, E, dtype=torch.float32)
    ws = torch.empty(bd.reverse_scan_backward_workspace_size(dims, B, L, 0), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def call():
        bd.reverse_scan_backward(d["u"], d["z"], d["dt_raw"], d["bc"], d["A_log"], d["D"], d["dt_b"], d["dy"],
                                 out["du"], out["dz"], out["ddt_raw"], out["dbc"], out["dA_log"], out["dD"],
                                 out["ddt_b"], dims, B, L, workspace=ws, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    st, fl = bd.get_device_status(ws, stream)
    if st != 0:
        raise RuntimeError(f"device status {st} flags {fl}")
    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    barrier()
    torch.cuda.synchronize()
    if rank == 0:
        clocks.start()
        time.sleep(0.3)
    t0.record(stream)
    for _ in range(K):
        call()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop() if rank == 0 else None
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev)

    e2e = None
    if not args.no_e2e:
        ins = {k: host[k].pin_memory() for k in ("u", "z", "dt_raw", "bc", "dy")}
        outs = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in out.items()}
        h2d = sum(v.numel() * v.element_size() for v in ins.values())
        d2h = sum(v.numel() * v.element_size() for v in outs.values())

        def e2e_step():
            for k, v in ins.items():
                d[k].copy_(v, non_blocking=True)
            call()
            for k, v in outs.items():
                v.copy_(out[k], non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ke = max(1, min(K, 5))
        e0.record(stream)
        for _ in range(ke):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        ms_e = max_over_ranks(e0.elapsed_time(e1), world, dev)
        # pipelined: inputs in, the call, gradients out on three streams over
        # E2E_BUFFERS device sets (the calls share one workspace on their stream)
        nb = E2E_BUFFERS
        sets = [({k: torch.empty_like(d[k]) for k in ins}, {k: torch.empty_like(v) for k, v in out.items()})
                for _ in range(nb)]
        s_in, s_fw, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(nb)]
        ev_fw = [torch.cuda.Event() for _ in range(nb)]
        ev_out = [torch.cuda.Event() for _ in range(nb)]

        def pipelined(n, t_start=None, t_end=None):
            if t_start is not None:
                t_start.record(s_in)
                s_fw.wait_event(t_start)
                s_out.wait_event(t_start)
            for k in range(n):
                i = k % nb
                di, do = sets[i]
                if k >= nb:
                    s_in.wait_event(ev_out[i])
                with torch.cuda.stream(s_in):
                    for key, v in ins.items():
                        di[key].copy_(v, non_blocking=True)
                ev_in[i].record(s_in)
                s_fw.wait_event(ev_in[i])
                bd.reverse_scan_backward(di["u"], di["z"], di["dt_raw"], di["bc"], d["A_log"], d["D"], d["dt_b"],
                                         di["dy"], do["du"], do["dz"], do["ddt_raw"], do["dbc"], do["dA_log"],
                                         do["dD"], do["ddt_b"], dims, B, L, workspace=ws, stream=s_fw)
                ev_fw[i].record(s_fw)
                s_out.wait_event(ev_fw[i])
                with torch.cuda.stream(s_out):
                    for key, v in outs.items():
                        v.copy_(do[key], non_blocking=True)
                ev_out[i].record(s_out)
            if t_end is not None:
                s_out.wait_stream(s_in)
                s_out.wait_stream(s_fw)
                t_end.record(s_out)

        pipelined(nb)
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        kp = max(nb + 1, min(K, 8))
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        pipelined(kp, p0, p1)
        torch.cuda.synchronize()
        barrier()
        ms_p = max_over_ranks(p0.elapsed_time(p1), world, dev)
        del sets
        e2e = {"value": round(whole_job_rate(M, world, kp, ms_p), 1), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": kp,
               "serial_value": round(whole_job_rate(M, world, ke, ms_e), 1),
               "api": "r2l_reverse_scan_backward via binding, pinned host inputs and gradients",
               "device_buffers": nb,
               "schedule": f"pipelined: copy-in, gradient and copy-out of successive steps on three streams over "
                           f"{nb} device buffer sets, one workspace (serial_value: one stream)"}
    if rank != 0:
        return None
    peaks, peak_kind = load_peaks()
    per_call = ms / K
    nbytes = bwd_bytes_per_token(E) * M
    achieved = nbytes / (per_call * 1e-3) / 1e9
    tag = f"scanbwd-B{B}-L{L}-E{E}"
    line = {
        "metric": BWD_METRIC, "value": round(whole_job_rate(M, world, K, ms), 1), "unit": "tokens/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": round(per_call, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded: u, z, dy ~ N(0,1); B, C ~ N(0,1); dt_raw ~ N(0,0.1) around a "
                "logUniform[1e-3,1e-1] step; A=-(1..16); D=1)",
        "config": {"workload": f"reverse-scan gradient fp32 B={B} L={L} E={E} N=16", "B": B, "L": L,
                   "d_inner": E, "d_state": 16, "chunk_tokens": 16,
                   "path": ("one 32-channel block walks each sequence, H checkpoints every 16 positions"
                            if bwd_walks_sequences(B, E) else "chunks of 16 positions with H and G carries"),
                   "l2": "inputs larger than L2 (~4 GB read and written per step), no flush",
                   "parallelism": f"dp{world}: one independent batch per GPU, no collective"},
        "roofline": {"kernel": f"r2l_reverse_scan_backward (the {bwd_launches(B, E)} launches of one call)",
                     "bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(achieved / peaks["hbm_gbs"], 4),
                     "peak_source": f"{peak_kind} HBM copy", "algorithmic_per_launch": nbytes,
                     "bytes_per_token": bwd_bytes_per_token(E), "ms_per_launch": round(per_call, 4),
                     "traffic": read_traffic("scan_bwd", tag)},
        "gpu_launches": bwd_launches(B, E) * K, "clocks": clk, "e2e": e2e, "source_sha": source_sha(),
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_backward(host, B, L, E)
    return line


def cpu_baseline_backward(host, B, L, E, n=256):
    """The float64 gradient oracle, as it stands, on a bounded sample: the
    first n positions of sequence 0, all channels."""
    import oracle as O
    from reverse_selective_ssm_b200 import synthetic as S
    f = lambda k: S.to_f64(host[k][:n])
    bc = f("bc")
    t = time.perf_counter()
    O.reverse_scan_backward(f("u"), f("dt_raw"), S.to_f64(host["dt_b"]), S.to_f64(host["A_log"]), bc[:, :16],
                            bc[:, 16:], S.to_f64(host["D"]), f("z"), f("dy"))
    dt = time.perf_counter() - t
    return {"value": round(n / dt, 2), "unit": "tokens/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"positions 0..{n - 1} of sequence 0, all {E} channels, numpy float64 gradient oracle, "
                      f"{dt:.1f} s"}


def run_reference_backward(args, rank, world):
    """The gradient oracle timed on the host cores, each step a bounded sample
    (the first 256 positions of one sequence, all channels)."""
    if rank != 0:
        return None
    from reverse_selective_ssm_b200 import synthetic as S
    B, L, E = args.batch or 8, args.seq or 4096, 4096
    host = S.make_scan_bwd_case(B, L, E, seed=64)
    for _ in range(args.warmup):
        cpu_baseline_backward(host, B, L, E)
    t = time.perf_counter()
    for _ in range(args.steps):
        cpu_baseline_backward(host, B, L, E)
    dt = time.perf_counter() - t
    v = round(256 * args.steps / dt, 2)
    cb = {"value": v, "unit": "tokens/s", "cores": _blas_threads(), "kind": "oracle",
          "sample": "per step positions 0..255 of sequence 0, all 4096 channels, numpy float64 gradient oracle"}
    return {"metric": BWD_METRIC, "value": v, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": f"reverse-scan gradient B={B} L={L} E={E} N=16"}, "cpu_baseline": cb,
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------- whole-hook gradient

HOOK_BWD_METRIC = "R2L sidecar hook backward tokens/sec at B=8,L=4096,d=2048 (dh, ds and every parameter gradient)"


def hook_bwd_gemm_flops(case):
    """Tensor-core work of one r2l_sidecar_backward call: the recomputed
    forward's projections, then for out_proj, dt_proj, x_proj and in_proj an
    input-gradient and a weight-gradient GEMM of the same size each."""
    d, E, R, N = case.dims.d_model, case.dims.d_inner, case.dims.dt_rank, case.dims.d_state
    T = float(case.valid_tokens)
    fwd = 2.0 * T * (d * 2 * E + E * (R + 2 * N) + R * E + E * d)
    return fwd + 2.0 * fwd


def hook_bwd_launches(case):
    """Kernels one r2l_sidecar_backward call launches at the bench's shapes
    (as the ncu launch list shows them): the recomputed forward (6, its scan
    storing the scan gradient's H checkpoints) and dt_raw, 4 weight
    transposes, the gate and LayerNorm gradient (4, or 2 without LayerNorm),
    the scan gradient, and 19 more: the padding rows of 3 activations zeroed,
    per projection its input-gradient and weight-gradient GEMMs (dt_proj and
    x_proj with a split-K sum) and operand conversions, the conv gradient and
    its column sum, dh = dh+ + dx, and h transposed; on the chunked scan
    gradient also ddt_raw and dz converted to bf16 (the walk writes them so)."""
    w = case.weights[0]
    ln = 4 if w.get("ln_w") is not None else 2
    # (on the walk along each sequence the recomputed forward scan stores the H
    # checkpoints of sequences whose length is a multiple of 16, and the
    # gradient's checkpoint pass launches but fills only the others)
    walk = bwd_walks_sequences(case.B, case.dims.d_inner)
    return 6 + 1 + 4 + ln + bwd_launches(case.B, case.dims.d_inner) + 19 + (0 if walk else 2)


def run_hook_e2e_pipelined(case, w, dims, lengths, ws, h_pin, g_pin, dh_pin, ds_pin, outs, K, warmup, barrier,
                           world, dev):
    """The hook gradient through host buffers as a pipelined loop (as run_e2e
    does for the forward): step k's hidden states and dh+ go in on one stream,
    its r2l_sidecar_backward runs on a second (all calls on that stream, so they
    share one workspace) and dh, ds and every parameter gradient come back on a
    third, over E2E_BUFFERS device buffer sets.  Returns (ms for the timed
    steps, their count)."""
    import torch
    from reverse_selective_ssm_b200 import binding as bd
    nb = E2E_BUFFERS
    sets = []
    for _ in range(nb):
        sets.append({"h": torch.empty(h_pin.shape, dtype=h_pin.dtype, device=dev),
                     "g": torch.empty(g_pin.shape, dtype=g_pin.dtype, device=dev),
                     "dh": torch.empty(dh_pin.shape, dtype=torch.float32, device=dev),
                     "ds": torch.zeros(4, dtype=torch.float32, device=dev),
                     "grads": bd.alloc_grads(w, dev)})
    s_in, s_fw, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(nb)]
    ev_fw = [torch.cuda.Event() for _ in range(nb)]
    ev_out = [torch.cuda.Event() for _ in range(nb)]

    def pipelined(n, t_start=None, t_end=None):
        if t_start is not None:
            t_start.record(s_in)
            s_fw.wait_event(t_start)
            s_out.wait_event(t_start)
        for k in range(n):
            i = k % nb
            b = sets[i]
            if k >= nb:
                s_in.wait_event(ev_out[i])          # set i is free once step k-nb is copied out
            with torch.cuda.stream(s_in):
                b["h"].copy_(h_pin, non_blocking=True)
                b["g"].copy_(g_pin, non_blocking=True)
            ev_in[i].record(s_in)
            s_fw.wait_event(ev_in[i])
            bd.sidecar_backward(b["h"], w, dims, case.s[0], b["g"], b["grads"], lengths, workspace=ws, stream=s_fw,
                                dh=b["dh"], ds=b["ds"])
            ev_fw[i].record(s_fw)
            s_out.wait_event(ev_fw[i])
            with torch.cuda.stream(s_out):
                dh_pin.copy_(b["dh"], non_blocking=True)
                ds_pin.copy_(b["ds"][:1], non_blocking=True)
                for key, v in outs.items():
                    v.copy_(b["grads"][key], non_blocking=True)
            ev_out[i].record(s_out)
        if t_end is not None:
            s_out.wait_stream(s_in)
            s_out.wait_stream(s_fw)
            t_end.record(s_out)

    pipelined(max(nb, warmup))
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    kp = max(nb + 1, min(K, 10))
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pipelined(kp, p0, p1)
    torch.cuda.synchronize()
    barrier()
    return max_over_ranks(p0.elapsed_time(p1), world, dev), kp


def run_hook_backward(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from reverse_selective_ssm_b200 import binding as bd
    from reverse_selective_ssm_b200 import synthetic as S

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    bd.load()
    case = S.make_case(args.config, B=args.batch, L=args.seq, shard=(rank, world))
    dims = bd.dims_of(case.dims, case.dtype)
    h = case.h.to(dev)
    w = bd.weights_to_device(case.weights[0], dev)
    grads = bd.alloc_grads(w, dev)
    lengths = None if case.lengths is None else case.lengths.to(dev)
    g = torch.Generator().manual_seed(90 + case.meta["first_sequence"])
    dh_host = torch.randn(case.h.shape, generator=g, dtype=torch.float32)
    dh_out = dh_host.to(dev)
    ws = torch.empty(bd.sidecar_backward_workspace_size(dims, case.B, case.L), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def call(x=h, gout=dh_out):
        return bd.sidecar_backward(x, w, dims, case.s[0], gout, grads, lengths, workspace=ws, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    st, fl = bd.get_device_status(ws, stream)
    if st != 0:
        raise RuntimeError(f"device status {st} flags {fl}")
    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    barrier()
    torch.cuda.synchronize()
    if rank == 0:
        clocks.start()
        time.sleep(0.3)
    t0.record(stream)
    for _ in range(K):
        call()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop() if rank == 0 else None
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev)

    # a training step of the hook: the training forward (h+ into its own
    # buffer, the intermediates and checkpoints left in the workspace), then the
    # gradient without recomputing the forward
    out_buf = torch.empty_like(h)
    sdims = bd.dims_of(case.dims, case.dtype, bd.R2L_FLAG_SAVED_FORWARD)

    def train_step(ev=None):
        if ev:
            ev[0].record(stream)
        bd.sidecar_forward_train(h, w, dims, case.s[0], lengths, workspace=ws, out=out_buf, stream=stream)
        if ev:
            ev[1].record(stream)
        bd.sidecar_backward(h, w, sdims, case.s[0], dh_out, grads, lengths, workspace=ws, stream=stream)
        if ev:
            ev[2].record(stream)

    for _ in range(max(2, args.warmup)):
        train_step()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    for k in range(K):
        train_step(evs[k])
    torch.cuda.synchronize()
    barrier()
    fwd_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = sum(e[1].elapsed_time(e[2]) for e in evs)
    step_ms = max_over_ranks(evs[0][0].elapsed_time(evs[-1][2]), world, dev)
    train = {"ms_per_step": round(step_ms / K, 4),
             "tokens_per_s": round(whole_job_rate(case.valid_tokens, world, K, step_ms), 1),
             "forward_ms": round(fwd_ms / K, 4), "backward_ms": round(bwd_ms / K, 4),
             "api": "r2l_sidecar_forward_train, then r2l_sidecar_backward with R2L_FLAG_SAVED_FORWARD"}

    e2e = None
    if not args.no_e2e:
        # the hidden states and dh⁺ come from pinned host memory and dh, ds and every
        # parameter gradient go back, every step
        h_pin, g_pin = case.h.pin_memory(), dh_host.pin_memory()
        outs = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in grads.items() if v is not None}
        dh_pin = torch.empty(case.h.shape, dtype=torch.float32).pin_memory()
        ds_pin = torch.empty(1, dtype=torch.float32).pin_memory()
        h2d = h_pin.numel() * h_pin.element_size() + g_pin.numel() * g_pin.element_size()
        d2h = sum(v.numel() * v.element_size() for v in outs.values()) + dh_pin.numel() * 4 + 4

        def e2e_step():
            h.copy_(h_pin, non_blocking=True)
            dh_out.copy_(g_pin, non_blocking=True)
            dh, ds = call()
            dh_pin.copy_(dh, non_blocking=True)
            ds_pin.copy_(ds, non_blocking=True)
            for k, v in outs.items():
                v.copy_(grads[k], non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ke = max(1, min(K, 5))
        e0.record(stream)
        for _ in range(ke):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        ms_e = max_over_ranks(e0.elapsed_time(e1), world, dev)
        ms_p, kp = run_hook_e2e_pipelined(case, w, dims, lengths, ws, h_pin, g_pin, dh_pin, ds_pin, outs, K,
                                          args.warmup, barrier, world, dev)
        e2e = {"value": round(whole_job_rate(case.valid_tokens, world, kp, ms_p), 1), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": kp,
               "serial_value": round(whole_job_rate(case.valid_tokens, world, ke, ms_e), 1),
               "api": "r2l_sidecar_backward via binding, pinned host hidden states, dh+ and gradients",
               "device_buffers": E2E_BUFFERS,
               "schedule": f"pipelined: copy-in, gradient and copy-out of successive steps on three streams over "
                           f"{E2E_BUFFERS} device buffer sets, one workspace (serial_value: one stream)"}
    if rank != 0:
        return None
    peaks, peak_kind = load_peaks()
    per_call = ms / K
    flops = hook_bwd_gemm_flops(case)
    tpeak, tnote = tensor_peak(peaks, peak_kind, clk, ms)
    achieved = flops / (per_call * 1e-3) / 1e12
    line = {
        "metric": HOOK_BWD_METRIC if args.config == 2 else f"R2L sidecar hook backward tokens/sec, {case.name}",
        "value": round(whole_job_rate(case.valid_tokens, world, K, ms), 1), "unit": "tokens/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": round(per_call, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (the workload's seeded hidden states and weights; dh+ ~ N(0, 1))",
        "config": {"workload": case.name, "B": case.B, "L": case.L, "global_batch": case.meta["global_batch"],
                   "s": case.s[0], "l2": "inputs larger than L2 (~10 GB of workspace touched per step), no flush",
                   "parallelism": f"dp{world}: rank r runs sequences [r*{case.B}, (r+1)*{case.B}) of the global "
                                  f"batch; parameter gradients would then take one all-reduce (not part of this "
                                  f"entry point)"},
        "roofline": {"kernel": "r2l_sidecar_backward (its tcgen05 GEMMs: the recomputed forward, then an input- "
                               "and a weight-gradient GEMM per projection) over the whole call",
                     "bound": "tensor", "achieved": round(achieved, 2), "peak": tpeak, "unit": "TFLOP/s",
                     "frac": round(achieved / tpeak, 4), "peak_source": tnote, "algorithmic_per_launch": flops,
                     "ms_per_launch": round(per_call, 4), "traffic": None},
        "gpu_launches": hook_bwd_launches(case) * K, "clocks": clk, "e2e": e2e, "source_sha": source_sha(),
        "train_step": train,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_hook_backward(case, dh_host)
    return line


def cpu_baseline_hook_backward(case, dh_host, n=128):
    """The whole-hook gradient oracle, as it stands, timed on a bounded
    sample: the last n positions of sequence 0 run as a sequence of their
    own (a timing sample only: the gradient at a position also depends on
    dh+ at the positions before it)."""
    import oracle as O
    from reverse_selective_ssm_b200 import synthetic as S
    L = case.L
    h = S.to_f64(case.h[0:1, L - n:])
    t = time.perf_counter()
    O.sidecar_backward_batch(h, S.weights_f64(case.weights[0]), case.s[0], S.to_f64(dh_host[0:1, L - n:]))
    dt = time.perf_counter() - t
    return {"value": round(n / dt, 2), "unit": "tokens/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"the last {n} positions of sequence 0 as a sequence of their own, numpy float64 "
                      f"whole-hook gradient oracle, {dt:.1f} s"}


# ---------------------------------------------------------------- reference arm

def run_reference(args, rank, world):
    """The oracle timed on the host cores, each step a bounded sample: the last
    512 positions of one sequence (exact for those positions, since the output
    at i depends on positions ≥ i only)."""
    if rank != 0:
        return None
    import numpy as np
    import oracle as O
    from reverse_selective_ssm_b200 import synthetic as S
    case = S.make_case(args.config)
    h = S.to_f64(case.h)
    ws = [S.weights_f64(w) for w in case.weights]
    span = min(512, case.L)

    def step(k):
        b = k % case.B
        n = case.L if case.lengths is None else int(case.lengths[b])
        sub = h[b:b + 1, max(0, n - span):n]
        if len(ws) == 1:
            O.sidecar_forward(sub, ws[0], case.s[0], None, "bf16")
        else:
            O.sidecar_stack(sub, ws, case.s, None, "bf16")
        return sub.shape[1]

    for k in range(args.warmup):
        step(k)
    t = time.perf_counter()
    tokens = 0
    for k in range(args.steps):
        tokens += step(k)
    dt = time.perf_counter() - t
    v = round(tokens / dt, 2)
    sample = f"per step the last {span} positions of one sequence, numpy float64 oracle"
    return {"metric": METRIC if args.config == 2 else f"R2L sidecar tokens/sec, {case.name}", "value": v, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": case.name, "B": case.B, "L": case.L, "hooks": len(ws)},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": _blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_reference_hook_backward(args, rank, world):
    """The whole-hook gradient oracle timed on the host cores, each step the
    bounded sample of cpu_baseline_hook_backward."""
    if rank != 0:
        return None
    import torch
    from reverse_selective_ssm_b200 import synthetic as S
    case = S.make_case(args.config, B=args.batch, L=args.seq)
    g = torch.Generator().manual_seed(90)
    dh_host = torch.randn(case.h.shape, generator=g, dtype=torch.float32)
    n = min(128, case.L)
    for _ in range(args.warmup):
        cpu_baseline_hook_backward(case, dh_host, n)
    t = time.perf_counter()
    for _ in range(args.steps):
        cpu_baseline_hook_backward(case, dh_host, n)
    dt = time.perf_counter() - t
    v = round(n * args.steps / dt, 2)
    cb = {"value": v, "unit": "tokens/s", "cores": _blas_threads(), "kind": "oracle",
          "sample": f"per step the last {n} positions of sequence 0 as a sequence of their own, numpy float64 "
                    f"whole-hook gradient oracle"}
    return {"metric": HOOK_BWD_METRIC if args.config == 2 else f"R2L sidecar hook backward tokens/sec, {case.name}",
            "value": v, "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": case.name, "B": case.B, "L": case.L}, "cpu_baseline": cb,
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main(argv=None):
    args = parse_args(argv)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference_backward(args, rank, world) if args.scan_backward else \
            run_reference_hook_backward(args, rank, world) if args.hook_backward else run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0
    import torch
    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        fn = run_scan_backward if args.scan_backward else run_hook_backward if args.hook_backward else run_ours
        line = fn(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
