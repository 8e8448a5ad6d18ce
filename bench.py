"""Benchmark of the DiT attention hot path (one line of JSON on rank 0).

One step = one pass of the hot path for one denoising step of the 77-frame
window (B=1, H=40, D=128, latent grid 20 x 30 x 52 -> S = 31200):
  1. 3D RoPE of Q and K, in place                       regen_rope3d
  2. self-attention, 31200 x 31200                      regen_attn_fwd
  3. cross-attention of the 31200 video tokens to the 1560 reference-frame
     and 512 conditioning tokens, one softmax over both key buffers in one
     launch                                             regen_attn_fwd_kv2
Each step rotates the Q/K left by the previous step again: the same work on
the same shapes. Beside it, timed in rounds alternating with it on the same
box: the step with the RoPE fused into the attention's Q load
(regen_attn_fwd_rope3d); and the cross-attention paths on the step's shapes,
including the Ring form (one call per key block merged by regen_lse_merge)
and one call over the concatenated keys.

value = attention FLOPs of the step (4*B*H*Sq*Skv*D, self + cross) / device
time of the step, summed over ranks (weak scaling: every rank runs its own
window). Inputs (320 MB per tensor) exceed the 126 MB L2, so no L2 flush is
used between steps.

--impl reference times the CPU fp64 oracle instead (bounded samples of rows).
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

METRIC = "attention fwd TFLOP/s and % of B200 BF16 dense peak at S=31200,H=40,D=128"
SELF = "win77_s31200"
CROSS = "cross_s31200_kv2072"
N_REF = 1560          # reference-frame latent tokens (one 30 x 52 latent frame)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="native", choices=["native", "reference"])
    p.add_argument("--e2e-steps", type=int, default=40)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=15.0)
    p.add_argument("--configs", action="store_true",
                   help="instead of the step: CUDA-event medians of every workload's kernels (1 GPU)")
    p.add_argument("--profile-case", choices=["attn", "fused", "kv2", "rope", "merge", "bwd", "fp8", "proj", "proj_ref"],
                   default=None,
                   help="instead of the step: a short, bounded launch sequence of one kernel for ncu (no timing)")
    p.add_argument("--heads", type=int, default=8, help="--profile-case: heads")
    p.add_argument("--seq", type=int, default=31200, help="--profile-case: query tokens (31200, 10920 or 1024)")
    p.add_argument("--kv", type=int, default=0, help="--profile-case: key count (default --seq; kv2: 1560 + rest)")
    p.add_argument("--dim", type=int, default=128, help="--profile-case: head dimension")
    p.add_argument("--iters", type=int, default=2, help="--profile-case: calls of the kernel")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def dist_env():
    """(rank, world, local_rank) from the torchrun environment."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def max_over_ranks(x: float, world: int, device) -> float:
    """Max of a per-rank scalar over all ranks (the step time every rank reports)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(flops_per_rank: float, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank runs its own replica (weak scaling)."""
    return world * flops_per_rank / (ms_per_step * 1e-3) / 1e12


def replica_inputs(workload, rank: int):
    """The seeded inputs of this rank's replica (seed offset = rank)."""
    from dit_attention_b200 import synth
    return synth.make_inputs(workload, seed_offset=rank)


def step_flops():
    from dit_attention_b200 import synth
    s = synth.WORKLOADS[SELF]
    c = synth.WORKLOADS[CROSS]
    return s.flops, c.flops


# ------------------------------------------------------------ clocks ---

class ClockSampler:
    """SM clock, board power and clock-event reasons of this process's GPU,
    sampled every 20 ms during the timed region by read-only NVML queries
    (nvidia-smi on the same GPU if NVML cannot be loaded). The GPU is found by
    its UUID: NVML numbers every GPU of the machine and ignores
    CUDA_VISIBLE_DEVICES, so an index could name another process's GPU."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))
    SMI_FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
                  "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                  "clocks_event_reasons.hw_power_brake_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        import torch
        u = str(torch.cuda.get_device_properties(device).uuid)
        self.uuid = u if u.startswith("GPU-") else "GPU-" + u
        self.samples = []          # (sm_mhz, power_w, set of reason names)
        self.sm_max = None
        self.source = None
        self._stop = threading.Event()
        self._first = threading.Event()
        self.proc = self.t = None
        self.power_kind = "1 s average"

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByUUID(self.uuid)
            self.sm_max = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            masks = [(n, getattr(pynvml, c)) for n, c in self.REASONS if hasattr(pynvml, c)]
            self.source = "nvml"
            self.power_kind = "instant" if self._instant_power(pynvml, h) is not None else "1 s average"
            self.t = threading.Thread(target=self._poll_nvml, args=(pynvml, h, masks), daemon=True)
        except Exception:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", "-i", self.uuid, f"--query-gpu={self.SMI_FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", "100"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except OSError:
                return
            self.source = "nvidia-smi"
            self.t = threading.Thread(target=self._read_smi, daemon=True)
        self.t.start()
        self._first.wait(timeout=10.0)   # the first sample precedes the timed region

    @staticmethod
    def _instant_power(pynvml, h):
        """Board power now, in W (the plain power query averages over a second,
        longer than a short timed region); None where the field is missing."""
        try:
            v = pynvml.nvmlDeviceGetFieldValues(h, [pynvml.NVML_FI_DEV_POWER_INSTANT])[0]
            if v.nvmlReturn != 0:
                return None
            raw = {0: "dVal", 1: "uiVal", 2: "ulVal", 3: "ullVal", 4: "sllVal"}.get(v.valueType)
            return float(getattr(v.value, raw)) / 1000.0 if raw else None
        except Exception:
            return None

    def _poll_nvml(self, pynvml, h, masks):
        while not self._stop.is_set():
            try:
                sm = float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                pw = self._instant_power(pynvml, h) if self.power_kind == "instant" else None
                if pw is None:
                    pw = pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0
                bits = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((sm, pw, {n for n, m in masks if bits & m}))
            except Exception:
                pass
            self._first.set()
            self._stop.wait(0.02)

    def _read_smi(self):
        names = [n for n, _ in self.REASONS]
        for line in self.proc.stdout:
            f = [x.strip() for x in line.split(",")]
            try:
                sm, self.sm_max, pw = float(f[0]), float(f[1]), float(f[2])
            except (ValueError, IndexError):
                continue
            self.samples.append((sm, pw, {n for n, v in zip(names, f[3:8]) if v.lower() == "active"}))
            self._first.set()

    def stop(self):
        if self.t is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.t.join(timeout=5)
        smax = self.sm_max
        busy = [x for x in self.samples if smax and x[0] > 0.3 * smax] or self.samples
        reasons = set().union(*(x[2] for x in self.samples)) if self.samples else set()
        return {"sm_mhz": statistics.median(x[0] for x in busy) if busy else None,
                "sm_max_mhz": smax, "reasons": sorted(reasons), "samples": len(self.samples),
                "power_w": statistics.median(x[1] for x in busy) if busy else None,
                "power_kind": self.power_kind, "source": self.source}


def step_config(world):
    """The workload one bench step runs (both arms report it)."""
    from dit_attention_b200 import synth
    ws, wc = synth.WORKLOADS[SELF], synth.WORKLOADS[CROSS]
    T, Hh, Ww = ws.grid
    return {
        "workload": "win77_s31200 3D RoPE + self-attention, cross-attention to 1560 reference + 512 "
                    "conditioning tokens under one softmax (one denoising step of the 77-frame window)",
        "B": ws.B, "H": ws.H, "S": ws.Sq, "D": ws.D, "Skv_cross": [N_REF, wc.Skv - N_REF],
        "latent_grid": [T, Hh, Ww], "scale": 1.0 / math.sqrt(ws.D),
        "l2": "inputs larger than L2 (320 MB per tensor vs 126 MB); no flush",
        "parallelism": f"replicas{world}",
    }


# ------------------------------------------------------- native (GPU) ---

def traffic_from_profile():
    """DRAM bytes per launch of the self-attention kernel from the committed ncu
    summary, if it was taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "attn_fwd_win77_s31200_traffic.txt")
    src = os.path.join(ROOT, "dit_attention_b200", "csrc", "attn_fwd.cuh")
    if not os.path.exists(path):
        return None
    kv = {}
    for line in open(path):
        if "=" in line and not line.startswith("#"):
            a, b = line.split("=", 1)
            kv[a.strip()] = b.strip()
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    if kv.get("kernel_source_sha256") != sha:
        return None
    try:
        return float(kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def tensor_roofline(kernel, flops, ms, region_ms, clk, pk, pk_src, peak_mult=1.0, peak_note="bf16"):
    """Roofline of a tensor-core kernel: achieved = algorithmic FLOPs per launch
    / its event-timed duration, against the measured burst peak when the timed
    region is short (under 3 s: the part runs at its boost clock before the
    power cap settles) or the sustained one otherwise; also the fractions of
    both peaks, of the sustained peak scaled to this run's SM clock, and the
    cycles per launch at the run's median SM clock (comparable across boxes)."""
    burst = float(pk["bf16_tflops"]) * peak_mult
    sust = float(pk.get("bf16_tflops_sustained") or pk["bf16_tflops"]) * peak_mult
    achieved = flops / (ms * 1e-3) / 1e12
    short = region_ms < 3000.0
    peak = burst if short else sust
    d = {"bound": "tensor", "kernel": kernel, "achieved": round(achieved, 2), "peak": round(peak, 1),
         "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
         "peak_source": (f"{pk_src} {'bf16_tflops (burst)' if short else 'bf16_tflops_sustained'}"
                         f"{'' if peak_mult == 1.0 else ' x %g (%s)' % (peak_mult, peak_note)}: the timed region "
                         f"lasts {region_ms / 1000:.2f} s"),
         "frac_of_burst_peak": round(achieved / burst, 4), "frac_of_sustained_peak": round(achieved / sust, 4),
         "frac_of_nominal": round(achieved / (2250.0 * peak_mult), 4),
         "algorithmic_flops_per_launch": flops, "ms_per_launch": round(ms, 4)}
    mhz = clk.get("sm_mhz") if clk else None
    if mhz:
        d["sm_mhz_median"] = mhz
        d["cycles_per_launch"] = int(round(ms * 1e-3 * mhz * 1e6))
        sust_mhz = (pk.get("clocks_under_load") or {}).get("sm_mhz_median")
        if sust_mhz:
            d["frac_of_sustained_peak_at_this_clock"] = round(achieved / (sust * mhz / float(sust_mhz)), 4)
    return d


def timed_region(fn, n, stream, world, dev, barrier, with_clocks=True):
    """n calls of fn between two events on `stream` (barrier + synchronize on
    both sides), max over ranks; returns (ms per call, clocks dict, region ms)."""
    import torch
    clocks = ClockSampler(dev) if with_clocks else None
    barrier()
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop() if clocks else {}
    barrier()
    total = max_over_ranks(e0.elapsed_time(e1), world, dev)
    return total / n, clk, total


def run_native(args, rank, world, local_rank):
    import torch
    import dit_attention_b200 as rg
    from dit_attention_b200 import synth

    torch.cuda.set_device(local_rank)
    rg.load()
    dev = torch.device("cuda", local_rank)
    ws = synth.WORKLOADS[SELF]
    wc = synth.WORKLOADS[CROSS]

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)

    q, k, v = replica_inputs(ws, rank)
    qc, kc, vc = replica_inputs(wc, rank)
    host = {
        "q": q, "k": k, "v": v, "qc": qc,
        "kr": np.ascontiguousarray(kc[:, :, :N_REF]), "vr": np.ascontiguousarray(vc[:, :, :N_REF]),
        "kx": np.ascontiguousarray(kc[:, :, N_REF:]), "vx": np.ascontiguousarray(vc[:, :, N_REF:]),
    }
    d = {name: to_dev(a) for name, a in host.items()}
    B, H, S, D = ws.B, ws.H, ws.Sq, ws.D
    n_ctx = wc.Skv - N_REF
    out = torch.empty_like(d["q"])
    lse = torch.empty((B, H, S), dtype=torch.float32, device=dev)
    oc = torch.empty_like(d["qc"])
    lc = torch.empty((B, H, S), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    scale = 1.0 / math.sqrt(D)
    T, Hh, Ww = ws.grid
    rope_ws_bytes = rg.regen_attn_fwd_rope3d_workspace_bytes(B, H, T, Hh, Ww, D)
    rope_ws = torch.empty(rope_ws_bytes, dtype=torch.uint8, device=dev)

    # One step: the 3D RoPE of Q and K in place, the self-attention, and the
    # cross-attention to the reference-frame and conditioning keys in one
    # launch over the two key buffers. In the timed loop each step rotates the
    # Q and K the previous step left: the same work on the same shapes.
    names = ["rope3d", "attn_self", "attn_cross_kv2"]
    LAUNCHES_PER_STEP = 3
    outs0 = dict(out=out, lse=lse, oc=oc, lc=lc)
    q_raw, k_raw = d["q"].clone(), d["k"].clone()   # the unrotated inputs, for the fused step and the snapshot

    def step(ev=None, inp=None, o=None):
        inp = d if inp is None else inp
        o = outs0 if o is None else o

        def mark(i):
            if ev is not None:
                ev[i].record(stream)
        mark(0)
        rg.regen_rope3d(inp["q"], inp["k"], T, Hh, Ww, ws.theta, B, H, D, sh)
        mark(1)
        rg.regen_attn_fwd(inp["q"], inp["k"], inp["v"], o["out"], o["lse"], B, H, S, S, D, scale, sh)
        mark(2)
        rg.regen_attn_fwd_kv2(inp["qc"], inp["kr"], inp["vr"], inp["kx"], inp["vx"], o["oc"], o["lc"], B, H, S,
                              N_REF, n_ctx, D, scale, sh)
        mark(3)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # ---- device-resident timing: K steps between two events, per-call events inside
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(dev)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier()
    ms_total = max_over_ranks(t0.elapsed_time(t1), world, dev)
    per_kernel = {n: 0.0 for n in names}
    for i in range(args.steps):
        for j, n in enumerate(names):
            per_kernel[n] += evs[i][j].elapsed_time(evs[i][j + 1])
    per_kernel = {n: t / args.steps for n, t in per_kernel.items()}

    f_self, f_cross = step_flops()
    flops_step = f_self + f_cross
    ms_step = ms_total / args.steps
    value = aggregate_tflops(flops_step, world, ms_step)

    # ---- the same step with the RoPE fused into the attention's Q load
    # (regen_attn_fwd_rope3d: the table, the K pass into workspace, the attention
    # with Q rotated in shared memory; q and k untouched), timed in rounds
    # alternating with the pre-pass step above, on the same box and clocks.
    fused_names = ["attn_self_rope_fused", "attn_cross_kv2"]

    def step_fused(ev=None):
        def mark(i):
            if ev is not None:
                ev[i].record(stream)
        mark(0)
        rg.regen_attn_fwd_rope3d(q_raw, k_raw, d["v"], out, lse, B, H, S, S, D, scale, sh, T, Hh, Ww, ws.theta,
                                 rope_ws, rope_ws_bytes)
        mark(1)
        rg.regen_attn_fwd_kv2(d["qc"], d["kr"], d["vr"], d["kx"], d["vx"], oc, lc, B, H, S, N_REF, n_ctx, D, scale,
                              sh)
        mark(2)

    n_alt = max(3, min(args.steps, 10))
    for _ in range(args.warmup):
        step_fused()
    fused_ms, pre_ms, fused_k = [], [], {n: [] for n in fused_names}
    for rnd in range(3):
        for which in ((0, 1) if rnd % 2 == 0 else (1, 0)):
            if which == 0:
                ms, _, _ = timed_region(step, n_alt, stream, world, dev, barrier, with_clocks=False)
                pre_ms.append(ms)
            else:
                fev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_alt)]
                ms, _, _ = timed_region(lambda it=iter(fev): step_fused(next(it)), n_alt, stream, world, dev,
                                        barrier, with_clocks=False)
                fused_ms.append(ms)
                for j, n in enumerate(fused_names):
                    fused_k[n].append(sum(e[j].elapsed_time(e[j + 1]) for e in fev) / n_alt)

    # One more step on the unrotated inputs: its out/lse serve the CPU leg's
    # accuracy check (rank 0 only, when that leg runs; the oracle gets the
    # host's unrotated q, k and applies the RoPE itself) and the backward below.
    d["q"].copy_(q_raw)
    d["k"].copy_(k_raw)
    step()
    torch.cuda.synchronize()
    snap = None
    if rank == 0 and not args.no_cpu_baseline:
        snap = dict(q=host["q"], k=host["k"], v=host["v"],
                    out=out.contiguous().view(torch.int16).cpu().numpy().view(np.uint16), lse=lse.cpu().numpy(),
                    scale=scale, grid=ws.grid, theta=ws.theta)

    # ---- cross-attention paths on the step's shapes: the one-launch two-source
    # call (the step's), the two key blocks as separate calls merged by
    # regen_lse_merge (the Ring form of the same result), and one call over the
    # keys concatenated in one buffer.
    oa, ob = torch.empty_like(oc), torch.empty_like(oc)
    la, lb = torch.empty_like(lc), torch.empty_like(lc)
    kcat = torch.cat([d["kr"], d["kx"]], dim=2).contiguous()
    vcat = torch.cat([d["vr"], d["vx"]], dim=2).contiguous()
    cross_fns = {
        "kv2": lambda: rg.regen_attn_fwd_kv2(d["qc"], d["kr"], d["vr"], d["kx"], d["vx"], oc, lc, B, H, S, N_REF,
                                             n_ctx, D, scale, sh),
        "ref_block": lambda: rg.regen_attn_fwd(d["qc"], d["kr"], d["vr"], oa, la, B, H, S, N_REF, D, scale, sh),
        "ctx_block": lambda: rg.regen_attn_fwd(d["qc"], d["kx"], d["vx"], ob, lb, B, H, S, n_ctx, D, scale, sh),
        "lse_merge": lambda: rg.regen_lse_merge(oa, la, ob, lb, oc, lc, B * H * S, D, sh),
        "concat_one_call": lambda: rg.regen_attn_fwd(d["qc"], kcat, vcat, oc, lc, B, H, S, wc.Skv, D, scale, sh),
    }
    cross_ms = {}
    for n, fn in cross_fns.items():
        for _ in range(args.warmup):
            fn()
        cross_ms[n] = timed_region(fn, max(5, min(args.steps, 20)), stream, world, dev, barrier,
                                   with_clocks=False)[0]
    del oa, ob, la, lb, kcat, vcat

    # ---- backward: the gradient step of the same window (the decoder is trained by
    # distillation). dO synthetic; the forward's out/lse of the snapshot step
    # (its q, k rotated once: the inputs the gradient kernels take).
    # Self: regen_attn_bwd then regen_rope3d_bwd on dq, dk (gradients w.r.t. the
    # unrotated Q, K). Cross: regen_attn_bwd_kv2 over both key sources with the
    # joint out/lse. Each gradient call is 3 launches.
    step_fused()          # cross out/lse again (the cross paths above overwrote them); same self out/lse
    bwd = run_backward(args, rg, synth, d, outs0, ws, wc, rank, dev, stream, world, barrier, to_dev)

    # ---- the projections around the attention of a 14B-class DiT block on the same
    # window: fused QKV projection (+ RMSNorm + RoPE) and the output projection.
    proj = run_proj(args, rg, synth, ws, dev, stream, world, barrier, to_dev, rank)

    # ---- the FP8 variant of the self-attention (on the rotated q, k): blockwise
    # E4M3 quantisation of Q, K, V (3 launches) and the E4M3 attention.
    fp8 = run_fp8(args, rg, d, ws, dev, stream, world, barrier)

    # ---- end to end: pinned host inputs -> device -> hot path -> outputs to pinned host
    pin = {n: torch.from_numpy(a.view(np.int16)).pin_memory() for n, a in host.items()}
    res_host = {"out": torch.empty(out.shape, dtype=torch.int16).pin_memory(),
                "lse": torch.empty(lse.shape, dtype=torch.float32).pin_memory(),
                "oc": torch.empty(oc.shape, dtype=torch.int16).pin_memory(),
                "lc": torch.empty(lc.shape, dtype=torch.float32).pin_memory()}
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = sum(t.numel() * t.element_size() for t in res_host.values())

    def read_back(o):
        res_host["out"].copy_(o["out"].view(torch.int16), non_blocking=True)
        res_host["lse"].copy_(o["lse"], non_blocking=True)
        res_host["oc"].copy_(o["oc"].view(torch.int16), non_blocking=True)
        res_host["lc"].copy_(o["lc"], non_blocking=True)

    # (a) serial: copy in, compute, copy out, one step after the other on one stream
    def e2e_serial_step():
        for n, t in pin.items():
            d[n].view(torch.int16).copy_(t, non_blocking=True)
        step()
        read_back(outs0)

    e2e_serial_step()
    torch.cuda.synchronize()
    n_serial = max(2, min(args.e2e_steps, 5))
    ms_e2e_serial = timed_region(e2e_serial_step, n_serial, stream, world, dev, barrier, with_clocks=False)[0]

    # (b) pipelined: step i's host->device copies (stream h2d) and step i-1's
    # device->host read-back (stream d2h) overlap step i-1's / i's kernels
    # (compute stream); two device buffer sets alternate, ordered by events.
    # Every step still moves all its inputs in and all its results out.
    d_alt = {n: torch.empty_like(t) for n, t in d.items()}
    outs_alt = {n: torch.empty_like(t) for n, t in outs0.items()}
    in_sets, out_sets = [d, d_alt], [outs0, outs_alt]
    s_h2d, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    comp_done = [torch.cuda.Event() for _ in range(2)]
    h2d_done = [torch.cuda.Event() for _ in range(2)]
    d2h_done = [torch.cuda.Event() for _ in range(2)]
    for bset in range(2):
        comp_done[bset].record(stream)
        d2h_done[bset].record(s_d2h)

    def e2e_pipelined_step(i):
        bset = i % 2
        with torch.cuda.stream(s_h2d):
            s_h2d.wait_event(comp_done[bset])            # step i-2 is done reading this input set
            for n, t in pin.items():
                in_sets[bset][n].view(torch.int16).copy_(t, non_blocking=True)
            h2d_done[bset].record(s_h2d)
        stream.wait_event(h2d_done[bset])
        stream.wait_event(d2h_done[bset])                # step i-2's results have been read back
        step(inp=in_sets[bset], o=out_sets[bset])
        comp_done[bset].record(stream)
        with torch.cuda.stream(s_d2h):
            s_d2h.wait_event(comp_done[bset])
            read_back(out_sets[bset])
            d2h_done[bset].record(s_d2h)

    e2e_pipelined_step(0)
    e2e_pipelined_step(1)
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_h2d)
    for i in range(args.e2e_steps):
        e2e_pipelined_step(i)
    stream.wait_event(d2h_done[(args.e2e_steps - 1) % 2])
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_e2e = max_over_ranks(e0.elapsed_time(e1), world, dev) / args.e2e_steps
    e2e_value = aggregate_tflops(flops_step, world, ms_e2e)
    del d_alt, outs_alt, rope_ws, q_raw, k_raw

    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if rank != 0:
        return None, None

    pk, pk_src = peaks()
    t_self = per_kernel["attn_self"]
    roof = tensor_roofline("attn_fwd self-attention (31200 x 31200, H=40, D=128)", f_self, t_self, ms_total, clk,
                           pk, pk_src)
    roof["traffic"] = traffic_from_profile()
    n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
    if "cycles_per_launch" in roof:
        ctas = B * H * -(-S // 256)
        roof["sm_cycles_per_key_block"] = round(roof["cycles_per_launch"] * n_sm / (ctas * -(-S // 128)), 1)
    med = statistics.median
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded splitmix64 normals; RMSNormed Q/K; no weights involved)",
        "config": step_config(world),
        "roofline": roof,
        "kernels_ms": {n: round(t, 4) for n, t in per_kernel.items()},
        "gpu_launches": LAUNCHES_PER_STEP * args.steps,
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "ms_per_step": round(ms_e2e, 3),
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
                "how": "pinned host inputs -> device -> the step's three C-ABI calls (three launches) -> outputs and "
                       "LSEs to pinned host every step; copies on their own streams overlap the neighbouring "
                       "steps' kernels (two device buffer sets); timed from the first copy to the last read-back",
                "serial_ms_per_step": round(ms_e2e_serial, 3),
                "serial_value": round(aggregate_tflops(flops_step, world, ms_e2e_serial), 2)},
        "clocks": clk,
    }
    line["rope_fused_step"] = {
        "what": "the same step with the RoPE fused into the attention's Q load (regen_attn_fwd_rope3d: table, K "
                "rotated into workspace, Q rotated on its tiles in shared memory) instead of the pre-pass; 3 rounds "
                "of n steps alternating with the pre-pass step",
        "steps_per_round": n_alt,
        "ms_per_step_rounds": [round(x, 4) for x in fused_ms],
        "prepass_ms_per_step_rounds": [round(x, 4) for x in pre_ms],
        "ms_per_step": round(med(fused_ms), 4), "prepass_ms_per_step": round(med(pre_ms), 4),
        "fused_minus_prepass_ms": round(med(fused_ms) - med(pre_ms), 4),
        "value": round(aggregate_tflops(flops_step, world, med(fused_ms)), 2), "unit": "TFLOP/s",
        "kernels_ms": {n: round(med(x), 4) for n, x in fused_k.items()},
        "launches_per_step": 4,
    }
    f_ref = 4.0 * B * H * S * N_REF * D
    line["cross_attention"] = {
        "what": "cross-attention of the 31200 video tokens to 1560 reference-frame + 512 conditioning keys: the "
                "step's one two-source launch, the Ring form (one call per key block merged by regen_lse_merge) "
                "and one call over the keys concatenated in one buffer",
        "ms": {n: round(x, 4) for n, x in cross_ms.items()},
        "kv2_tflops": round(f_cross / (cross_ms["kv2"] * 1e-3) / 1e12, 2),
        "two_calls_plus_merge_ms": round(cross_ms["ref_block"] + cross_ms["ctx_block"] + cross_ms["lse_merge"], 4),
        "ref_block_tflops": round(f_ref / (cross_ms["ref_block"] * 1e-3) / 1e12, 2),
        "ctx_block_tflops": round((f_cross - f_ref) / (cross_ms["ctx_block"] * 1e-3) / 1e12, 2),
    }
    s_merge = cross_ms["lse_merge"]
    s_rope = per_kernel["rope3d"]
    line["hbm"] = {
        "rope3d_gbs": round(4 * B * H * S * D * 2 / (s_rope * 1e-3) / 1e9, 1),
        "lse_merge_gbs": round((3 * B * H * S * D * 2 + 3 * B * H * S * 4) / (s_merge * 1e-3) / 1e9, 1),
        "peak_gbs": float(pk["hbm_gbs"]),
        "rope3d_frac": round(4 * B * H * S * D * 2 / (s_rope * 1e-3) / 1e9 / float(pk["hbm_gbs"]), 4),
        "lse_merge_frac": round((3 * B * H * S * D * 2 + 3 * B * H * S * 4) / (s_merge * 1e-3) / 1e9
                                / float(pk["hbm_gbs"]), 4),
    }
    line["backward"] = bwd
    line["fp8"] = fp8
    line["projections"] = proj
    return line, snap


def run_backward(args, rg, synth, d, outs, ws, wc, rank, dev, stream, world, barrier, to_dev):
    """Times the gradient step; returns its JSON object (rank 0 uses it)."""
    import torch
    B, H, S, D = ws.B, ws.H, ws.Sq, ws.D
    T, Hh, Ww = ws.grid
    scale = 1.0 / math.sqrt(D)
    sh = stream.cuda_stream
    g_self = to_dev(synth.make_dout(ws, seed_offset=rank))
    g_cross = to_dev(synth.make_dout(wc, seed_offset=rank))
    n_ref, n_ctx = N_REF, wc.Skv - N_REF
    dq, dk, dv = (torch.empty_like(d[n]) for n in ("q", "k", "v"))
    dqc = torch.empty_like(d["qc"])
    dkr, dvr = torch.empty_like(d["kr"]), torch.empty_like(d["vr"])
    dkx, dvx = torch.empty_like(d["kx"]), torch.empty_like(d["vx"])
    wsb = rg.regen_attn_bwd_workspace_bytes(B, H, S, D)
    work = torch.empty(wsb, dtype=torch.uint8, device=dev)
    names = ["attn_bwd_self", "rope3d_bwd", "attn_bwd_cross_kv2"]

    def cross_kv2():
        rg.regen_attn_bwd_kv2(d["qc"], d["kr"], d["vr"], d["kx"], d["vx"], outs["oc"], outs["lc"], g_cross, dqc,
                              dkr, dvr, dkx, dvx, B, H, S, n_ref, n_ctx, D, scale, sh, work, wsb, 0)

    def cross_per_source():
        rg.regen_attn_bwd(d["qc"], d["kr"], d["vr"], outs["oc"], outs["lc"], g_cross, dqc, dkr, dvr, B, H, S,
                          n_ref, D, scale, sh, work, wsb, 0)
        rg.regen_attn_bwd(d["qc"], d["kx"], d["vx"], outs["oc"], outs["lc"], g_cross, dqc, dkx, dvx, B, H, S,
                          n_ctx, D, scale, sh, work, wsb, 1)

    def step(ev=None):
        def mark(i):
            if ev is not None:
                ev[i].record(stream)
        mark(0)
        rg.regen_attn_bwd(d["q"], d["k"], d["v"], outs["out"], outs["lse"], g_self, dq, dk, dv, B, H, S, S, D,
                          scale, sh, work, wsb, 0)
        mark(1)
        rg.regen_rope3d_bwd(dq, dk, T, Hh, Ww, ws.theta, B, H, D, sh)
        mark(2)
        cross_kv2()
        mark(3)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    n = max(3, min(args.steps, 10))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n)]
    ms, clk, region = timed_region(lambda it=iter(evs): step(next(it)), n, stream, world, dev, barrier)
    per = {nm: sum(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(n)) / n for j, nm in enumerate(names)}
    # the cross-attention gradient in one two-source call against one call per
    # key source (the second accumulating dq): alternating rounds, outside the step
    cmp = {"kv2": [], "per_source": []}
    for rnd in range(4):
        order = (("kv2", cross_kv2), ("per_source", cross_per_source))
        for nm, fn in (order if rnd % 2 == 0 else order[::-1]):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(3):
                fn()
            e1.record(stream)
            e1.synchronize()
            cmp[nm].append(e0.elapsed_time(e1) / 3)
    f_self, f_cross = step_flops()
    flops = 2.5 * (f_self + f_cross)      # S, dP, dV, dK, dQ: five products of the forward's two sizes
    pk, pk_src = peaks()
    roof = tensor_roofline("regen_attn_bwd self-attention (prep + dK/dV + dQ launches)", 2.5 * f_self,
                           per["attn_bwd_self"], region, clk, pk, pk_src)
    roof["issued_tensor_flops_frac"] = round(roof["frac"] * 7 / 5, 4)
    del work
    return {
        "what": "gradient step of the same window: regen_attn_bwd (self) + regen_rope3d_bwd + regen_attn_bwd_kv2 "
                "(the cross-attention's two key sources with the joint out/LSE, one dQ pass over both); synthetic dO",
        "steps": n, "ms_per_step": round(ms, 4),
        "value": round(aggregate_tflops(flops, world, ms), 2), "unit": "TFLOP/s",
        "flops_note": "algorithmic: 2.5x the forward's (QK^T, dO V^T, P^T dO, dS^T Q, dS K); the kernels also "
                      "recompute QK^T and dO V^T once more (7 products in all, no atomics)",
        "kernels_ms": {nm: round(t, 4) for nm, t in per.items()},
        "launches_per_step": 3 + 1 + 3,
        "cross_attention_ms": {"kv2": round(min(cmp["kv2"]), 4), "per_source_calls": round(min(cmp["per_source"]), 4),
                               "what": "best of 4 alternating rounds of 3 calls: regen_attn_bwd_kv2 against one "
                                       "regen_attn_bwd per key source (6 launches, dq accumulated)"},
        "roofline": roof,
        "clocks": clk,
    }


C_MODEL = 5120   # model width of the 14B-class DiT (40 heads x 128)


def run_proj(args, rg, synth, ws, dev, stream, world, barrier, to_dev, rank):
    """Times regen_qkv_proj and regen_out_proj on the 77-frame window of a 14B-class
    DiT block (C = 5120, 40 heads); a cuBLAS GEMM of the same shapes is timed beside
    them for comparison only. Returns the JSON object."""
    import torch
    B, H, S, D = ws.B, ws.H, ws.Sq, ws.D
    T, Hh, Ww = ws.grid
    C = C_MODEL
    sh = stream.cuda_stream
    seed = 100 + rank
    x = to_dev(synth._normal_bf16(seed, 0, (B, S, C), False))
    w = to_dev(synth.f64_to_bf16_bits(synth.normal(seed, 1, 3 * H * D * C).reshape(3 * H * D, C) / math.sqrt(C)))
    wo = to_dev(synth.f64_to_bf16_bits(synth.normal(seed, 2, C * H * D).reshape(C, H * D) / math.sqrt(H * D)))
    bias = torch.from_numpy((synth.normal(seed, 3, 3 * H * D) * 0.1).astype(np.float32)).to(dev)
    bo = torch.from_numpy((synth.normal(seed, 4, C) * 0.1).astype(np.float32)).to(dev)
    q, k, v = (torch.empty((B, H, S, D), dtype=torch.bfloat16, device=dev) for _ in range(3))
    y = torch.empty((B, S, C), dtype=torch.bfloat16, device=dev)
    o = to_dev(synth._normal_bf16(seed, 5, (B, H, S, D), False))
    wsb = rg.regen_qkv_proj_workspace_bytes(T, Hh, Ww, D)
    work = torch.empty(wsb, dtype=torch.uint8, device=dev)

    def qkv():
        rg.regen_qkv_proj(x, w, bias, None, None, q, k, v, B, S, C, H, D, T, Hh, Ww, ws.theta, 1e-6, sh, work, wsb)

    def outp():
        rg.regen_out_proj(o, wo, bo, y, B, S, H, D, C, sh)

    xm = x.view(B * S, C)
    om = o.permute(0, 2, 1, 3).reshape(B * S, H * D).contiguous()
    res = torch.empty((B * S, 3 * H * D), dtype=torch.bfloat16, device=dev)
    reso = torch.empty((B * S, C), dtype=torch.bfloat16, device=dev)

    def cublas_qkv():
        torch.matmul(xm, w.t(), out=res)

    def cublas_out():
        torch.matmul(om, wo.t(), out=reso)

    def timed(fn, n, clocks=False):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        return timed_region(fn, n, stream, world, dev, barrier, with_clocks=clocks)

    n = max(5, min(args.steps, 40))
    t_qkv, clk_qkv, region_qkv = timed(qkv, n, clocks=True)
    t_out = timed(outp, n)[0]
    t_cq, t_co = timed(cublas_qkv, n)[0], timed(cublas_out, n)[0]
    f_qkv = 2.0 * B * S * C * 3 * H * D
    f_out = 2.0 * B * S * H * D * C
    pk, pk_src = peaks()
    tf = lambda f, ms: f / (ms * 1e-3) / 1e12  # noqa: E731
    del work, x, w, wo, o, q, k, v, y, res, reso, om
    return {
        "what": "DiT block projections on the 77-frame window, 14B-class (C = 5120, 40 heads x 128): regen_qkv_proj "
                "(x W^T + b, per-head RMSNorm + 3D RoPE on q and k, q/k/v written as [B,H,S,128]) and regen_out_proj "
                "(attention output read in place as token rows); a plain cuBLAS GEMM of each shape (torch.matmul, "
                "no epilogue) timed beside them for comparison only",
        "steps": n,
        "qkv_proj": {"ms": round(t_qkv, 4), "tflops": round(tf(f_qkv, t_qkv), 2), "M": B * S, "N": 3 * H * D, "K": C,
                     "cublas_gemm_ms": round(t_cq, 4), "cublas_tflops": round(tf(f_qkv, t_cq), 2)},
        "out_proj": {"ms": round(t_out, 4), "tflops": round(tf(f_out, t_out), 2), "M": B * S, "N": C, "K": H * D,
                     "cublas_gemm_ms": round(t_co, 4), "cublas_tflops": round(tf(f_out, t_co), 2)},
        "roofline": tensor_roofline("proj_gemm_kernel<QKV> (31200 x 15360 x 5120)", f_qkv, t_qkv, region_qkv, clk_qkv,
                                    pk, pk_src),
        "launches_per_step": 3,
    }


def run_fp8(args, rg, d, ws, dev, stream, world, barrier):
    """Times quantise + FP8 self-attention on the 77-frame window; returns its JSON object."""
    import torch
    B, H, S, D = ws.B, ws.H, ws.Sq, ws.D
    scale = 1.0 / math.sqrt(D)
    sh = stream.cuda_stream
    nb = -(-S // 128)
    codes = {n: torch.empty((B, H, S, D), dtype=torch.uint8, device=dev) for n in ("q", "k", "v")}
    scales = {n: torch.empty((B, H, nb), dtype=torch.float32, device=dev) for n in ("q", "k", "v")}
    out = torch.empty((B, H, S, D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H, S), dtype=torch.float32, device=dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        for n in ("q", "k", "v"):
            rg.regen_quant_e4m3(d[n], codes[n], scales[n], B, H, S, D, sh)
        if ev is not None:
            ev[1].record(stream)
        rg.regen_attn_fwd_fp8(codes["q"], scales["q"], codes["k"], scales["k"], codes["v"], scales["v"], out, lse,
                              B, H, S, S, D, scale, sh)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    n = max(3, min(args.steps, 20))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n)]
    ms, clk, region = timed_region(lambda it=iter(evs): step(next(it)), n, stream, world, dev, barrier)
    t_q = sum(e[0].elapsed_time(e[1]) for e in evs) / n
    t_a = sum(e[1].elapsed_time(e[2]) for e in evs) / n
    f_self = step_flops()[0]
    pk, pk_src = peaks()
    qbytes = 3 * B * H * S * D * 3 + 3 * B * H * nb * 4    # read bf16, write codes, write scales
    return {
        "what": "FP8 (E4M3) variant of the 77-frame self-attention after its RoPE: blockwise quantisation of Q, K, V "
                "(regen_quant_e4m3 x3) + regen_attn_fwd_fp8; accuracy contract in the tests (E4M3 rounding of P)",
        "steps": n, "ms_per_step": round(ms, 4),
        "value": round(aggregate_tflops(f_self, world, ms), 2), "unit": "TFLOP/s",
        "kernels_ms": {"quant_e4m3_x3": round(t_q, 4), "attn_fwd_fp8": round(t_a, 4)},
        "quant_gbs": round(qbytes / (t_q * 1e-3) / 1e9, 1),
        "roofline": tensor_roofline("attn_fwd_fp8 (31200 x 31200, H=40, D=128)", f_self, t_a, region, clk, pk, pk_src,
                                    peak_mult=2.0, peak_note="dense E4M3 : BF16 nominal ratio"),
        "clocks": clk,
        "launches_per_step": 4,
    }


# ------------------------------------------------------ CPU (oracle) ---

def cpu_sample_rate(target_s: float, seed_rows: int = 0, snap=None):
    """Time the fp64 oracle on a bounded sample of query rows of the 77-frame
    self-attention. With `snap` (the last timed GPU step's bf16 inputs and
    output) the oracle runs on exactly those inputs, so that its rows also
    check the GPU's; without it (the reference arm) on the workload's
    generated inputs, whose values do not change the oracle's cost."""
    import oracle
    from dit_attention_b200 import synth
    w = synth.WORKLOADS[SELF]
    if snap is not None:   # the step's unrotated inputs: the oracle applies the RoPE itself (not timed)
        qr = oracle.rope3d(snap["q"], snap["grid"], snap["theta"])
        kr = oracle.rope3d(snap["k"], snap["grid"], snap["theta"])
        v = snap["v"]
    else:
        qr, kr, v = synth.make_inputs(w)
    rng = np.random.default_rng(seed_rows)
    BH = w.B * w.H
    # calibrate t(rows) = a + b*rows on two sizes, then size the sample to about target_s
    def timed(n):
        rows = rng.choice(BH * w.Sq, size=n, replace=False)
        t = time.perf_counter()
        oracle.attention(qr, kr, v, w.scale, rows=rows)
        return time.perf_counter() - t
    n1, n2 = 32, 256
    t1, t2 = timed(n1), timed(n2)
    per_row = max((t2 - t1) / (n2 - n1), 1e-6)
    fixed = max(t1 - per_row * n1, 0.0)
    n_full = int(min(BH * w.Sq, max(64, (target_s - fixed) / per_row)))
    return dict(q=qr, k=kr, v=v, w=w, rng=rng, rows=n_full, threads=oracle.num_threads())


def time_cpu(sample, rows, keep=None):
    """TFLOP/s and seconds of the oracle on `rows` random query rows; with a
    dict `keep`, also stores the row indices and the oracle's out and lse rows."""
    import oracle
    w = sample["w"]
    r = sample["rng"].choice(w.B * w.H * w.Sq, size=rows, replace=False)
    t = time.perf_counter()
    ref, ref_lse = oracle.attention(sample["q"], sample["k"], sample["v"], w.scale, rows=r)
    dt = time.perf_counter() - t
    if keep is not None:
        keep.update(rows=r, out=ref, lse=ref_lse)
    flops = 4.0 * rows * w.Skv * w.D
    return flops / dt / 1e12, dt


def accuracy(snap, kept):
    """The GPU's rows against the oracle's on the same bf16 inputs: the
    attention contract |out - ref| <= 1e-2 + 1e-2|ref|, |lse - ref| <= 1e-3, and
    the error normalised by RMS(ref). The diagnostic flag is on the MEAN error
    over RMS(ref), above 5e-3: the roundings of P and of the output keep it
    near u/4 (u = 2^-8), while a real defect (a wrong scale, a dropped block)
    moves every element. The maximum is reported beside it: over a million
    elements the rounding of P alone reaches ~2 % of RMS on a few of them."""
    import oracle
    D = snap["out"].shape[-1]
    got = oracle.bf16_to_f64(snap["out"].reshape(-1, D)[kept["rows"]])
    ref = kept["out"].reshape(got.shape)
    err = np.abs(got - ref)
    rms = float(np.sqrt(np.mean(ref ** 2))) or 1.0
    lse_err = np.abs(snap["lse"].reshape(-1)[kept["rows"]].astype(np.float64) - kept["lse"].reshape(-1))
    within = bool(np.all(err <= 1e-2 + 1e-2 * np.abs(ref)) and np.all(lse_err <= 1e-3))
    return {"rows": int(len(kept["rows"])),
            "inputs": "one more step after the timed ones, on the unrotated bf16 q, k, v; the oracle applies the "
                      "3D RoPE to q and k itself",
            "max_abs_err": float(err.max()), "max_err_over_rms": float(err.max() / rms),
            "mean_rel_err": float(np.mean(err) / (np.mean(np.abs(ref)) or 1.0)),
            "max_lse_err": float(lse_err.max()), "contract": "|out-ref| <= 1e-2 + 1e-2|ref|, |lse-ref| <= 1e-3",
            "mean_err_over_rms": float(np.mean(err) / rms), "within_contract": within,
            "flag_mean_err_over_rms_5e-3": bool(np.mean(err) / rms > 5e-3)}


def run_configs(args):
    """CUDA-event medians (20 launches after 5 warm-ups, L2 flushed between
    launches) of the kernels of every workload, through the C ABI:
    tiny (D = 64, no RoPE), the 25- and 77-frame windows (RoPE, then the
    self-attention; for the 77-frame one also four back-to-back calls, one per
    denoising step), the cross-attention over the 2072 concatenated reference
    + conditioning keys in one call, and the stress workload whole, as two
    5460-key halves, and their merge. Prints one JSON object."""
    import torch
    import dit_attention_b200 as rg
    from dit_attention_b200 import synth

    torch.cuda.set_device(0)
    rg.load()
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # > L2 (126 MB)
    REPS, WARM = 20, 5

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)

    def median_ms(fn, reps=REPS, warm=WARM):
        for _ in range(warm):
            fn()
        ts = []
        for _ in range(reps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    def tflops(w, skv, ms):
        return 4.0 * w.B * w.H * w.Sq * skv * w.D / (ms * 1e-3) / 1e12

    rows = []
    for name, w in synth.WORKLOADS.items():
        q, k, v = (to_dev(x) for x in synth.make_inputs(w))
        B, H, Sq, Skv, D = w.B, w.H, w.Sq, w.Skv, w.D
        scale = w.scale
        out = torch.empty((B, H, Sq, D), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((B, H, Sq), dtype=torch.float32, device=dev)
        rec = {"workload": name, "B": B, "H": H, "Sq": Sq, "Skv": Skv, "D": D}
        if w.rope:
            T, Hh, Ww = w.grid
            qr, kr = q.clone(), k.clone()
            ms = median_ms(lambda: rg.regen_rope3d(qr, kr, T, Hh, Ww, w.theta, B, H, D, sh))
            rec["rope3d_ms"] = round(ms, 4)
            rec["rope3d_gbs"] = round(2 * 2 * B * H * Sq * D * 2 / (ms * 1e-3) / 1e9, 1)
            rg.regen_rope3d(q, k, T, Hh, Ww, w.theta, B, H, D, sh)   # attention on the rotated inputs
        ms = median_ms(lambda: rg.regen_attn_fwd(q, k, v, out, lse, B, H, Sq, Skv, D, scale, sh))
        rec["attn_ms"] = round(ms, 4)
        rec["attn_tflops"] = round(tflops(w, Skv, ms), 1)
        if name == SELF:
            def four():
                for _ in range(4):
                    rg.regen_attn_fwd(q, k, v, out, lse, B, H, Sq, Skv, D, scale, sh)
            rec["attn_four_calls_ms"] = round(median_ms(four, reps=5, warm=1), 3)
        if w.merge_split:
            h = w.merge_split
            ka, va = k[:, :, :h].contiguous(), v[:, :, :h].contiguous()
            kb, vb = k[:, :, h:].contiguous(), v[:, :, h:].contiguous()
            oa, ob, om = (torch.empty_like(out) for _ in range(3))
            la, lb, lm = (torch.empty_like(lse) for _ in range(3))
            ma = median_ms(lambda: rg.regen_attn_fwd(q, ka, va, oa, la, B, H, Sq, h, D, scale, sh))
            mb = median_ms(lambda: rg.regen_attn_fwd(q, kb, vb, ob, lb, B, H, Sq, Skv - h, D, scale, sh))
            mm = median_ms(lambda: rg.regen_lse_merge(oa, la, ob, lb, om, lm, B * H * Sq, D, sh))
            rec.update(half_a_ms=round(ma, 4), half_b_ms=round(mb, 4), merge_ms=round(mm, 4),
                       merge_gbs=round(B * H * Sq * (3 * D * 2 + 3 * 4) / (mm * 1e-3) / 1e9, 1),
                       split_path_ms=round(ma + mb + mm, 4))
        rows.append(rec)
        del q, k, v, out, lse
        torch.cuda.empty_cache()
    return {"what": "CUDA-event medians per workload (20 launches after 5 warm-ups, 256 MB L2 flush "
                    "between launches); TFLOP/s = 4 B H Sq Skv D / time", "configs": rows}


PROFILE_GRIDS = {31200: (20, 30, 52), 10920: (7, 30, 52), 1024: (1, 32, 32)}


def run_profile_case(args):
    """One kernel of the hot path on a synthetic shape, --iters calls, for a
    profiler (ncu): attn (self-attention over --seq keys, or --kv for
    cross-attention), fused (the RoPE-fused self-attention: table, K pass and
    attention launches), kv2 (two-source cross-attention: 1560 reference keys
    plus the rest of --kv), rope (3D RoPE on the latent grid of --seq), merge
    (two-block LSE merge), bwd (one forward, then gradient calls: prep, dK/dV
    and dQ launches each), fp8 (Q, K, V quantised once, then FP8 attention
    calls), proj (regen_qkv_proj at the model width C = 5120 with --heads
    heads, on the latent grid of --seq) or proj_ref (a cuBLAS GEMM of the same
    shape, the comparison point the bench times beside it). No timing is done
    here."""
    import torch
    import dit_attention_b200 as rg
    from dit_attention_b200 import synth
    if args.kernel_case in ("proj", "proj_ref"):
        T, Hh, Ww = PROFILE_GRIDS[args.seq]
        H, C, S = args.heads, C_MODEL, args.seq
        x = torch.from_numpy(synth._normal_bf16(100, 0, (1, S, C), False).view(np.int16)).cuda().view(torch.bfloat16)
        w = torch.from_numpy(synth.f64_to_bf16_bits(synth.normal(100, 1, 3 * H * 128 * C).reshape(3 * H * 128, C)
                                                    / math.sqrt(C)).view(np.int16)).cuda().view(torch.bfloat16)
        rg.load()
        if args.kernel_case == "proj":
            bias = torch.from_numpy((synth.normal(100, 3, 3 * H * 128) * 0.1).astype(np.float32)).cuda()
            for _ in range(args.iters):
                rg.qkv_proj(x, w, H, (T, Hh, Ww), bias=bias)
        else:
            xm, res = x.view(S, C), torch.empty((S, 3 * H * 128), dtype=torch.bfloat16, device="cuda")
            for _ in range(args.iters):
                torch.matmul(xm, w.t(), out=res)
        torch.cuda.synchronize()
        rc, site = rg.regen_last_device_error()
        if rc != 0:
            raise SystemExit(f"device error {rc} at wait site {site}")
        return
    skv = args.kv or args.seq
    w = synth.Workload("profile", B=1, H=args.heads, D=args.dim, Sq=args.seq, Skv=skv, seed=7)
    q, k, v = synth.make_inputs(w)

    def dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)

    dq, dk, dv = dev(q), dev(k), dev(v)
    rg.load()
    scale = 1.0 / math.sqrt(args.dim)
    if args.kernel_case == "bwd":
        out, lse = rg.attn_fwd(dq, dk, dv, scale)
        g = dev(synth.make_dout(w))
    if args.kernel_case == "fp8":
        quant = [rg.quant_e4m3(x) for x in (dq, dk, dv)]
    if args.kernel_case == "kv2":
        n_ref = min(N_REF, skv - 1)
        ka, va = dk[:, :, :n_ref].contiguous(), dv[:, :, :n_ref].contiguous()
        kb, vb = dk[:, :, n_ref:].contiguous(), dv[:, :, n_ref:].contiguous()
    for _ in range(args.iters):
        if args.kernel_case == "fp8":
            rg.attn_fwd_fp8(*quant[0], *quant[1], *quant[2], scale)
        elif args.kernel_case == "attn":
            rg.attn_fwd(dq, dk, dv, scale)
        elif args.kernel_case == "fused":
            rg.attn_fwd_rope3d(dq, dk, dv, PROFILE_GRIDS[args.seq], scale=scale)
        elif args.kernel_case == "kv2":
            rg.attn_fwd_kv2(dq, ka, va, kb, vb, scale)
        elif args.kernel_case == "bwd":
            rg.attn_bwd(dq, dk, dv, out, lse, g, scale)
        elif args.kernel_case == "rope":
            rg.rope3d_(dq, dk, PROFILE_GRIDS[args.seq])
        else:
            lse = torch.zeros((1, args.heads, args.seq), dtype=torch.float32, device="cuda")
            rg.lse_merge(dq, lse, dk[:, :, :args.seq], lse)
    torch.cuda.synchronize()
    rc, site = rg.regen_last_device_error()
    if rc != 0:
        raise SystemExit(f"device error {rc} at wait site {site}")


def run_reference(args, rank, world):
    if rank != 0:
        return None
    sample = cpu_sample_rate(min(3.0, args.cpu_seconds))
    for _ in range(args.warmup):
        time_cpu(sample, max(16, sample["rows"] // 8))
    vals, secs = [], 0.0
    for _ in range(args.steps):
        v, dt = time_cpu(sample, sample["rows"])
        vals.append(v)
        secs += dt
    value = statistics.mean(vals)
    desc = (f"{sample['rows']} random query rows per step of the 77-frame self-attention, the step's "
            f"dominant part (all 31200 keys, D=128), fp64; TFLOP/s over those rows")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1000 * secs / args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": step_config(world),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": sample["threads"], "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def main():
    args = parse()
    rank, world, local_rank = dist_env()
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if args.configs:
        if rank == 0:
            print(json.dumps(run_configs(args)), flush=True)
        return
    if args.profile_case:
        args.kernel_case = args.profile_case
        if rank == 0:
            run_profile_case(args)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    line, snap = run_native(args, rank, world, local_rank)
    if line is not None and not args.no_cpu_baseline:
        import oracle
        sample = cpu_sample_rate(args.cpu_seconds, snap=snap)
        kept = {}
        v, dt = time_cpu(sample, sample["rows"], keep=kept)
        line["accuracy"] = accuracy(snap, kept)
        # the same oracle once more on one thread, on a smaller sample (~1/3 of the time above)
        threads = sample["threads"]
        rows1 = max(16, sample["rows"] // max(1, 3 * threads))
        oracle.set_num_threads(1)
        try:
            v1, dt1 = time_cpu(sample, rows1)
        finally:
            oracle.set_num_threads(threads)
        line["cpu_baseline"] = {
            "value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"{sample['rows']} random query rows of the 77-frame self-attention (all 31200 keys, "
                      f"D=128), fp64, {dt:.1f} s",
            "single_thread": {"value": v1, "unit": "TFLOP/s", "cores": 1,
                              "sample": f"{rows1} random query rows, same workload, {dt1:.1f} s"},
        }
    if line is not None:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
