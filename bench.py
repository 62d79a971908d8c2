"""Benchmark of the weight-only quantized matmul on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

Default workload (the metric's headline case): the four LLaMA-7B linear-layer
shapes of one decoder layer -- fused QKV (K 4096, N 12288), O (4096, 4096),
fused gate/up (4096, 22016), down (11008, 4096) -- at M = 1, 2, 4, 8 and 16
tokens: 20 qmm calls per step, symmetric int4, group 128, fp16 activations.
Each call has its own weights (522 MB in all, over 4x the 126 MB L2), so every
call streams its codes from HBM; smaller workloads get as many weight copies
as it takes to pass twice the L2 size, rotated step by step.  The launches of
a step are captured in a CUDA graph (one per weight copy) and a step is one
replay.

Prints one JSON line (rank 0).  `value` is HBM throughput in GB/s: algorithmic
bytes (codes + scales + x + y) of all calls on all ranks / max-over-ranks
device time.  With --gpus N (under torchrun) every rank runs the same
workload on its own GPU: independent replicas, weak scaling.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A16 qmm: HBM GB/s (M<=16), TFLOP/s (M>=256), % of roofline"

WORKLOADS = {
    # name: (mode, bits, group, xdtype, [(K, N)], [M])
    "llama7b_decode": ("sym", 4, 128, "f16",
                       [(4096, 12288), (4096, 4096), (4096, 22016), (11008, 4096)],
                       [1, 2, 4, 8, 16]),
    "decode_4096sq": ("sym", 4, 128, "f16", [(4096, 4096)], [1]),
    "gateup_m1": ("sym", 4, 128, "f16", [(4096, 22016)], [1]),
    "gateup_m16": ("sym", 4, 128, "f16", [(4096, 22016)], [16]),
    "prefill_m64": ("sym", 4, 128, "f16", [(4096, 11008)], [64]),
    "prefill_m256": ("sym", 4, 128, "f16", [(4096, 11008)], [256]),
    "prefill_m1024": ("sym", 4, 128, "f16", [(4096, 11008)], [1024]),
    "prefill_m4096": ("sym", 4, 128, "f16", [(4096, 11008)], [4096]),
    "prefill_m64_rowscale": ("sym", 4, -1, "f16", [(4096, 11008)], [64]),
    "prefill_m256_rowscale": ("sym", 4, -1, "f16", [(4096, 11008)], [256]),
    "prefill_m1024_rowscale": ("sym", 4, -1, "f16", [(4096, 11008)], [1024]),
    "prefill_m4096_rowscale": ("sym", 4, -1, "f16", [(4096, 11008)], [4096]),
    "llama70b_asym_bf16": ("asym", 4, 128, "bf16",
                           [(8192, 10240), (8192, 57344), (28672, 8192)], [1, 16, 64]),
    "lut4_nf4": ("lut", 4, 64, "f16", [(4096, 14336)], [1, 8, 32]),
    "lut2": ("lut", 2, 64, "f16", [(4096, 14336)], [1, 8, 32]),
    "lut3_nf3": ("lut", 3, 64, "f16", [(4096, 14336)], [1, 8]),
    # LLaMA-7B feed-forward gate fused into the matmul: gate and up (I = 11008
    # each, N = 2 I rows packed together), y[M, I] = silu(gate) * up
    "ffn_gated": ("sym", 4, 128, "f16", [(4096, 22016)], [1, 2, 4, 8, 16]),
    # zero-point options (Marlin zero-point issue): scale per row with a 4-bit
    # zero-point per 8 columns (mobicham's HQQ+ layout); and the 70B asymmetric
    # layers with their zero-points stored in 4 bits
    "asym_rowscale_zg8_u4": ("asym", 4, -1, "f16", [(4096, 14336)], [1, 8]),
    "llama70b_asym_zq4_bf16": ("asym", 4, 128, "bf16",
                               [(8192, 10240), (8192, 57344), (28672, 8192)], [1, 16]),
    # act-order groups (GPTQ-Triton summary, Limitations): the LLaMA-7B decode
    # layers with a random column order per matrix; x gathered per call
    "actorder_llama7b": ("sym", 4, 128, "f16",
                         [(4096, 12288), (4096, 4096), (4096, 22016), (11008, 4096)],
                         [1, 2, 4, 8, 16]),
}
GATED = {"ffn_gated"}
# The five benchmark configurations and the workloads that time them (the
# default run reports every one of them beside its headline, config 2).
CONFIG_WORKLOADS = {
    "1_4096sq_m1": ["decode_4096sq"],
    "3_llama70b_asym_bf16": ["llama70b_asym_bf16"],
    "4_lut_k4096_n14336": ["lut4_nf4", "lut2"],
    "5_prefill_k4096_n11008": ["prefill_m64", "prefill_m256", "prefill_m1024", "prefill_m4096",
                               "prefill_m64_rowscale", "prefill_m256_rowscale",
                               "prefill_m1024_rowscale", "prefill_m4096_rowscale"],
}
# workload -> zero-point options (zero group, zero bits)
ZOPTS = {"asym_rowscale_zg8_u4": (8, 4), "llama70b_asym_zq4_bf16": (128, 4)}
ACTORDER = {"actorder_llama7b"}
SIGMA = {"sym": 0.02, "asym": 0.015, "lut": 0.02}
L2_BYTES = 126 * 1000 * 1000     # B200 L2
SKINNY_SOURCES = ("weight_only_quantized_int4_b200/csrc/skinny.cu",
                  "weight_only_quantized_int4_b200/csrc/common.cuh")


def alg_bytes(mode, bits, group, M, K, N, gated=False, zopts=None, actorder=False):
    """Bytes a call must move at least once: codes, scales (+ zeros), x, y
    (y has N / 2 columns for the fused gate); with zero-point options the zero
    records of their own group and width; with act-order the int32 column
    permutation."""
    G = 1 if group == -1 else K // group
    if zopts is not None:
        zg, zbits = zopts
        GZ = K // (K if zg == -1 else zg)
        meta = N * G * 2 + N * GZ * zbits // 8
    else:
        meta = N * G * 2 * (2 if mode == "asym" else 1)
    perm = 4 * K if actorder else 0
    return N * K * bits // 8 + meta + perm + M * K * 2 + M * (N // 2 if gated else N) * 2


def problems(name):
    mode, bits, group, xdt, shapes, Ms = WORKLOADS[name]
    return [(mode, bits, group, xdt, M, K, N) for M in Ms for (K, N) in shapes]


def peaks():
    """(HBM GB/s, source) of the roofline's memory bound."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def tensor_peak():
    """(TFLOP/s, source) of the dense fp16/bf16 tensor bound.  The bench loops
    for seconds under the power cap, so the sustained figure applies."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["bf16_tflops_sustained"]), "measured, sustained"
    except Exception:
        return 1400.0, "fallback, sustained"


def tensor_bound(name):
    """Workloads whose every call has M >= 256: reported in TFLOP/s against the
    tensor roofline (the rest in GB/s against HBM)."""
    return min(WORKLOADS[name][5]) >= 256


def alg_flops(M, K, N):
    return 2.0 * M * N * K


def sources_hash():
    h = hashlib.sha256()
    for s in SKINNY_SOURCES:
        with open(os.path.join(ROOT, s), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_per_byte():
    """DRAM bytes per algorithmic byte from the committed ncu summary, if it was
    taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "skinny_llama7b_decode_traffic.txt")
    try:
        kv = {}
        with open(path) as f:
            for line in f:
                if ":" in line and not line.startswith("#"):
                    k, v = line.split(":", 1)
                    kv[k.strip()] = v.strip()
        if kv.get("source_hash") != sources_hash():
            return None
        return float(kv["dram_bytes_per_algorithmic_byte"])
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi samples (every 100 ms) of SM clock and throttle reasons."""

    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- ours

def max_over_ranks(value, dist=None, device="cpu"):
    """The largest `value` over all ranks; every rank gets it (one all-reduce)."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world, bytes_per_step, steps, ms):
    """Algorithmic GB/s of all ranks together: every rank streams `bytes_per_step`
    per step (replicas, weak scaling) and the job takes `ms` (the slowest rank)."""
    return world * bytes_per_step * steps / (ms / 1e3) / 1e9


def arena_of(tensors, align=256):
    """One uint8 buffer holding copies of `tensors` at `align`-byte offsets, and
    views of it with each tensor's dtype and shape: (buffer, [views])."""
    import torch
    offs, total = [], 0
    for t in tensors:
        offs.append(total)
        total += -(-t.numel() * t.element_size() // align) * align
    device = tensors[0].device if tensors else "cpu"
    arena = torch.empty(total, dtype=torch.uint8, device=device)
    views = []
    for t, o in zip(tensors, offs):
        v = arena[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
        v.copy_(t)
        views.append(v)
    return arena, views


class Workload:
    """Every call of one step of a workload on the device: packed weights in
    as many copies as it takes to pass twice the L2 size (rotated step by
    step), activations and outputs (each set in one buffer, so the end-to-end
    leg moves a step's inputs and results with one copy each way), workspaces,
    and one CUDA graph of a round of steps, one per weight copy (a graph launch
    costs microseconds: a round keeps it off single-call steps).  The default
    workload has one copy, so a round is one step.

    Inputs come from the seed-0 counter generator of `synth` (drawn on the
    device): call c's weights are stream "W{c}.{copy}", its activations "x{c}".
    """

    def __init__(self, name, dev):
        import torch
        import weight_only_quantized_int4_b200 as q
        from weight_only_quantized_int4_b200 import synth

        self.name, self.dev = name, dev
        probs = problems(name)
        self.gated = name in GATED
        self.zopts = ZOPTS.get(name)
        self.actorder = name in ACTORDER
        self.codes_per_copy = sum(N * K * bits // 8 for (_, bits, _, _, _, K, N) in probs)
        self.copies = max(1, -(-2 * L2_BYTES // self.codes_per_copy))
        gen = torch.Generator(device=dev).manual_seed(0)
        self.sets, self.xarenas, self.yarenas = [], [], []
        for cp in range(self.copies):
            calls = []
            for ci, (mode, bits, group, xdt, M, K, N) in enumerate(probs):
                W = synth.weights_torch(0, f"W{ci}.{cp}", N, K, SIGMA[mode], device=dev)
                lut = None
                if mode == "lut":
                    t = {4: synth.nf4_table, 3: synth.nf3_table, 2: lambda: synth.lut2_table(0)}[bits]()
                    lut = torch.from_numpy(t.view(np.int16)).to(dev)
                perm = None
                if self.gated:
                    qw, sc, ze = q.pack_gated(W[: N // 2], W[N // 2:], mode, bits, group, lut=lut)
                elif self.zopts is not None:
                    qw, sc, ze = q.pack_asym(W, group, self.zopts[0], self.zopts[1])
                elif self.actorder:
                    perm = torch.randperm(K, generator=gen, device=dev).to(torch.int32)
                    qw, sc, ze = q.pack_actorder(W, perm, mode, bits, group, lut=lut)
                else:
                    qw, sc, ze = q.pack(W, mode, bits, group, lut=lut)
                del W
                x = synth.activations_torch(0, f"x{ci}", M, K, xdt, device=dev)
                tdt = x.dtype
                y = torch.empty(M, N // 2 if self.gated else N, dtype=tdt, device=dev)
                if self.zopts is not None:
                    ws = q.workspace_asym(M, N, K, group, self.zopts[0], self.zopts[1], device=dev)
                elif self.actorder:
                    ws = q.workspace_actorder(M, N, K, mode, bits, group, device=dev)
                else:
                    ws = q.workspace(M, N, K, mode, bits, group, device=dev)
                zl = ze if mode == "asym" else lut
                calls.append(dict(x=x, qw=qw, sc=sc, zl=zl, y=y, ws=ws, M=M, N=N, K=K, mode=mode,
                                  bits=bits, group=group, perm=perm,
                                  bytes=alg_bytes(mode, bits, group, M, K, N, self.gated,
                                                  self.zopts, self.actorder)))
            for key, arenas in (("x", self.xarenas), ("y", self.yarenas)):
                arena, views = arena_of([c[key] for c in calls])
                for c, v in zip(calls, views):
                    c[key] = v
                arenas.append(arena)
            self.sets.append(calls)
        torch.cuda.synchronize()
        calls = self.sets[0]
        self.n_calls = len(calls)
        self.step_bytes = sum(c["bytes"] for c in calls)
        self.step_flops = sum(alg_flops(c["M"], c["K"], c["N"]) for c in calls)
        self.dtype = WORKLOADS[name][3]
        # warm-up outside the graphs (first calls set kernel attributes), then
        # one graph per weight copy
        for i in range(self.copies):
            self.step(i)
        torch.cuda.synchronize()
        self.stream = torch.cuda.Stream(device=dev)
        with torch.cuda.stream(self.stream):
            self.step()
            torch.cuda.synchronize()
            self.graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.graph, stream=self.stream):
                for i in range(self.copies):
                    self.step(i)
        torch.cuda.synchronize()

    def step(self, i=0):
        """The step's calls through the Python API (weight copy i % copies)."""
        import weight_only_quantized_int4_b200 as q
        z = self.zopts
        for c in self.sets[i % self.copies]:
            if self.gated:
                q.qmm_gated(c["x"], c["qw"], c["sc"], c["zl"], c["N"] // 2, c["K"], c["mode"],
                            c["bits"], c["group"], y=c["y"], ws=c["ws"])
            elif z is not None:
                q.qmm_asym(c["x"], c["qw"], c["sc"], c["zl"], c["N"], c["K"], c["group"], z[0],
                           z[1], y=c["y"], ws=c["ws"])
            elif self.actorder:
                q.qmm_actorder(c["x"], c["perm"], c["qw"], c["sc"], c["zl"], c["N"], c["K"],
                               c["mode"], c["bits"], c["group"], y=c["y"], ws=c["ws"])
            else:
                q.qmm(c["x"], c["qw"], c["sc"], c["zl"], c["N"], c["K"], c["mode"], c["bits"],
                      c["group"], y=c["y"], ws=c["ws"])

    def rounds(self, steps):
        """Graph replays that cover at least `steps` steps."""
        return max(1, -(-steps // self.copies))

    def time_steps(self, steps, warmup, barrier=lambda: None):
        """(device ms, steps timed): rounds covering `steps` steps (exactly
        `steps` when a round is one step) after rounds covering `warmup`, CUDA
        events on the replay stream, synchronized and barriered on both sides."""
        import torch
        with torch.cuda.stream(self.stream):
            for _ in range(self.rounds(warmup)):
                self.graph.replay()
            torch.cuda.synchronize()
            barrier()
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(self.stream)
            n = self.rounds(steps)
            for _ in range(n):
                self.graph.replay()
            e1.record(self.stream)
            torch.cuda.synchronize()
            barrier()
            torch.cuda.synchronize()
        return e0.elapsed_time(e1), n * self.copies

    def busy(self, seconds):
        """Replays for about `seconds` (so that clock samples see the GPU under load)."""
        import torch
        t_end = time.time() + seconds
        with torch.cuda.stream(self.stream):
            while time.time() < t_end:
                for _ in range(max(1, 50 // self.copies)):
                    self.graph.replay()
                torch.cuda.synchronize()

    def l2_note(self):
        return (f"inputs larger than L2: {self.copies} weight cop"
                f"{'y' if self.copies == 1 else 'ies'} of the step rotated, "
                f"{self.copies * self.codes_per_copy / 1e6:.0f} MB of codes in all "
                f"(L2 {L2_BYTES / 1e6:.0f} MB)")

    def result(self, ms_per_step, world=1):
        """(value, unit, roofline) of a measured step time."""
        if tensor_bound(self.name):
            peak, kind = tensor_peak()
            achieved = self.step_flops / (ms_per_step / 1e3) / 1e12
            roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                    "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "peak_source": kind}
            return world * achieved, "TFLOP/s", roof
        peak, kind = peaks()
        achieved = self.step_bytes / (ms_per_step / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "peak_source": kind}
        return world * achieved, "GB/s", roof

    def release(self):
        del self.graph, self.sets, self.xarenas, self.yarenas


def steps_for(wl, seconds, lo=20, hi=20000):
    """Timed steps worth about `seconds` of device time (from a short probe)."""
    ms, n = wl.time_steps(5, 2)
    return int(min(hi, max(lo, seconds * 1e3 / max(ms / n, 1e-4))))


def measure_configs(dev):
    """Every benchmark configuration with the headline's protocol (graphs of
    the step's calls, weights past L2, CUDA events), each with its roofline
    fraction: value, unit, ms per step and calls per step."""
    import torch
    out = {}
    for cfg, names in CONFIG_WORKLOADS.items():
        recs = []
        for name in names:
            wl = Workload(name, dev)
            ms, steps = wl.time_steps(steps_for(wl, 0.3), 5)
            ms /= steps
            value, unit, roof = wl.result(ms)
            recs.append({"workload": name, "value": round(value, 1), "unit": unit,
                         "frac": roof["frac"], "bound": roof["bound"],
                         "ms_per_step": round(ms, 5), "calls_per_step": wl.n_calls,
                         "steps": steps, "dtype": wl.dtype})
            wl.release()
            del wl
            torch.cuda.empty_cache()
        out[cfg] = recs
    return out


def run_ours(args, rank, world, local_rank):
    import torch
    import weight_only_quantized_int4_b200 as q

    torch.cuda.set_device(local_rank)
    q.load()
    dev = torch.device("cuda", local_rank)
    wl = Workload(args.workload, dev)
    actorder = wl.actorder

    dist = None
    if world > 1:
        import torch.distributed as dist

    def barrier():
        if dist is not None:
            dist.barrier()

    clock = ClockSampler(local_rank)
    clock.start()
    wl.busy(0.3)
    ms, steps = wl.time_steps(args.steps, args.warmup, barrier)
    ms = max_over_ranks(ms, dist, dev)
    clocks = clock.stop()
    ms_per_step = ms / steps
    value, unit, roofline = wl.result(ms_per_step, world)

    # ---- end to end through the public API: pinned host x in, y out, per step
    # (the calls are issued from Python one by one, not replayed from a graph)
    hx = wl.xarenas[0].cpu().pin_memory()
    hy = torch.empty_like(wl.yarenas[0], device="cpu").pin_memory()
    e2e_steps = max(3, min(args.steps, 50))
    with torch.cuda.stream(wl.stream):
        for i in range(2):
            wl.xarenas[i % wl.copies].copy_(hx, non_blocking=True)
            wl.step(i)
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(wl.stream)
        for i in range(e2e_steps):
            wl.xarenas[i % wl.copies].copy_(hx, non_blocking=True)
            wl.step(i)
            hy.copy_(wl.yarenas[i % wl.copies], non_blocking=True)
        a1.record(wl.stream)
        torch.cuda.synchronize()
        barrier()
    e2e_ms = max_over_ranks(a0.elapsed_time(a1), dist, dev)
    e2e_value, _, _ = wl.result(e2e_ms / e2e_steps, world)

    kernel = ("tc_kernel (all launches of the step)" if roofline["bound"] == "tensor" else
              "permute_x_kernel + skinny_kernel (all launches of the step)" if actorder else
              "skinny_kernel (all launches of the step)")
    roofline["kernel"] = kernel
    roofline["algorithmic_bytes_per_launch"] = round(wl.step_bytes / wl.n_calls)
    if roofline["bound"] == "tensor":
        roofline["algorithmic_flops_per_launch"] = wl.step_flops / wl.n_calls
        roofline["traffic"] = None
    else:
        # DRAM bytes per algorithmic byte come from the ncu capture of the
        # default workload; other workloads report none
        tpb = traffic_per_byte() if args.workload == "llama7b_decode" else None
        roofline["traffic"] = None if tpb is None else round(tpb * wl.step_bytes / wl.n_calls)
    w = WORKLOADS[args.workload]
    out = {"metric": METRIC, "value": round(value, 1), "unit": unit, "n_gpus": world,
           "steps": steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype,
           "data": "synthetic: seed-0 counter generator (SplitMix64 + Box-Muller, drawn on the "
                   "device), weights N(0, sigma) per the configs, activations N(0, 1)",
           "config": {"workload": args.workload, "calls_per_step": wl.n_calls,
                      "shapes_KN": w[4], "M": w[5], "mode": w[0], "group": w[2], "x_dtype": w[3],
                      **({"zero_group": wl.zopts[0], "zero_bits": wl.zopts[1]} if wl.zopts else {}),
                      **({"act_order": "random column order per matrix"} if actorder else {}),
                      "l2": wl.l2_note(),
                      "launch": "CUDA graph of the step, programmatic dependent launch",
                      "parallelism": f"replicas x{world}"},
           "roofline": roofline,
           "e2e": {"value": round(e2e_value, 1), "unit": unit, "h2d_bytes_per_step": hx.numel(),
                   "d2h_bytes_per_step": hy.numel(), "steps": e2e_steps,
                   "how": f"per step: the step's pinned x buffer -> device (one copy), the "
                          f"{wl.n_calls} calls issued one by one through the Python API (no "
                          "graph), the y buffer -> pinned host (one copy); CUDA events on the "
                          "stream"},
           "gpu_launches": wl.n_calls * steps * (2 if actorder else 1),
           "clocks": clocks}
    wl.release()
    del wl
    torch.cuda.empty_cache()
    if rank == 0 and args.workload == "llama7b_decode" and not args.no_configs and world == 1:
        cfgs = {"2_llama7b_decode": [{"workload": args.workload, "value": out["value"],
                                      "unit": unit, "frac": roofline["frac"],
                                      "bound": roofline["bound"], "ms_per_step": out["ms_per_step"],
                                      "calls_per_step": out["config"]["calls_per_step"],
                                      "steps": out["steps"], "dtype": out["dtype"],
                                      "note": "the headline measurement above"}]}
        cfgs.update(measure_configs(dev))
        out["configs"] = dict(sorted(cfgs.items()))
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args.workload, args.cpu_seconds,
                                           roofline["bound"] == "tensor")
    return out


# ------------------------------------------------------------------ CPU oracle

def _oracle_sample(workload, rows_per_problem, seed=0):
    """Host inputs of a sample: for every call, `rows_per_problem` rows of W."""
    import oracle
    from weight_only_quantized_int4_b200 import synth
    items = []
    gated = workload in GATED
    zopts = ZOPTS.get(workload)
    actorder = workload in ACTORDER
    for i, (mode, bits, group, xdt, M, K, N) in enumerate(problems(workload)):
        if gated:   # whole (gate, up) block pairs
            rows_per_problem = max(32, rows_per_problem // 32 * 32)
        rows = np.arange(rows_per_problem)
        W = synth.weights(seed, f"W{i}.0", N, K, SIGMA[mode], rows=rows)
        lut = None
        if mode == "lut":
            lut = {4: synth.nf4_table, 3: synth.nf3_table, 2: lambda: synth.lut2_table(0)}[bits]()
        x = synth.activations(seed, f"x{i}", M, K, xdt)
        n = rows_per_problem
        b = n / N * alg_bytes(mode, bits, group, M, K, N, gated, zopts, actorder)
        f = alg_flops(M, K, n)
        if zopts is not None:
            codes, scales, zeros = oracle.quantize_asym(W, group, zopts[0])
            qw, sp, zp = oracle.pack_asym(codes, scales, zeros, group, zopts[0], zopts[1])
            fn = (lambda a, b, x=x, xdt=xdt, qw=qw, sp=sp, zp=zp, M=M, n=n, K=K, group=group:
                  oracle.qmm_asym(x, xdt, qw, sp, zp, M, n, K, group, zopts[0], zopts[1], a, b))
            parts = n
        elif actorder:
            gidx = np.empty(K, np.int32)
            gidx[np.random.default_rng(seed + i).permutation(K)] = np.arange(K) // group
            codes, scales, zeros = oracle.quantize_gidx(W, mode, bits, group, gidx, lut=lut)
            qw, sp, zp = oracle.pack_gidx(codes, scales, zeros, gidx, mode, bits, group)
            zl = zp if mode == "asym" else lut
            fn = (lambda a, b, x=x, xdt=xdt, qw=qw, sp=sp, zl=zl, gidx=gidx, M=M, n=n, K=K,
                  mode=mode, bits=bits, group=group:
                  oracle.qmm_gidx(x, xdt, qw, sp, zl, gidx, M, n, K, mode, bits, group, a, b))
            parts = n
        else:
            codes, scales, zeros = oracle.quantize(W, mode, bits, group, lut=lut)
            qw, sp, zp = oracle.pack(codes, scales, zeros, mode, bits, group)
            zl = zp if mode == "asym" else lut
            if gated:   # outputs i = 0 .. n/2 - 1
                fn = (lambda a, b, x=x, xdt=xdt, qw=qw, sp=sp, zl=zl, M=M, n=n, K=K, mode=mode,
                      bits=bits, group=group:
                      oracle.qmm_gated(x, xdt, qw, sp, zl, M, n // 2, K, mode, bits, group, a, b))
                parts = n // 2
            else:
                fn = (lambda a, b, x=x, xdt=xdt, qw=qw, sp=sp, zl=zl, M=M, n=n, K=K, mode=mode,
                      bits=bits, group=group:
                      oracle.qmm(x, xdt, qw, sp, zl, M, n, K, mode, bits, group, a, b))
                parts = n
        items.append((fn, parts, b, f))
    return items


def _split_run(fn, parts, threads):
    """fn(a, b) over [0, parts) in `threads` contiguous ranges on host threads
    (ctypes releases the GIL during each oracle call)."""
    bounds = np.linspace(0, parts, threads + 1).astype(int)
    ts = [threading.Thread(target=fn, args=(int(bounds[i]), int(bounds[i + 1])))
          for i in range(threads) if bounds[i + 1] > bounds[i]]
    for t in ts:
        t.start()
    for t in ts:
        t.join()


def _run_oracle(items, threads, flops=False):
    """Runs every sampled call, its output columns split over `threads` host
    threads; returns (seconds, algorithmic bytes or flops)."""
    t0 = time.perf_counter()
    total = 0.0
    for fn, parts, b, f in items:
        _split_run(fn, parts, threads)
        total += f if flops else b
    return time.perf_counter() - t0, total


def cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(workload, seconds, tensor=False):
    """The oracle (plain C++, double sums) on a bounded sample of the workload:
    the same calls restricted to their first R rows of W (whole 16-row
    blocks), R chosen so the timed run takes about `seconds`.  Reported in the
    bench line's unit (GB/s of algorithmic bytes, or TFLOP/s)."""
    threads = cpu_threads()
    probe = _oracle_sample(workload, 16)
    dt, _ = _run_oracle(probe, threads)
    rows = int(16 * max(1, round(seconds / max(dt, 1e-3))))
    rows = max(16, min(rows // 16 * 16, 4096))
    items = _oracle_sample(workload, rows)
    dt, work = _run_oracle(items, threads, tensor)
    # the sample's inputs are capped (they are generated on the host); repeat
    # the oracle on them until the CPU work reaches about `seconds`
    reps = max(1, int(round(seconds / max(dt, 1e-3))))
    for _ in range(reps - 1):
        d, w = _run_oracle(items, threads, tensor)
        dt += d
        work += w
    what = (f"{work / reps / 1e9:.2f} GFLOP" if tensor
            else f"{work / reps / 1e6:.1f} MB of algorithmic bytes")
    scale = 1e12 if tensor else 1e9
    # the same oracle on one host thread, on a smaller sample (16 rows per call)
    one_items = _oracle_sample(workload, 16)
    dt1, work1 = _run_oracle(one_items, 1, tensor)
    reps1 = max(1, int(round(min(seconds / 2, 5.0) / max(dt1, 1e-3))))
    for _ in range(reps1 - 1):
        d, w = _run_oracle(one_items, 1, tensor)
        dt1 += d
        work1 += w
    return {"value": round(work / dt / scale, 6),
            "unit": "TFLOP/s" if tensor else "GB/s", "cores": threads,
            "kind": "oracle", "seconds": round(dt, 2),
            "sample": f"every call of the step on its first {rows} rows of W "
                      f"({what}), run {reps} times, columns split over {threads} threads",
            "single_thread": {"value": round(work1 / dt1 / scale, 6),
                              "unit": "TFLOP/s" if tensor else "GB/s", "cores": 1,
                              "seconds": round(dt1, 2),
                              "sample": f"every call of the step on its first 16 rows of W, "
                                        f"run {reps1} times on one thread"}}


def run_reference(args):
    """The oracle as the reference arm: each step is the bounded CPU sample."""
    threads = cpu_threads()
    probe = _oracle_sample(args.workload, 16)
    dt, _ = _run_oracle(probe, threads)
    budget = max(2.0, 120.0 / max(1, args.steps + args.warmup))   # whole run ~2 minutes
    rows = max(16, min(int(16 * round(budget / max(dt, 1e-3))) // 16 * 16, 4096))
    items = _oracle_sample(args.workload, rows)
    tensor = tensor_bound(args.workload)
    unit = "TFLOP/s" if tensor else "GB/s"
    for _ in range(args.warmup):
        _run_oracle(items, threads, tensor)
    tot_t, tot_b = 0.0, 0.0
    for _ in range(args.steps):
        t, b = _run_oracle(items, threads, tensor)
        tot_t += t
        tot_b += b
    value = tot_b / tot_t / (1e12 if tensor else 1e9)
    sample = (f"every call of the step on its first {rows} rows of W, columns split over "
              f"{threads} threads")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": unit,
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * tot_t / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "calls_per_step": len(items)},
            "cpu_baseline": {"value": round(value, 6), "unit": unit, "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=list(WORKLOADS), default="llama7b_decode")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other benchmark configurations after the default workload")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    out = run_ours(args, rank, world, local_rank)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
