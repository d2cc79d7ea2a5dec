#!/usr/bin/env python
"""Benchmark of the affine group-quantized GEMV on B200.

Default workload: the decode bit-width sweep (M=1, K=4096, N=14336,
group_size=64, bits in {2,3,4,5,6,8}).  One step = one quantized GEMV at each
of the six bit widths (six kernel launches).  Metric: achieved HBM GB/s over
the step, with algorithmic bytes = packed W + scales + biases + x + y.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode_sweep|qmv_small|ffn_int8|batched|moe_gather]

Prints ONE JSON line on rank 0.  Under torchrun (N > 1) every rank runs the
same workload on its own GPU (independent replicas, no collective on the data
path); the step time is the max over ranks and `value` counts all ranks' bytes.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from affine_group_quantized_b200 import synth  # noqa: E402

METRIC = "quantized GEMV achieved HBM GB/s (and % of B200 peak); tokens/s-equivalent"
UNIT = "GB/s"
L2_BYTES = 126 * 1024 * 1024


# ---------------------------------------------------------------------------
# Workloads: host inputs + algorithmic byte counts (shared by both arms)
# ---------------------------------------------------------------------------

def qmv_bytes(M, N, K, bits, gs):
    return N * K * bits // 8 + 2 * 2 * N * (K // gs) + 2 * M * K + 2 * M * N


def quant_bytes(N, K, bits, gs):
    """Bytes one quantize (or dequantize) of an [N, K] matrix moves: the bf16
    matrix, the packed codes, and the bf16 scales and biases."""
    return 2 * N * K + N * K * bits // 8 + 2 * 2 * N * (K // gs)


class Launch:
    """One kernel launch of a step: label, algorithmic bytes, host inputs."""

    def __init__(self, label, kind, nbytes, **kw):
        self.label, self.kind, self.nbytes = label, kind, nbytes
        self.__dict__.update(kw)


def workload(name):
    L = []
    if name == "decode_sweep":
        M, N, K, gs = 1, 14336, 4096, 64
        for bits in (2, 3, 4, 5, 6, 8):
            x, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=2000 + bits)
            L.append(Launch(f"qmv_b{bits}", "qmv", qmv_bytes(M, N, K, bits, gs),
                            M=M, N=N, K=K, bits=bits, gs=gs, x=x, w=w, s=s, b=b))
        cfg = {"workload": "decode GEMV bit sweep", "M": M, "K": K, "N": N,
               "group_size": gs, "bits": [2, 3, 4, 5, 6, 8]}
    elif name == "qmv_small":
        M, N, K, bits, gs = 1, 256, 512, 4, 64
        x, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=1000, bias_jitter=1e-3)
        L.append(Launch("qmv_small", "qmv", qmv_bytes(M, N, K, bits, gs),
                        M=M, N=N, K=K, bits=bits, gs=gs, x=x, w=w, s=s, b=b))
        cfg = {"workload": "single small qmv", "M": M, "K": K, "N": N,
               "group_size": gs, "bits": bits}
    elif name == "ffn_int8":
        M, N, K, bits, gs = 1, 14336, 4096, 8, 64
        kw = dict(scale_lo=0.002, scale_hi=0.01)
        x, wg, sg, bg = synth.qmv_inputs(M, N, K, bits, gs, seed=3000, **kw)
        _, wu, su, bu = synth.qmv_inputs(M, N, K, bits, gs, seed=3001, **kw)
        _, wd, sd, bd = synth.qmv_inputs(M, K, N, bits, gs, seed=3002, **kw)
        resid = synth.normal_bf16((M, K), seed=3003)
        gu_bytes = 2 * (N * K + 4 * N * (K // gs)) + 2 * K + 2 * 2 * N
        dn_bytes = K * N + 4 * K * (N // gs) + 2 * 2 * N + 2 * K + 2 * K
        L.append(Launch("gate_up_int8", "gate_up", gu_bytes, M=M, N=N, K=K, bits=bits,
                        gs=gs, x=x, wg=wg, sg=sg, bg=bg, wu=wu, su=su, bu=bu))
        L.append(Launch("silu_down_int8", "silu", dn_bytes, M=M, N=K, K=N, bits=bits,
                        gs=gs, w=wd, s=sd, b=bd, resid=resid))
        cfg = {"workload": "fused FFN decode int8", "K": K, "N": N, "group_size": gs,
               "bits": bits}
    elif name == "batched":
        N, K, bits = 28672, 8192, 4
        for gs in (32, 128):
            for M in (1, 2, 4, 8):
                x, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=4000 + 10 * M + gs)
                L.append(Launch(f"qmv_M{M}_gs{gs}", "qmv", qmv_bytes(M, N, K, bits, gs),
                                M=M, N=N, K=K, bits=bits, gs=gs, x=x, w=w, s=s, b=b))
        cfg = {"workload": "batched decode qmv", "M": [1, 2, 4, 8], "K": K, "N": N,
               "group_size": [32, 128], "bits": bits}
    elif name == "moe_gather":
        E, N, K, bits, gs, T, k = 64, 1536, 2048, 4, 64, 32, 4
        _, w, s, b = synth.qmv_inputs(1, E * N, K, bits, gs, seed=5000)
        x = synth.normal_bf16((T, K), seed=5001)
        lhs, rhs = synth.topk_routing(T, E, k, seed=5002)
        lhs_s, rhs_s, _ = synth.sort_pairs_by_expert(lhs, rhs)
        touched = len(np.unique(rhs))
        per_expert = N * K * bits // 8 + 4 * N * (K // gs)
        nb = touched * per_expert + 2 * T * K + 2 * T * k * N + 2 * 4 * T * k
        for srt, (l_, r_) in (("unsorted", (lhs, rhs)), ("sorted", (lhs_s, rhs_s))):
            L.append(Launch(f"gather_{srt}", "gather", nb, E=E, N=N, K=K, bits=bits,
                            gs=gs, T=T, P=T * k, x=x, w=w, s=s, b=b, lhs=l_, rhs=r_,
                            sorted=srt == "sorted"))
        cfg = {"workload": "MoE gather_qmv", "experts": E, "N": N, "K": K, "bits": bits,
               "group_size": gs, "tokens": T, "top_k": k, "touched_experts": touched}
    elif name == "quantize":
        # the producer side of the format on the decode weight shape: one
        # quantize of a bf16 matrix and one dequantize of a packed matrix
        N, K, bits, gs = 14336, 4096, 4, 64
        w = synth.normal_bf16((N, K), seed=6000)
        _, wq, s, b = synth.qmv_inputs(1, N, K, bits, gs, seed=6001)
        nb = quant_bytes(N, K, bits, gs)
        L.append(Launch(f"quantize_b{bits}", "quantize", nb, N=N, K=K, bits=bits, gs=gs,
                        w=w))
        L.append(Launch(f"dequantize_b{bits}", "dequantize", nb, N=N, K=K, bits=bits,
                        gs=gs, w=wq, s=s, b=b))
        cfg = {"workload": "affine quantize + dequantize", "N": N, "K": K,
               "group_size": gs, "bits": bits}
    else:
        raise SystemExit(f"unknown workload {name}")
    return L, cfg


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def _dev(a, torch):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a.view(np.int32)).cuda()


class DeviceLaunch:
    """Device buffers of one Launch, with `copies` rotating weight copies."""

    def __init__(self, l, copies, torch):
        import affine_group_quantized_b200 as agq
        self.l, self.agq, self.torch = l, agq, torch
        d = lambda a: _dev(a, torch)  # noqa: E731
        self.copies = []
        for _ in range(copies):
            if l.kind == "qmv":
                self.copies.append(dict(w=d(l.w), s=d(l.s), b=d(l.b)))
            elif l.kind == "gate_up":
                self.copies.append(dict(wg=d(l.wg), sg=d(l.sg), bg=d(l.bg),
                                        wu=d(l.wu), su=d(l.su), bu=d(l.bu)))
            elif l.kind == "silu":
                self.copies.append(dict(w=d(l.w), s=d(l.s), b=d(l.b)))
            elif l.kind == "gather":
                self.copies.append(dict(w=d(l.w), s=d(l.s), b=d(l.b)))
        bf = torch.bfloat16
        if l.kind == "qmv":
            self.x = d(l.x)
            self.y = torch.empty((l.M, l.N), dtype=bf, device="cuda")
        elif l.kind == "gate_up":
            self.x = d(l.x)
            self.yg = torch.empty((l.M, l.N), dtype=bf, device="cuda")
            self.yu = torch.empty((l.M, l.N), dtype=bf, device="cuda")
            self.y = self.yg
        elif l.kind == "silu":
            # input of the down projection: gate/up activations (synthetic)
            self.gate = d(synth.normal_bf16((l.M, l.K), seed=3004))
            self.up = d(synth.normal_bf16((l.M, l.K), seed=3005))
            self.x = self.gate
            self.resid = d(l.resid)
            self.y = torch.empty((l.M, l.N), dtype=bf, device="cuda")
        elif l.kind == "gather":
            self.x = d(l.x)
            self.lhs, self.rhs = d(l.lhs), d(l.rhs)
            self.y = torch.empty((l.P, l.N), dtype=bf, device="cuda")

    def __call__(self, k):
        l, c, agq = self.l, self.copies[k % len(self.copies)], self.agq
        if l.kind == "qmv":
            agq.qmv(self.x, c["w"], c["s"], c["b"], self.y, l.M, l.N, l.K, l.bits, l.gs)
        elif l.kind == "gate_up":
            agq.qmv_gate_up(self.x, c["wg"], c["sg"], c["bg"], c["wu"], c["su"], c["bu"],
                            self.yg, self.yu, l.M, l.N, l.K, l.bits, l.gs)
        elif l.kind == "silu":
            agq.qmv_silu_gate_resid(self.gate, self.up, self.resid, c["w"], c["s"], c["b"],
                                    self.y, l.M, l.N, l.K, l.bits, l.gs)
        elif l.kind == "gather":
            agq.gather_qmv(self.x, c["w"], c["s"], c["b"], self.lhs, self.rhs, self.y,
                           l.P, l.T, l.E, l.N, l.K, l.bits, l.gs, sorted_indices=l.sorted)


class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML while running."""

    def __init__(self, torch):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.ok = False
        try:
            import pynvml as nv
            nv.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            try:
                self.h = nv.nvmlDeviceGetHandleByUUID(uuid)
            except Exception:  # noqa: BLE001  (older bindings take bytes)
                self.h = nv.nvmlDeviceGetHandleByUUID(uuid.encode())
            self.nv = nv
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = repr(e)
        self._stop = threading.Event()

    _REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting",
                0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x10: "sync_boost",
                0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
                0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self._REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.err}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(self.samples)}


# The sources the GEMV kernels and their launch plans are built from: the
# recorded DRAM traffic is valid while these are unchanged.  (The producer
# side of the format, qmv_quant.cu, has kernels of its own.)
GEMV_SOURCES = ("qmv_api.cu", "qmv_device.cuh", "qmv_mma.cuh", "qmv_stream.cuh")


def source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "affine_group_quantized_b200", "csrc")
    for f in sorted(GEMV_SOURCES):
        p = os.path.join(csrc, f)
        if not os.path.exists(p):
            continue
        with open(p, "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def recorded_traffic(kernel_label, workload_name):
    """DRAM bytes per launch from a committed ncu summary, if the kernel
    source has not changed since it was captured."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload_name, {}).get(kernel_label)
    if not e or e.get("source_hash") != source_hash():
        return None
    return e.get("dram_bytes_per_launch")


def max_over_ranks(value, device):
    """The largest of `value` over the ranks of the default process group
    (the slowest replica times the job); the value itself with one rank."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbs(world, bytes_per_step, steps, ms):
    """Whole-job throughput: every replica's bytes over the slowest time."""
    return world * bytes_per_step * steps / (ms * 1e-3) / 1e9


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    import affine_group_quantized_b200 as agq
    agq.lib()

    launches, cfg = workload(args.workload)
    step_bytes = sum(l.nbytes for l in launches)
    # Inputs larger than L2: rotate weight copies so that more than twice the
    # L2 capacity streams through between two reads of the same bytes.  Small
    # workloads instead flush L2 before every step (outside the per-launch
    # events, which then give the value).
    flush = step_bytes < 64 * 2**20
    copies = 1 if flush else max(2, -(-2 * L2_BYTES // step_bytes) + 1)
    # Each launch also gets enough weight copies that timing it alone (below)
    # streams more than twice the L2 capacity between two reads of the same
    # bytes; a step uses the first `copies` of them.
    dls = [DeviceLaunch(l, copies if flush else max(copies, -(-2 * L2_BYTES // l.nbytes) + 1),
                        torch) for l in launches]
    scrub = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda") if flush else None

    def step(k):
        if scrub is not None:
            scrub.fill_(k & 0xFF)
        for dl in dls:
            dl(k)

    for k in range(max(args.warmup, copies)):
        step(k)
    torch.cuda.synchronize()

    # Every timed region replays CUDA graphs captured from the public API
    # calls, so the host's per-call enqueue cost does not pace the GPU.
    # graphs[c] = one full step using weight copy c; cycle = the `copies`
    # steps of one rotation in a single graph (fewer graph launches per
    # step, as a decode loop captured whole would run).
    graphs = []
    for c in range(copies):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step(c)
        graphs.append(g)
    cycle = torch.cuda.CUDAGraph()
    with torch.cuda.graph(cycle):
        for c in range(copies):
            step(c)
    for c in range(copies):
        graphs[c].replay()
    cycle.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()

    K = args.steps
    stream = torch.cuda.current_stream()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(torch)
    torch.cuda.synchronize()
    with sampler:
        t0.record(stream)
        for _ in range(K // copies):  # exactly K steps: whole rotations ...
            cycle.replay()
        for k in range(K % copies):   # ... then the remaining single steps
            graphs[k].replay()
        t1.record(stream)
        torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), "cuda")

    # Average duration of each launch: a graph of R back-to-back launches of
    # that kernel alone (rotating through all of its weight copies, more than
    # twice the L2 capacity; L2 scrubbed first for the small workloads), timed
    # with events around the replays.
    dur = []
    for dl in dls:
        R = 3 * len(dl.copies)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for r in range(R):
                if scrub is not None:
                    scrub.fill_(r & 0xFF)
                dl(r)
        g.replay()
        torch.cuda.synchronize()
        reps = max(1, min(200, (K * len(dls)) // R))
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b_.record(stream)
        torch.cuda.synchronize()
        d = a.elapsed_time(b_) / (reps * R)
        if scrub is not None:  # remove the scrub's own time
            gs_ = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gs_):
                for r in range(R):
                    scrub.fill_(r & 0xFF)
            gs_.replay()
            torch.cuda.synchronize()
            a.record(stream)
            for _ in range(reps):
                gs_.replay()
            b_.record(stream)
            torch.cuda.synchronize()
            d -= a.elapsed_time(b_) / (reps * R)
        dur.append(d)

    # End to end through the public API: per step, copy x in from pinned host
    # memory, run the step's launches, copy y out to pinned host memory (one
    # CUDA graph per step).
    hx = [dl.x.detach().cpu().pin_memory() for dl in dls]
    hy = [torch.empty_like(dl.y, device="cpu").pin_memory() for dl in dls]
    h2d = sum(t.numel() * t.element_size() for t in hx)
    d2h = sum(t.numel() * t.element_size() for t in hy)

    def e2e_step(k):
        for i, dl in enumerate(dls):
            dl.x.copy_(hx[i], non_blocking=True)
            dl(k)
            hy[i].copy_(dl.y, non_blocking=True)

    for k in range(copies):
        e2e_step(k)
    torch.cuda.synchronize()
    egraphs = []
    for c in range(copies):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            e2e_step(c)
        egraphs.append(g)
    for g in egraphs:
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for k in range(K):
        egraphs[k % copies].replay()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), "cuda")
    del graphs, egraphs

    peak, peak_kind = measured_peaks()
    per = {}
    for l, d in zip(launches, dur):
        gbs = l.nbytes / (d * 1e-3) / 1e9
        per[l.label] = {"us": round(d * 1e3, 3), "GB/s": round(gbs, 1),
                        "frac_of_measured_peak": round(gbs / peak, 4),
                        "bytes": l.nbytes}
    dom = max(range(len(dls)), key=lambda i: dur[i])
    ach = launches[dom].nbytes / (dur[dom] * 1e-3) / 1e9
    value = job_gbs(world, step_bytes, K, ms)
    if flush:  # the step region includes the L2 scrub: use kernel time only
        value = world * step_bytes / (sum(dur) * 1e-3) / 1e9
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms / K, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32 accumulate (bf16 in/out)", "data": "synthetic",
        "config": dict(cfg, l2=(f"L2 flushed before every step ({2 * L2_BYTES >> 20} MiB "
                                f"write); value from per-launch events" if flush else
                                f"inputs larger than L2: {copies} rotating weight copies, "
                                f"{step_bytes * copies / 2**20:.0f} MiB between reuse; each "
                                f"launch timed alone rotates through more than "
                                f"{2 * L2_BYTES >> 20} MiB of its own copies"),
                       parallelism=f"replicas x{world}" if world > 1 else "single GPU",
                       graphs=f"timed steps replayed as CUDA graphs of {copies} steps (one "
                              f"weight rotation); the remainder one step per graph"),
        "roofline": {"bound": "hbm", "kernel": launches[dom].label,
                     "achieved": round(ach, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(ach / peak, 4), "peak_kind": peak_kind,
                     "traffic": recorded_traffic(launches[dom].label, args.workload),
                     "algorithmic_bytes_per_launch": launches[dom].nbytes},
        "per_launch": per,
        "tokens_per_s_equiv": {l.label: round(1e6 / (d * 1e3), 1)
                               for l, d in zip(launches, dur)},
        "e2e": {"value": round(job_gbs(world, step_bytes, K, e2e_ms), 1),
                "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "note": "weights resident in HBM (decode); x copied in and y copied "
                        "out every step; each step replayed as one CUDA graph"},
        "gpu_launches": K * len(dls),
        "clocks": sampler.summary(),
        "source_hash": source_hash(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(launches, budget_s=args.cpu_budget)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_quant(args):
    """GPU arm of the quantize workload: one step = affine_quantize of a bf16
    matrix and affine_dequantize of a packed one.  Inputs rotate through
    copies so that more than twice the L2 capacity streams between two reads
    of the same bytes; the dequantize of step k reads the codes the quantize
    of an earlier step wrote (copy k + 1), so it never reads L2-hot output."""
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    import affine_group_quantized_b200 as agq
    agq.lib()

    launches, cfg = workload("quantize")
    lq, ld = launches
    N, K, bits, gs = lq.N, lq.K, lq.bits, lq.gs
    step_bytes = lq.nbytes + ld.nbytes
    copies = max(3, -(-2 * L2_BYTES // (2 * N * K)) + 1)
    bf, i32, i16 = torch.bfloat16, torch.int32, torch.int16
    W = [_dev(lq.w, torch) for _ in range(copies)]
    Q = [_dev(ld.w, torch) for _ in range(copies)]
    S = [_dev(ld.s, torch) for _ in range(copies)]
    B = [_dev(ld.b, torch) for _ in range(copies)]
    Y = torch.empty((N, K), dtype=bf, device="cuda")

    def quant(k):
        c = k % copies
        agq.affine_quantize(W[c], Q[c], S[c], B[c], N, K, bits, gs)

    def dequant(k):
        c = (k + 1) % copies
        agq.affine_dequantize(Q[c], S[c], B[c], Y, N, K, bits, gs)

    def step(k):
        quant(k)
        dequant(k)

    for k in range(max(args.warmup, copies)):
        step(k)
    torch.cuda.synchronize()
    graphs = []
    for c in range(copies):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step(c)
        graphs.append(g)
    for g in graphs:
        g.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()

    Ks = args.steps
    stream = torch.cuda.current_stream()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(torch)
    torch.cuda.synchronize()
    with sampler:
        t0.record(stream)
        for k in range(Ks):
            graphs[k % copies].replay()
        t1.record(stream)
        torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), "cuda")

    # each kernel alone: a graph of 3 * copies back-to-back launches
    dur = []
    for fn in (quant, dequant):
        R = 3 * copies
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for r in range(R):
                fn(r)
        g.replay()
        torch.cuda.synchronize()
        reps = max(1, min(100, 2 * Ks // R))
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b_.record(stream)
        torch.cuda.synchronize()
        dur.append(a.elapsed_time(b_) / (reps * R))

    # end to end: the bf16 matrix in from pinned host memory, quantize,
    # dequantize the result, and the packed matrix and the bf16 round trip out
    hw = W[0].detach().cpu().pin_memory()
    outs = (Q[0], S[0], B[0], Y)
    houts = [torch.empty_like(t, device="cpu").pin_memory() for t in outs]
    h2d = hw.numel() * hw.element_size()
    d2h = sum(t.numel() * t.element_size() for t in houts)

    def e2e_step():
        W[0].copy_(hw, non_blocking=True)
        agq.affine_quantize(W[0], Q[0], S[0], B[0], N, K, bits, gs)
        agq.affine_dequantize(Q[0], S[0], B[0], Y, N, K, bits, gs)
        for h, d in zip(houts, outs):
            h.copy_(d, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    eg = torch.cuda.CUDAGraph()
    with torch.cuda.graph(eg):
        e2e_step()
    eg.replay()
    torch.cuda.synchronize()
    ek = max(3, min(Ks, 20))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(ek):
        eg.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), "cuda")
    del graphs, eg

    peak, peak_kind = measured_peaks()
    per = {}
    for l, d in zip(launches, dur):
        gbs = l.nbytes / (d * 1e-3) / 1e9
        per[l.label] = {"us": round(d * 1e3, 3), "GB/s": round(gbs, 1),
                        "frac_of_measured_peak": round(gbs / peak, 4), "bytes": l.nbytes}
    dom = 0 if dur[0] >= dur[1] else 1
    ach = launches[dom].nbytes / (dur[dom] * 1e-3) / 1e9
    out = {
        "metric": METRIC, "value": round(job_gbs(world, step_bytes, Ks, ms), 1),
        "unit": UNIT, "n_gpus": world, "steps": Ks, "warmup": args.warmup,
        "ms_per_step": round(ms / Ks, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32 (bf16 in/out)", "data": "synthetic",
        "config": dict(cfg, l2=f"inputs larger than L2: {copies} rotating copies of every "
                               f"input; dequantize reads codes written one step earlier",
                       parallelism=f"replicas x{world}" if world > 1 else "single GPU",
                       graphs="timed steps replayed as one CUDA graph per step"),
        "roofline": {"bound": "hbm", "kernel": launches[dom].label, "achieved": round(ach, 1),
                     "peak": peak, "unit": "GB/s", "frac": round(ach / peak, 4),
                     "peak_kind": peak_kind,
                     "traffic": recorded_traffic(launches[dom].label, "quantize"),
                     "algorithmic_bytes_per_launch": launches[dom].nbytes},
        "per_launch": per,
        "e2e": {"value": round(job_gbs(world, step_bytes, ek, e2e_ms), 1), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "note": "bf16 matrix copied in, packed matrix and round trip copied out "
                        "every step; each step replayed as one CUDA graph"},
        "gpu_launches": 2 * Ks,
        "clocks": sampler.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(launches, budget_s=args.cpu_budget)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# CPU oracle arm (reference) and CPU baseline
# ---------------------------------------------------------------------------

def _oracle_launch(l, rows, nthreads):
    import oracle
    if l.kind == "qmv":
        oracle.qmv(l.x, l.w, l.s, l.b, l.M, l.N, l.K, l.bits, l.gs, rows=rows,
                   nthreads=nthreads)
    elif l.kind == "gate_up":
        oracle.qmv(l.x, l.wg, l.sg, l.bg, l.M, l.N, l.K, l.bits, l.gs, rows=rows,
                   nthreads=nthreads)
        oracle.qmv(l.x, l.wu, l.su, l.bu, l.M, l.N, l.K, l.bits, l.gs, rows=rows,
                   nthreads=nthreads)
    elif l.kind == "silu":
        g = synth.normal_bf16((l.M, l.K), seed=3004)
        u = synth.normal_bf16((l.M, l.K), seed=3005)
        oracle.silu_gate_resid(g, u, l.resid, l.w, l.s, l.b, l.M, l.N, l.K, l.bits,
                               l.gs, rows=rows, nthreads=nthreads)
    elif l.kind == "gather":
        oracle.gather(l.x, l.w, l.s, l.b, l.lhs, l.rhs, l.P, l.T, l.E, l.N, l.K,
                      l.bits, l.gs, nthreads=nthreads)
    elif l.kind == "quantize":
        n = l.N if rows is None else len(rows)
        oracle.affine_quantize(l.w[:n], n, l.K, l.bits, l.gs)
    elif l.kind == "dequantize":
        n = l.N if rows is None else len(rows)
        oracle.dequantize_bf16(l.w[:n], l.s[:n], l.b[:n], n, l.K, l.bits, l.gs)


QUANT_KINDS = ("quantize", "dequantize")


def _threads_used(launches, nthreads):
    """The oracle's GEMVs run on `nthreads` threads; its quantizer and
    dequantizer on one."""
    return 1 if all(l.kind in QUANT_KINDS for l in launches) else nthreads


def _sample(l, frac):
    """Rows evaluated per launch and the bytes that sample stands for."""
    if l.kind == "gather":
        return None, l.nbytes
    nr = max(1, int(l.N * frac))
    rows = np.arange(nr, dtype=np.int32)
    return rows, int(l.nbytes * nr / l.N)


def cpu_baseline(launches, budget_s=20.0, frac=None):
    import oracle  # noqa: F401  (loads liboracle.so)
    nthreads = len(os.sched_getaffinity(0))
    if frac is None:
        # calibrate on a small slice, then size the sample to the budget
        t = time.perf_counter()
        nb = 0
        for l in launches:
            rows, b = _sample(l, 1 / 64)
            _oracle_launch(l, rows, nthreads)
            nb += b
        dt = time.perf_counter() - t
        full = sum(l.nbytes for l in launches)
        frac = min(1.0, max(1 / 64, budget_s / max(dt * full / max(nb, 1), 1e-9)))
    # whole passes over the sample until about half the budget has run
    t = time.perf_counter()
    nb = 0
    passes = 0
    while passes == 0 or (time.perf_counter() - t < budget_s / 2 and passes < 64):
        for l in launches:
            rows, b = _sample(l, frac)
            _oracle_launch(l, rows, nthreads)
            nb += b
        passes += 1
    dt = time.perf_counter() - t
    return {"value": round(nb / dt / 1e9, 4), "unit": UNIT,
            "cores": _threads_used(launches, nthreads),
            "kind": "oracle", "seconds": round(dt, 2),
            "sample": f"{passes} pass(es) over the first {frac:.3f} of the rows of "
                      f"every launch of one step (gather: all pairs), plain-C "
                      f"oracle, {_threads_used(launches, nthreads)} thread(s)"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    launches, cfg = workload(args.workload)
    nthreads = len(os.sched_getaffinity(0))
    # bounded sample per step so the whole run stays within a few minutes
    total_steps = args.steps + args.warmup
    frac = min(1.0, 8.0 / max(total_steps, 1))
    for _ in range(args.warmup):
        for l in launches:
            _oracle_launch(l, _sample(l, frac)[0], nthreads)
    t = time.perf_counter()
    nb = 0
    for _ in range(args.steps):
        for l in launches:
            rows, b = _sample(l, frac)
            _oracle_launch(l, rows, nthreads)
            nb += b
    dt = time.perf_counter() - t
    value = nb / dt / 1e9
    out = {"metric": METRIC, "value": round(value, 4), "unit": UNIT,
           "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(dt * 1e3 / max(args.steps, 1), 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
           "dtype": "f32 quantize, f64 dequantize" if args.workload == "quantize" else "f64",
           "data": "synthetic", "config": cfg, "impl": "reference",
           "cpu_baseline": {"value": round(value, 4), "unit": UNIT,
                            "cores": _threads_used(launches, nthreads),
                            "kind": "oracle",
                            "sample": f"first {frac:.3f} of the rows of every launch per "
                                      f"step (gather: all pairs)"},
           "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0},
           "gpu_launches": 0}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode_sweep",
                    choices=["decode_sweep", "qmv_small", "ffn_int8", "batched",
                             "moe_gather", "quantize"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "quantize":
        run_quant(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
