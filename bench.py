#!/usr/bin/env python
"""Benchmark of the affine group-quantized GEMV on B200.

Default workload: the decode bit-width sweep (M=1, K=4096, N=14336,
group_size=64, bits in {2,3,4,5,6,8}).  One step = one quantized GEMV at each
of the six bit widths (six kernel launches).  Metric: achieved HBM GB/s over
the step, with algorithmic bytes = packed W + scales + biases + x + y.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode_sweep|qmv_small|ffn_int8|batched|prefill|moe_gather|...]

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
import torch

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
        # input of the down projection: gate and up activations (synthetic)
        gate = synth.normal_bf16((M, N), seed=3004)
        up = synth.normal_bf16((M, N), seed=3005)
        gu_bytes = 2 * (N * K + 4 * N * (K // gs)) + 2 * K + 2 * 2 * N
        dn_bytes = K * N + 4 * K * (N // gs) + 2 * 2 * N + 2 * K + 2 * K
        L.append(Launch("gate_up_int8", "gate_up", gu_bytes, M=M, N=N, K=K, bits=bits,
                        gs=gs, x=x, wg=wg, sg=sg, bg=bg, wu=wu, su=su, bu=bu))
        L.append(Launch("silu_down_int8", "silu", dn_bytes, M=M, N=K, K=N, bits=bits,
                        gs=gs, w=wd, s=sd, b=bd, resid=resid, gate=gate, up=up))
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
    elif name == "prefill":
        # many activation rows (the pages' qmm_t) on the batched matrix: the
        # tensor-core contraction; M=32 is memory bound, M=128 tensor bound
        N, K, bits = 28672, 8192, 4
        for gs in (32, 128):
            for M in (32, 128):
                x, w, s, b = synth.qmv_inputs(M, N, K, bits, gs, seed=4500 + M + gs)
                L.append(Launch(f"qmm_M{M}_gs{gs}", "qmv", qmv_bytes(M, N, K, bits, gs),
                                M=M, N=N, K=K, bits=bits, gs=gs, x=x, w=w, s=s, b=b,
                                flops=2 * M * N * K))
        cfg = {"workload": "prefill qmm", "M": [32, 128], "K": K, "N": N,
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
    elif name == "qvm":
        # the non-transposed product over the decode weight shape read the
        # other way: x [1, 14336] @ dequant(W [14336 rows of 4096 codes])
        M, K, N, bits, gs = 1, 14336, 4096, 4, 64
        _, w, s, b = synth.qmv_inputs(1, K, N, bits, gs, seed=7004)
        x = synth.normal_bf16((M, K), seed=7005)
        nb = K * N * bits // 8 + 2 * 2 * K * (N // gs) + 2 * M * K + 2 * M * N
        L.append(Launch(f"qvm_b{bits}", "qvm", nb, M=M, K=K, N=N, bits=bits, gs=gs,
                        x=x, w=w, s=s, b=b))
        cfg = {"workload": "qvm (x @ dequant(W))", "M": M, "K": K, "N": N,
               "group_size": gs, "bits": bits}
    elif name == "trellis":
        # the trellis-mode decode GEMV on the decode shape, 2- and 4-bit
        M, N, K = 1, 14336, 4096
        for bits in (2, 4):
            rng = np.random.default_rng(8100 + bits)
            w = rng.integers(0, 1 << 32, size=(N, K * bits // 32), dtype=np.uint64).astype(np.uint32)
            x = synth.normal_bf16((M, K), seed=8110 + bits)
            s = synth.bf16_bits(torch.tensor([0.0123]))
            nb = N * K * bits // 8 + 2 + 2 * M * K + 2 * M * N
            # ALU bound: per value the state's inst3 multiply-add, its mask
            # and XOR (one 3-input logic op), the binary16 addition of the two
            # halves, the conversion to fp32 and the fused multiply-add
            L.append(Launch(f"trellis_b{bits}", "trellis", nb, M=M, N=N, K=K, bits=bits, gs=0,
                            x=x, w=w, s=s, alu_ops=TRELLIS_OPS_PER_VALUE * M * N * K))
        cfg = {"workload": "trellis-mode decode GEMV", "M": M, "K": K, "N": N, "bits": [2, 4]}
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


# Per launch kind: the arrays rotated across weight copies, the per-step
# inputs (copied from the host in the end-to-end timing) and the outputs.
_WEIGHTS = {"qmv": ("w", "s", "b"), "qvm": ("w", "s", "b"), "trellis": ("w", "s"), "gate_up": ("wg", "sg", "bg", "wu", "su", "bu"),
            "silu": ("w", "s", "b"), "gather": ("w", "s", "b"),
            "quantize": ("w",), "dequantize": ("w", "s", "b")}
_INPUTS = {"qmv": ("x",), "qvm": ("x",), "trellis": ("x",), "gate_up": ("x",), "silu": ("gate", "up", "resid"),
           "gather": ("x", "lhs", "rhs"), "quantize": ("w",), "dequantize": ()}


def _outputs(l):
    """(name, shape, numpy dtype) of the arrays a launch writes."""
    if l.kind in ("qmv", "qvm", "trellis"):
        return [("y", (l.M, l.N), np.uint16)]
    if l.kind == "gate_up":
        return [("yg", (l.M, l.N), np.uint16), ("yu", (l.M, l.N), np.uint16)]
    if l.kind == "silu":
        return [("y", (l.M, l.N), np.uint16)]
    if l.kind == "gather":
        return [("y", (l.P, l.N), np.uint16)]
    if l.kind == "quantize":
        G = l.K // l.gs
        return [("q", (l.N, l.K * l.bits // 32), np.uint32), ("s", (l.N, G), np.uint16),
                ("b", (l.N, G), np.uint16)]
    return [("y", (l.N, l.K), np.uint16)]   # dequantize


class _Packed:
    """Device buffers (and pinned host buffers) holding several arrays back to
    back at 16-byte aligned offsets, each reachable as a typed view: a step's
    host copies are then one transfer each way.  `slots` independent copies
    (one per step of a weight rotation) let the copies of one step overlap
    the launches of another."""

    def __init__(self, specs, torch, slots=1):
        self.offsets, off = [], 0
        for _, shape, dt in specs:
            nb = int(np.prod(shape)) * np.dtype(dt).itemsize
            self.offsets.append((off, nb, shape, dt))
            off += (nb + 15) // 16 * 16
        self.nbytes = max(off, 16)
        self.slots = slots
        self.dev = torch.empty((slots, self.nbytes), dtype=torch.uint8, device="cuda")
        self.host = torch.empty((slots, self.nbytes), dtype=torch.uint8).pin_memory()
        self.names = [n for n, _, _ in specs]
        self.torch = torch

    def view(self, i, slot=0):
        torch = self.torch
        off, nb, shape, dt = self.offsets[i]
        t = self.dev[slot % self.slots][off:off + nb]
        td = {np.uint16: torch.bfloat16, np.uint32: torch.int32, np.int32: torch.int32}[dt]
        return t.view(td).view(shape)

    def fill_host(self, arrays):
        h = self.host.numpy()
        for slot in range(self.slots):
            for (off, nb, _, _), a in zip(self.offsets, arrays):
                h[slot, off:off + nb] = np.frombuffer(np.ascontiguousarray(a).tobytes(), np.uint8)


class DeviceWorkload:
    """Device buffers of a workload's launches.  Weights rotate over
    `copies[i]` copies per launch i; each launch's per-step inputs and its
    outputs are views into one packed input and one packed output buffer."""

    def __init__(self, launches, copies, torch, slots=1):
        import affine_group_quantized_b200 as agq
        self.agq, self.torch, self.launches = agq, torch, launches
        self.weights = []
        for l, c in zip(launches, copies):
            self.weights.append([{k: _dev(getattr(l, k), torch) for k in _WEIGHTS[l.kind]}
                                 for _ in range(c)])
        in_specs, out_specs, self.in_idx, self.out_idx = [], [], [], []
        for l in launches:
            idx = {}
            for k in _INPUTS[l.kind]:
                a = np.ascontiguousarray(getattr(l, k))
                idx[k] = len(in_specs)
                in_specs.append((k, a.shape, a.dtype.type))
            self.in_idx.append(idx)
            idx = {}
            for k, shape, dt in _outputs(l):
                idx[k] = len(out_specs)
                out_specs.append((k, shape, dt))
            self.out_idx.append(idx)
        self.slots = slots
        self.inp = _Packed(in_specs, torch, self.slots)
        self.out = _Packed(out_specs, torch, self.slots)
        arrays = [np.ascontiguousarray(getattr(l, k)) for l in launches for k in _INPUTS[l.kind]]
        self.inp.fill_host(arrays)
        self.inp.dev.copy_(self.inp.host)
        self.h2d_bytes = sum(int(np.prod(s)) * np.dtype(d).itemsize for _, s, d in in_specs)
        self.d2h_bytes = sum(int(np.prod(s)) * np.dtype(d).itemsize for _, s, d in out_specs)

    def run(self, i, k, e2e=False):
        """Launch i with weight copy k (modulo its copies); end to end, the
        quantizer reads the matrix just copied in from the host."""
        l, agq = self.launches[i], self.agq
        c = self.weights[i][k % len(self.weights[i])]
        I = {n: self.inp.view(j, k) for n, j in self.in_idx[i].items()}
        O = {n: self.out.view(j, k) for n, j in self.out_idx[i].items()}
        if l.kind == "qmv":
            agq.qmv(I["x"], c["w"], c["s"], c["b"], O["y"], l.M, l.N, l.K, l.bits, l.gs)
        elif l.kind == "trellis":
            agq.qmv_trellis(I["x"], c["w"], c["s"], O["y"], l.M, l.N, l.K, l.bits)
        elif l.kind == "qvm":
            agq.qvm(I["x"], c["w"], c["s"], c["b"], O["y"], l.M, l.K, l.N, l.bits, l.gs)
        elif l.kind == "gate_up":
            agq.qmv_gate_up(I["x"], c["wg"], c["sg"], c["bg"], c["wu"], c["su"], c["bu"],
                            O["yg"], O["yu"], l.M, l.N, l.K, l.bits, l.gs)
        elif l.kind == "silu":
            agq.qmv_silu_gate_resid(I["gate"], I["up"], I["resid"], c["w"], c["s"], c["b"],
                                    O["y"], l.M, l.N, l.K, l.bits, l.gs)
        elif l.kind == "gather":
            agq.gather_qmv(I["x"], c["w"], c["s"], c["b"], I["lhs"], I["rhs"], O["y"],
                           l.P, l.T, l.E, l.N, l.K, l.bits, l.gs, sorted_indices=l.sorted)
        elif l.kind == "quantize":
            src = I["w"] if e2e else c["w"]
            agq.affine_quantize(src, O["q"], O["s"], O["b"], l.N, l.K, l.bits, l.gs)
        else:
            agq.affine_dequantize(c["w"], c["s"], c["b"], O["y"], l.N, l.K, l.bits, l.gs)

    def step(self, k, e2e=False):
        for i in range(len(self.launches)):
            self.run(i, k, e2e)

    def e2e_step(self, k):
        """One step as a user runs it: inputs in from pinned host memory, the
        launches, the outputs back to pinned host memory."""
        slot = k % self.slots
        self.inp.dev[slot].copy_(self.inp.host[slot], non_blocking=True)
        self.step(k, e2e=True)
        self.out.host[slot].copy_(self.out.dev[slot], non_blocking=True)

    def e2e_rotation(self, side):
        """The steps of one weight rotation as a pipelined serving loop runs
        them: every step's inputs go in from pinned host memory and its
        outputs come back, one copy each way per step, on a second stream;
        step k's launches wait for its own inputs only, and its outputs leave
        once its launches are done, while later steps compute."""
        torch = self.torch
        main = torch.cuda.current_stream()
        fork = torch.cuda.Event()
        fork.record(main)
        side.wait_event(fork)
        landed = []
        with torch.cuda.stream(side):
            for k in range(self.slots):
                self.inp.dev[k].copy_(self.inp.host[k], non_blocking=True)
                e = torch.cuda.Event()
                e.record(side)
                landed.append(e)
        done = []
        for k in range(self.slots):
            main.wait_event(landed[k])
            self.step(k, e2e=True)
            e = torch.cuda.Event()
            e.record(main)
            done.append(e)
        with torch.cuda.stream(side):
            for k in range(self.slots):
                side.wait_event(done[k])
                self.out.host[k].copy_(self.out.dev[k], non_blocking=True)
            join = torch.cuda.Event()
            join.record(side)
        main.wait_event(join)


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
GEMV_SOURCES = ("qmv_api.cu", "qmv_decode.cuh", "qmv_device.cuh", "qmv_mma.cuh",
                "qmv_qmm.cu", "qmv_qmm.h", "qmv_quant.cu", "qmv_qvm.cuh", "qmv_stream.cuh",
                "qmv_trellis.cuh")


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


# Operations per trellis value (see the trellis workload) and the ALU peak:
# 148 SMs x 128 FP32 lanes x the maximum SM clock (operations per second).
TRELLIS_OPS_PER_VALUE = 5
ALU_LANES = 148 * 128


def alu_peak():
    """Lane operations per second at the maximum SM clock, in Gop/s."""
    mhz = 1965.0
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            mhz = float(json.load(f).get("sm_max_mhz", mhz))
    return ALU_LANES * mhz * 1e6 / 1e9, "derived (148 SMs x 128 lanes x max SM clock)"


def measured_tensor_peak():
    """Dense bf16 TFLOP/s: the burst figure (a kernel timed alone)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


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


def recorded_ncu_time(kernel_label, workload_name):
    """ncu gpu__time_duration of one launch (cold L2, launches serialised)
    from the committed profile record, while the kernel sources still match."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        e = json.load(f).get(workload_name, {}).get(kernel_label)
    if not e or e.get("source_hash") != source_hash():
        return None
    return e.get("ncu_us")


def _graph(torch, fn):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def _time_graph(torch, g, min_ms):
    """Average ms per replay of CUDA graph g: one warm replay, a one-replay
    estimate, then enough replays for at least `min_ms` of device time."""
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g.replay()
    torch.cuda.synchronize()
    a.record()
    g.replay()
    b.record()
    torch.cuda.synchronize()
    one = max(a.elapsed_time(b), 1e-3)
    reps = int(min(20000, max(3, -(-min_ms // one))))
    a.record()
    for _ in range(reps):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def measure_workload(name, args, torch, world, with_cpu):
    """One workload on this GPU: the step time over exactly `--steps` steps,
    each launch's time back to back and alone, the end-to-end step time and
    the CPU oracle baseline.  Returns the JSON object of the workload."""
    launches, cfg = workload(name)
    step_bytes = sum(l.nbytes for l in launches)
    # Inputs larger than L2: rotate weight copies so that more than twice the
    # L2 capacity streams through between two reads of the same bytes.  Small
    # workloads flush L2 before every step instead (outside the per-launch
    # events, which then give the value).
    flush = step_bytes < 64 * 2**20
    copies = 1 if flush else max(2, -(-2 * L2_BYTES // step_bytes) + 1)
    per = [copies if flush else max(copies, -(-2 * L2_BYTES // l.nbytes) + 1) for l in launches]
    dw = DeviceWorkload(launches, per, torch, slots=copies)
    scrub = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")

    def step(k):
        if flush:
            scrub.fill_(k & 0xFF)
        dw.step(k)

    for k in range(max(args.warmup, copies)):
        step(k)
    torch.cuda.synchronize()
    # the timed steps replay CUDA graphs of the public API calls: graphs[c]
    # is one step on weight copy c, cycle the `copies` steps of a rotation
    graphs = [_graph(torch, lambda c=c: step(c)) for c in range(copies)]
    cycle = _graph(torch, lambda: [step(c) for c in range(copies)])
    for g in graphs:
        g.replay()
    cycle.replay()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    K = args.steps
    stream = torch.cuda.current_stream()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(torch)
    torch.cuda.synchronize()
    with sampler:
        t0.record(stream)
        for _ in range(K // copies):   # exactly K steps: whole rotations ...
            cycle.replay()
        for k in range(K % copies):    # ... then the remaining single steps
            graphs[k].replay()
        t1.record(stream)
        torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), "cuda")
    del graphs, cycle

    # Each launch alone, two ways, each replayed for at least --min-ms:
    #  back to back: a graph of R launches of that kernel rotating its own
    #    weight copies (more than twice L2 between reuses); a launch may be
    #    scheduled while the previous one drains (programmatic dependent
    #    launch), as in a decode loop;
    #  isolated: a graph of R (L2 scrub, launch) pairs, minus a graph of the R
    #    scrubs alone: every launch starts cold, behind a kernel that does not
    #    let it start early.
    chained, isolated = [], []
    for i in range(len(launches)):
        if flush:
            chained.append(None)
        else:
            R = 3 * per[i]
            g = _graph(torch, lambda i=i, R=R: [dw.run(i, r) for r in range(R)])
            chained.append(max_over_ranks(_time_graph(torch, g, args.min_ms) / R, "cuda"))
            del g
        R = 8
        g1 = _graph(torch, lambda i=i: [(scrub.fill_(r), dw.run(i, r)) for r in range(R)])
        g2 = _graph(torch, lambda: [scrub.fill_(r) for r in range(R)])
        d = (_time_graph(torch, g1, args.min_ms) - _time_graph(torch, g2, args.min_ms)) / R
        isolated.append(max_over_ranks(d, "cuda"))
        del g1, g2

    # End to end through the public API: per step, the step's inputs in from
    # pinned host memory (one copy), the launches, the outputs back to pinned
    # host memory (one copy).  A weight rotation's steps run as one CUDA
    # graph in which the copies go over a second stream and overlap the
    # other steps' launches (a pipelined serving loop); the remaining steps
    # run one graph each.
    side = torch.cuda.Stream()
    for k in range(copies):
        dw.e2e_step(k)
    torch.cuda.synchronize()
    erot = _graph(torch, lambda: dw.e2e_rotation(side))
    egraphs = [_graph(torch, lambda c=c: dw.e2e_step(c)) for c in range(copies)]
    erot.replay()
    for g in egraphs:
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(K // copies):
        erot.replay()
    for k in range(K % copies):
        egraphs[k].replay()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), "cuda")
    del egraphs, erot

    peak, peak_kind = measured_peaks()
    out_launch = {}
    basis = "isolated" if flush else "back to back"
    us_of = []
    for l, c, iso in zip(launches, chained, isolated):
        d = iso if c is None else c
        us_of.append(d)
        gbs = l.nbytes / (d * 1e-3) / 1e9
        out_launch[l.label] = {
            "us": round(d * 1e3, 3), "us_back_to_back": None if c is None else round(c * 1e3, 3),
            "us_isolated": round(iso * 1e3, 3), "us_basis": basis, "GB/s": round(gbs, 1),
            "frac_of_measured_peak": round(gbs / peak, 4), "bytes": l.nbytes,
            "ncu_us": recorded_ncu_time(l.label, name)}
    tpeak, tpeak_kind = measured_tensor_peak()
    for l, d in zip(launches, us_of):
        if getattr(l, "flops", None):
            tfs = l.flops / (d * 1e-3) / 1e12
            out_launch[l.label]["TFLOP/s"] = round(tfs, 1)
            out_launch[l.label]["frac_of_measured_tensor_peak"] = round(tfs / tpeak, 4)
    dom = max(range(len(launches)), key=lambda i: us_of[i])
    ach = launches[dom].nbytes / (us_of[dom] * 1e-3) / 1e9
    value = job_gbs(world, step_bytes, K, ms)
    if flush:   # the step region includes the L2 scrub: use kernel time only
        value = world * step_bytes / (sum(isolated) * 1e-3) / 1e9
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms / K, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32 accumulate (bf16 in/out)" if name != "quantize" else "f32 (bf16 in/out)",
        "data": "synthetic",
        "config": dict(cfg, l2=(f"L2 flushed before every step ({2 * L2_BYTES >> 20} MiB "
                                f"write); value from the isolated per-launch times" if flush else
                                f"inputs larger than L2: {copies} rotating weight copies, "
                                f"{step_bytes * copies / 2**20:.0f} MiB between reuse; each "
                                f"launch timed back to back rotates through more than "
                                f"{2 * L2_BYTES >> 20} MiB of its own copies"),
                       parallelism=f"replicas x{world}" if world > 1 else "single GPU",
                       graphs=f"timed steps replayed as CUDA graphs of {copies} steps (one "
                              f"weight rotation); the remainder one step per graph"),
        "roofline": _roofline(launches[dom], us_of[dom], peak, peak_kind, tpeak, tpeak_kind,
                              basis, recorded_traffic(launches[dom].label, name)),
        "per_launch": out_launch,
        "tokens_per_s_equiv": {l.label: round(1e6 / (d * 1e3), 1)
                               for l, d in zip(launches, us_of)},
        "e2e": {"value": round(job_gbs(world, step_bytes, K, e2e_ms), 1),
                "unit": UNIT, "h2d_bytes_per_step": dw.h2d_bytes,
                "d2h_bytes_per_step": dw.d2h_bytes,
                "note": "weights resident in HBM; each step's inputs copied in from "
                        "pinned host memory (one copy) and outputs copied out (one "
                        "copy); the copies of a weight rotation's steps run on a second "
                        "stream and overlap the other steps' launches (a step's "
                        "launches wait for its own inputs, its outputs leave when its "
                        "launches are done); each rotation replayed as one CUDA graph"},
        "gpu_launches": K * len(launches),
        "clocks": sampler.summary(),
    }
    if with_cpu:
        budget = args.cpu_budget if name == args.workload else args.cpu_budget_config
        res["cpu_baseline"] = cpu_baseline(launches, budget_s=budget)
    del dw, scrub
    torch.cuda.empty_cache()
    return res


def _roofline(l, ms, peak, peak_kind, tpeak, tpeak_kind, basis, traffic):
    """The bound of launch l: HBM bytes, or tensor FLOPs where the launch
    carries them and their time at the measured tensor peak is the longer."""
    t_mem = l.nbytes / (peak * 1e9)
    ops = getattr(l, "alu_ops", None)
    if ops:
        apeak, akind = alu_peak()
        if ops / (apeak * 1e9) > t_mem:
            ach = ops / (ms * 1e-3) / 1e9
            return {"bound": "alu", "kernel": l.label, "achieved": round(ach, 1),
                    "peak": round(apeak, 1), "unit": "Gop/s", "frac": round(ach / apeak, 4),
                    "peak_kind": akind, "timing": basis, "traffic": traffic,
                    "algorithmic_ops_per_launch": ops,
                    "algorithmic_bytes_per_launch": l.nbytes}
    flops = getattr(l, "flops", None)
    if flops and flops / (tpeak * 1e12) > t_mem:
        ach = flops / (ms * 1e-3) / 1e12
        return {"bound": "tensor", "kernel": l.label, "achieved": round(ach, 1),
                "peak": tpeak, "unit": "TFLOP/s", "frac": round(ach / tpeak, 4),
                "peak_kind": tpeak_kind, "timing": basis, "traffic": traffic,
                "algorithmic_flops_per_launch": flops,
                "algorithmic_bytes_per_launch": l.nbytes}
    ach = l.nbytes / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "kernel": l.label, "achieved": round(ach, 1), "peak": peak,
            "unit": "GB/s", "frac": round(ach / peak, 4), "peak_kind": peak_kind,
            "timing": basis, "traffic": traffic, "algorithmic_bytes_per_launch": l.nbytes}


def _spawn_replicas(args):
    """`--gpus N` without torchrun: relaunch this command under torchrun, one
    process per GPU, or stop with an error when fewer GPUs are visible."""
    import subprocess
    import torch
    have = torch.cuda.device_count() if torch.cuda.is_available() else 0
    if have < args.gpus:
        sys.stderr.write(f"bench.py: --gpus {args.gpus} needs {args.gpus} visible GPUs, "
                         f"found {have}\n")
        return 2
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={args.gpus}", "--master-addr=127.0.0.1",
           f"--master-port={args.master_port}", os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


ALL_WORKLOADS = ("decode_sweep", "qmv_small", "ffn_int8", "batched", "prefill", "moe_gather",
                 "qvm", "trellis", "quantize")


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
    with_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    out = measure_workload(args.workload, args, torch, world, with_cpu)
    if args.configs == "all":
        out["per_config"] = {}
        for name in ALL_WORKLOADS:
            if name != args.workload:
                out["per_config"][name] = measure_workload(name, args, torch, world, with_cpu)
    out["source_hash"] = source_hash()
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
        oracle.silu_gate_resid(l.gate, l.up, l.resid, l.w, l.s, l.b, l.M, l.N, l.K, l.bits,
                               l.gs, rows=rows, nthreads=nthreads)
    elif l.kind == "qvm":
        oracle.qvm(l.x, l.w, l.s, l.b, l.M, l.K, l.N, l.bits, l.gs)
    elif l.kind == "trellis":
        n = l.N if rows is None else len(rows)
        oracle.qmv_trellis(l.x, l.w[:n], l.s, l.M, n, l.K, l.bits)
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
    if l.kind in ("gather", "qvm"):
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
                      f"every launch of one step (gather and qvm: whole), plain-C "
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


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode_sweep", choices=list(ALL_WORKLOADS))
    ap.add_argument("--configs", default="all", choices=["all", "none"],
                    help="also measure every other workload (per_config)")
    ap.add_argument("--min-ms", type=float, default=100.0,
                    help="device time each per-launch timing graph is replayed for")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--cpu-budget-config", type=float, default=6.0)
    ap.add_argument("--master-port", type=int, default=29533)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    world = os.environ.get("WORLD_SIZE")
    if world is not None and int(world) != args.gpus:
        sys.stderr.write(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}\n")
        return 2
    if args.impl == "reference":
        run_reference(args)
        return 0
    if args.gpus > 1 and world is None:
        return _spawn_replicas(args)
    run_ours(args)
    return 0


if __name__ == "__main__":
    sys.exit(main())
