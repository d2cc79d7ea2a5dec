"""Host-side logic of bench.py, checked on the CPU: the algorithmic byte
counts behind every GB/s figure, the clock sampler's decoding of NVML's
clock-event reasons (against a fake NVML), and the lookups of the measured
peak and of the recorded DRAM traffic."""
import json
import os
import sys
import time
import types

import numpy as np
import pytest

import bench


def _arrays_bytes(*arrays):
    return sum(np.asarray(a).nbytes for a in arrays)


@pytest.mark.parametrize("name", ["qmv_small", "decode_sweep"])
def test_qmv_bytes_are_the_arrays_read_and_written(name):
    # read: packed codes, scales, biases, activations; written: bf16 y
    launches, _ = bench.workload(name)
    for l in launches:
        assert l.nbytes == _arrays_bytes(l.w, l.s, l.b, l.x) + 2 * l.M * l.N, l.label


def test_ffn_bytes_are_the_arrays_read_and_written():
    gate_up, silu = bench.workload("ffn_int8")[0]
    # gate/up: two weight sets, one x; two bf16 outputs of N
    assert gate_up.nbytes == (_arrays_bytes(gate_up.wg, gate_up.sg, gate_up.bg,
                                            gate_up.wu, gate_up.su, gate_up.bu,
                                            gate_up.x) + 2 * 2 * gate_up.N)
    # SiLU down: its weights and residual, the gate and up vectors (bf16 of
    # its K) and the bf16 output of its N
    assert silu.nbytes == (_arrays_bytes(silu.w, silu.s, silu.b, silu.resid) +
                           2 * 2 * silu.K + 2 * silu.N)


def test_quantize_bytes_are_the_matrix_and_its_packed_form():
    quant, dequant = bench.workload("quantize")[0]
    bf16_matrix = 2 * quant.N * quant.K
    for l in (quant, dequant):
        # one side is the bf16 matrix, the other the codes, scales and biases
        assert l.nbytes == bf16_matrix + _arrays_bytes(dequant.w, dequant.s, dequant.b)
    assert quant.w.nbytes == bf16_matrix
    assert bench._threads_used([quant, dequant], 8) == 1


def test_gather_bytes_count_touched_experts_only():
    launches, cfg = bench.workload("moe_gather")
    for l in launches:
        touched = np.unique(l.rhs)
        assert len(touched) == cfg["touched_experts"]
        per_w = l.w.nbytes // l.E
        per_sb = l.s.nbytes // l.E
        weights = len(touched) * (per_w + 2 * per_sb)
        index = _arrays_bytes(l.lhs, l.rhs)
        assert l.nbytes == weights + l.x.nbytes + 2 * l.P * l.N + index, l.label


class _FakeNvml(types.ModuleType):
    """NVML stand-in: fixed clock readings and event-reason masks."""

    NVML_CLOCK_SM = 1

    def __init__(self, clocks, masks, fail_init=False):
        super().__init__("pynvml")
        self._clocks, self._masks, self._fail = list(clocks), list(masks), fail_init
        self.calls = 0

    def nvmlInit(self):
        if self._fail:
            raise RuntimeError("NVML Shared Library Not Found")

    def nvmlDeviceGetHandleByUUID(self, uuid):
        assert uuid.startswith("GPU-")
        return "handle"

    def nvmlDeviceGetMaxClockInfo(self, h, clock):
        assert h == "handle" and clock == self.NVML_CLOCK_SM
        return 1965

    def nvmlDeviceGetClockInfo(self, h, clock):
        i = min(self.calls, len(self._clocks) - 1)
        self.calls += 1
        return self._clocks[i]

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self._masks[min(self.calls - 1, len(self._masks) - 1)]


def _fake_torch():
    props = types.SimpleNamespace(uuid="0d4e5c6a-0000-0000-0000-000000000001")
    cuda = types.SimpleNamespace(current_device=lambda: 0,
                                 get_device_properties=lambda i: props)
    return types.SimpleNamespace(cuda=cuda)


def test_clock_reason_bits_are_nvml_constants():
    nv = pytest.importorskip("pynvml")
    names = {"gpu_idle": "GpuIdle", "applications_clocks_setting": "ApplicationsClocksSetting",
             "sw_power_cap": "SwPowerCap", "hw_slowdown": "HwSlowdown",
             "sync_boost": "SyncBoost", "sw_thermal_slowdown": "SwThermalSlowdown",
             "hw_thermal_slowdown": "HwThermalSlowdown",
             "hw_power_brake_slowdown": "HwPowerBrakeSlowdown",
             "display_clock_setting": "DisplayClockSetting"}
    for bit, name in bench.ClockSampler._REASONS.items():
        assert getattr(nv, "nvmlClocksEventReason" + names[name]) == bit, name


def test_clock_sampler_decodes_reasons_and_takes_the_median(monkeypatch):
    fake = _FakeNvml(clocks=[1965, 1950, 1965, 1300, 1965],
                     masks=[0x1, 0x4, 0x4 | 0x40, 0x0, 0x20])
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    cs = bench.ClockSampler(_fake_torch())
    assert cs.ok
    deadline = time.monotonic() + 10.0
    with cs:
        while fake.calls < 8 and time.monotonic() < deadline:
            time.sleep(0.001)
    s = cs.summary()
    assert s["sm_max_mhz"] == 1965
    assert s["sm_mhz"] == 1965          # the median, not the mean or the minimum
    # gpu_idle is dropped; every other bit seen in any sample is reported
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap", "sw_thermal_slowdown"]
    assert s["samples"] == len(cs.samples) >= 8


def test_clock_sampler_without_nvml_reports_the_error(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", _FakeNvml([], [], fail_init=True))
    cs = bench.ClockSampler(_fake_torch())
    with cs:
        pass
    s = cs.summary()
    assert not cs.ok and s["sm_mhz"] is None and s["reasons"] == []
    assert "NVML Shared Library Not Found" in s["error"]


def test_measured_peak_and_fallback(monkeypatch, tmp_path):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_peaks() == (6650.0, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6537.5}))
    assert bench.measured_peaks() == (6537.5, "measured")


def test_recorded_traffic_only_for_the_captured_source(monkeypatch, tmp_path):
    csrc = tmp_path / "affine_group_quantized_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "qmv_stream.cuh").write_text("kernel v1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("qmv_b4", "decode_sweep") is None
    h = bench.source_hash()
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"decode_sweep": {"qmv_b4": {"source_hash": h,
                                     "dram_bytes_per_launch": 33067008}}}))
    assert bench.recorded_traffic("qmv_b4", "decode_sweep") == 33067008
    assert bench.recorded_traffic("qmv_b8", "decode_sweep") is None
    (csrc / "notes.txt").write_text("not a kernel source\n")
    assert bench.source_hash() == h
    assert bench.recorded_traffic("qmv_b4", "decode_sweep") == 33067008
    (csrc / "qmv_stream.cuh").write_text("kernel v2\n")     # source changed since
    assert bench.source_hash() != h
    assert bench.recorded_traffic("qmv_b4", "decode_sweep") is None


def test_committed_traffic_names_known_launches():
    # every recorded entry belongs to a launch label of the workload it is
    # filed under, so the bench's lookup by (label, workload) can find it
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        d = json.load(f)
    recorded = {k: v for k, v in d.items() if not k.startswith("_")}
    assert recorded
    for name, entries in recorded.items():
        if name == "batched":   # its launch labels, without building its inputs
            labels = {f"qmv_M{M}_gs{gs}" for M in (1, 2, 4, 8) for gs in (32, 128)}
        else:
            labels = {l.label for l in bench.workload(name)[0]}
        assert set(entries) <= labels, name
        for e in entries.values():
            assert e["dram_bytes_per_launch"] > 0 and len(e["source_hash"]) == 16


def test_gpus_flag_without_torchrun_needs_that_many_gpus(monkeypatch, capsys):
    # `--gpus 2` outside torchrun relaunches under torchrun only when two GPUs
    # are visible; on a box with fewer it stops with an error, never printing
    # a one-GPU line
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    import torch
    if torch.cuda.is_available() and torch.cuda.device_count() >= 2:
        pytest.skip("two GPUs visible: the flag would launch the replicas")
    assert bench.main(["--gpus", "2", "--steps", "3"]) == 2
    err = capsys.readouterr().err
    assert "--gpus 2 needs 2 visible GPUs" in err


def test_gpus_flag_must_match_the_launcher(monkeypatch, capsys):
    monkeypatch.setenv("WORLD_SIZE", "4")
    assert bench.main(["--gpus", "2"]) == 2
    assert "WORLD_SIZE=4" in capsys.readouterr().err


@pytest.mark.parametrize("name", bench.ALL_WORKLOADS)
def test_every_workload_has_inputs_outputs_and_weights(name):
    # the packed per-step input and output buffers cover every array the
    # launches read per step and write
    launches, _ = bench.workload(name)
    for l in launches:
        for k in bench._WEIGHTS[l.kind] + bench._INPUTS[l.kind]:
            assert getattr(l, k) is not None, (l.label, k)
        outs = bench._outputs(l)
        assert outs and all(int(np.prod(s)) > 0 for _, s, _ in outs)


def test_qvm_workload_arrays_have_the_launch_shapes():
    (l,), _ = bench.workload("qvm")
    assert l.x.shape == (l.M, l.K)
    assert l.w.shape == (l.K, l.N * l.bits // 32) and l.s.shape == (l.K, l.N // l.gs)
    assert l.nbytes == _arrays_bytes(l.w, l.s, l.b, l.x) + 2 * l.M * l.N


def test_roofline_takes_the_longer_of_memory_and_tensor_time():
    # a launch whose FLOPs at the tensor peak take longer than its bytes at
    # the HBM peak is tensor bound; otherwise memory bound
    L = bench.Launch("t", "qmv", nbytes=1_000_000, flops=2 * 128 * 28672 * 8192)
    r = bench._roofline(L, 0.1, 6537.0, "measured", 1627.7, "measured", "b", None)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert abs(r["achieved"] - L.flops / 1e-4 / 1e12) < 0.1
    L2 = bench.Launch("m", "qmv", nbytes=147_000_000, flops=2 * 32 * 28672 * 8192)
    r2 = bench._roofline(L2, 0.05, 6537.0, "measured", 1627.7, "measured", "b", None)
    assert r2["bound"] == "hbm" and r2["unit"] == "GB/s"


def test_prefill_launches_carry_their_flops():
    launches, cfg = bench.workload("prefill")
    for l in launches:
        assert l.flops == 2 * l.M * l.N * l.K
        assert l.nbytes == _arrays_bytes(l.w, l.s, l.b, l.x) + 2 * l.M * l.N


def test_trellis_roofline_is_alu_bound():
    # 5 operations per value over 58.7M values at the derived ALU peak take
    # longer than the launch's 29 MB at the HBM peak
    launches, _ = bench.workload("trellis")
    for l in launches:
        assert l.alu_ops == bench.TRELLIS_OPS_PER_VALUE * l.M * l.N * l.K
        r = bench._roofline(l, 0.036, 6537.0, "measured", 1627.7, "measured", "b", None)
        assert r["bound"] == "alu" and r["unit"] == "Gop/s"
        assert abs(r["peak"] - bench.alu_peak()[0]) < 0.1
        assert abs(r["achieved"] * 0.036e-3 * 1e9 - l.alu_ops) < 1e-3 * l.alu_ops
