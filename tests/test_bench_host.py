"""Host-side pieces of the benchmark, on CPU: the algorithmic byte model, the
traffic lookup keyed by the kernel sources, and the argument defaults."""
import json
import os
import shutil

import bench
import workloads as W


def test_algorithmic_bytes_of_the_fp8_workloads():
    w = W.WORKLOADS["prefill_skew"]                       # FP8 codes + fp32 scales
    Na, T, H = w.n_assign, w.T, w.H
    ab = bench.algorithmic_bytes(w)
    assert ab["dispatch"] == T * H * 2 + Na * H + Na * (H // 128) * 4 + 4 * Na
    assert ab["combine"] == Na * H * 2 + T * H * 2 + 8 * Na
    d = W.WORKLOADS["decode"]                             # FP8 codes + UE8M0 bytes
    ab = bench.algorithmic_bytes(d)
    assert ab["dispatch"] == d.T * d.H * 2 + d.n_assign * d.H + d.n_assign * (d.H // 128) + 4 * d.n_assign
    s = W.WORKLOADS["streaming"]
    assert bench.algorithmic_bytes(s)["consumer"] == 2 * s.n_assign * s.H * 2


def test_traffic_is_reported_only_for_the_profiled_sources(tmp_path, monkeypatch):
    root = tmp_path / "repo"
    csrc = root / "combine_route_layout_02_b200" / "csrc"
    shutil.copytree(os.path.join(bench.ROOT, "combine_route_layout_02_b200", "csrc"), csrc,
                    ignore=shutil.ignore_patterns("*.o", "*.so"))
    (root / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(root))
    h = bench.kernel_source_hash("dispatch")
    table = {"train8k": {"dispatch": {"bytes_per_launch": 123.0, "source_hash": h}}}
    (root / "profiles" / "dram_traffic.json").write_text(json.dumps(table))
    assert bench.profiled_traffic("train8k", "dispatch") == 123.0
    assert bench.profiled_traffic("train8k", "combine") is None
    assert bench.profiled_traffic("decode", "dispatch") is None
    # an unrelated file changing keeps the figure; the kernel's own file changing drops it
    (csrc / "scatter.cu").write_text((csrc / "scatter.cu").read_text() + "\n// edit\n")
    assert bench.profiled_traffic("train8k", "dispatch") == 123.0
    (csrc / "dispatch.cu").write_text((csrc / "dispatch.cu").read_text() + "\n// edit\n")
    assert bench.profiled_traffic("train8k", "dispatch") is None


def test_argument_defaults():
    a = bench.parse_args([])
    assert a.extras.split(",") == ["borrowed", "backward", "gate", "scatter", "ep", "budget", "overlap"]
    assert not a.no_graph and not a.no_extras and a.gate_ctas == 0 and a.consumer_ctas == 64


def test_reference_arm_line_on_the_host_cores():
    """`--impl reference` times the oracle on the host cores (no GPU): rank 0
    prints the contract's line with the cpu_baseline description and a zero-copy
    e2e; any other rank does no work."""
    args = bench.parse_args(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "1"])
    assert bench.run_reference(args, rank=1) is None
    res = bench.run_reference(args, rank=0)
    assert res["impl"] == "reference" and res["metric"] == bench.METRIC and res["unit"] == "tokens/s"
    assert res["value"] > 0 and res["ms_per_step"] > 0 and res["higher_is_better"] is True
    assert (res["steps"], res["warmup"], res["n_gpus"]) == (2, 1, 1)
    cb = res["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == res["value"] and cb["sample"]
    assert res["e2e"] == {"value": res["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                          "d2h_bytes_per_step": 0}
    assert res["gpu_launches"] == 0 and res["config"]["workload"] == "tiny"
    json.dumps(res)                                       # one JSON line


def test_cpu_baseline_reports_the_oracle_on_a_bounded_sample():
    """The cpu_baseline object of our arm's line: the oracle on one core and on
    every core, the faster reported, both kept; bounded by the budget."""
    import time
    w = W.WORKLOADS["tiny"]
    d = W.make_inputs(w)
    t0 = time.perf_counter()
    cb = bench.cpu_baseline(w, d, 0.5)
    assert time.perf_counter() - t0 < 60
    assert cb["kind"] == "oracle" and cb["unit"] == "tokens/s" and cb["value"] > 0 and cb["sample"]
    assert cb["single_core"]["cores"] == 1 and cb["single_core"]["value"] > 0
    assert cb["value"] == max(cb["single_core"]["value"], cb["all_cores"].get("value", 0))
    assert cb["cores"] == (cb["all_cores"]["cores"] if cb["value"] == cb["all_cores"].get("value") else 1)


class _FakeNvml:
    """Stands in for pynvml: read-only clock queries on a fake device."""
    NVML_CLOCK_SM = 1
    nvmlClocksEventReasonHwSlowdown = 0x8
    nvmlClocksEventReasonHwThermalSlowdown = 0x40
    nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nvmlClocksEventReasonSwPowerCap = 0x4
    nvmlClocksEventReasonHwPowerBrakeSlowdown = 0x80

    def __init__(self, clocks, reasons, fail_init=False):
        self.clocks, self.reasons, self.fail_init = list(clocks), reasons, fail_init
        self.opened = None

    def nvmlInit(self):
        if self.fail_init:
            raise RuntimeError("no driver")

    def nvmlDeviceGetHandleByIndex(self, i):
        self.opened = i
        return ("dev", i)

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        return self.clocks.pop(0) if len(self.clocks) > 1 else self.clocks[0]

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.reasons


def test_clock_sampler_reads_clocks_and_reasons_from_nvml(monkeypatch):
    import sys
    import time
    fake = _FakeNvml([1965, 1890, 1965, 1965], _FakeNvml.nvmlClocksEventReasonSwPowerCap)
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "3,5")
    with bench.ClockSampler(1, period_s=0.001) as s:
        time.sleep(0.05)
    got = s.summary()
    assert fake.opened == 5                               # the physical index behind device 1
    assert got["sm_max_mhz"] == 1965 and got["sm_mhz"] == 1965 and got["samples"] >= 4
    assert got["reasons"] == ["sw_power_cap"] and got["source"] == "nvml"
    fake.reasons = _FakeNvml.nvmlClocksEventReasonHwThermalSlowdown | _FakeNvml.nvmlClocksEventReasonHwSlowdown
    with bench.ClockSampler(0, period_s=0.001) as s:
        time.sleep(0.02)
    assert s.summary()["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]


def test_clock_sampler_without_nvml_reports_it(monkeypatch):
    import sys
    monkeypatch.setitem(sys.modules, "pynvml", _FakeNvml([1965], 0, fail_init=True))
    with bench.ClockSampler(0) as s:
        pass
    got = s.summary()
    assert got["sm_mhz"] is None and got["source"] == "nvml unavailable" and got["samples"] == 0
