"""Host logic of bench.py on CPU: the per-mode position and byte counts, the
traffic record's gating, the per-call percentiles, the clock-sample parser, the workload selection,
and the JSON line of the CPU-only reference arm."""
import datetime
import time
import json
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_positions_per_mode():
    assert bench.positions(dict(mode="stochastic", B=3, k=4)) == 15
    assert bench.positions(dict(mode="greedy", B=2, k=0)) == 2
    assert bench.positions(dict(mode="multi", B=2, G=8, k=4)) == 80
    assert bench.positions(dict(mode="tree", B=5, N=26)) == 130
    assert bench.positions(dict(mode="tree_stochastic", B=5, N=26)) == 130


def test_full_read_bytes_per_mode():
    B, k, V = 2, 3, 10
    g = dict(mode="greedy", B=B, k=k, V=V, t_dtype="bf16")
    assert bench.full_bytes(g) == B * (k + 1) * V * 2 + 4 * B * k + 4 * B * (k + 2)
    m = dict(mode="multi", B=B, G=3, k=k, V=V, t_dtype="f32")
    assert bench.full_bytes(m) == B * 3 * (k + 1) * V * 4 + 4 * B * 3 * k + 4 * B * (k + 3)
    s = dict(mode="stochastic", B=B, k=k, V=V, t_dtype="bf16", d_dtype="f32")
    assert bench.full_bytes(s) == \
        B * (k + 1) * V * 2 + B * k * V * 4 + 4 * B * k + 4 * B * (k + 2)
    for mode in ("tree", "tree_stochastic"):
        t = dict(mode=mode, B=B, N=7, V=V, t_dtype="bf16")
        assert bench.full_bytes(t) == B * 7 * V * 2 + 8 * B * 7 + 4 * B + 8 * B * 7
    # rows form: each distinct row once
    row_of = np.array([[[0, 1], [0, 2]], [[0, 1], [0, 1]]], np.int32)  # B=2, G=2, k+1=2
    r = dict(mode="multi_rows", B=2, G=2, k=1, V=V, t_dtype="bf16", row_of=row_of)
    assert bench.full_bytes(r) == \
        (3 + 2) * V * 2 + 4 * 2 * 2 * 2 + 4 * 2 * 2 * 1 + 4 * 2 * (1 + 3)


def test_needed_bytes_follow_the_oracle_outcome():
    B, k, V = 3, 3, 10
    s = dict(mode="stochastic", B=B, k=k, V=V, t_dtype="bf16", d_dtype="f32")
    # n = 0: pair 0; n = 2: pairs 0..2; n = k: pairs 0..k-1 and target row k
    o = {"accepted_len": np.array([0, 2, k])}
    assert bench.needed_bytes(s, o) == \
        (1 + 3 + 3) * V * (2 + 4) + 1 * V * 2 + 4 * B * k + 4 * B * (k + 2)
    g = dict(mode="greedy", B=B, k=k, V=V, t_dtype="bf16")
    assert bench.needed_bytes(g, o) == (1 + 3 + 4) * V * 2 + 4 * B * k + 4 * B * (k + 2)
    m = dict(mode="multi", B=1, G=2, k=k, V=V, t_dtype="bf16")
    o = {"branch_len": np.array([[1, 3]])}
    assert bench.needed_bytes(m, o) == (2 + 4) * V * 2 + 4 * 2 * k + 4 * (k + 3)
    assert bench.needed_bytes(g, None) is None
    full = bench.full_bytes(s)
    assert bench.needed_bytes(s, {"accepted_len": np.full(B, k)}) == full


def test_parity_record_counts_mismatches_and_near_ties():
    w = dict(mode="stochastic", B=3, k=2)
    o = {"accepted_len": np.array([0, 2, 1]), "out_tokens": np.array([[5, -1, -1],
                                                                     [1, 2, 7], [3, 4, -1]]),
         "margins": np.array([[0.5, 1e-7], [0.3, 0.2], [2e-6, 0.4]]),
         "gaps": np.array([0.1, 3e-6, 0.2])}
    gpu = {"accepted_len": np.array([0, 2, 0]),
           "out_tokens": np.array([[5, -1, -1], [1, 2, 8], [9, -1, -1]])}
    rec = bench.parity_record(w, gpu, o)
    # sequence 0: margin past n is not examined, no near tie; 1: gap near tie;
    # 2: margin near tie at position 0
    assert rec["sequences"] == 3 and rec["mismatches"] == 2
    assert rec["near_ties"] == 2 and rec["mismatches_outside_near_ties"] == 0
    g = dict(mode="greedy", B=2, k=1)
    rec = bench.parity_record(g, {"accepted_len": np.array([1, 0]),
                                  "out_tokens": np.array([[3, 4], [6, -1]])},
                              {"accepted_len": np.array([1, 0]),
                               "out_tokens": np.array([[3, 4], [5, -1]])})
    assert rec == {"sequences": 2, "mismatches": 1, "rule": "bit-exact"}


def test_traffic_record_applies_only_to_its_kernel_sources_and_workload(tmp_path, monkeypatch):
    rec = {"kernel_source_sha256": bench.kernel_source_hash(), "dram_bytes_per_launch": 123.0}
    f = tmp_path / "traffic.json"
    f.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.recorded_traffic("stoch_b256_k8_v128256", False) == 123.0
    assert bench.recorded_traffic("stoch_b256_k8_v128256", True) is None
    assert bench.recorded_traffic("stoch_b64_k4_v128256", False) is None
    rec["kernel_source_sha256"] = "0" * 64
    f.write_text(json.dumps(rec))
    assert bench.recorded_traffic("stoch_b256_k8_v128256", False) is None
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "missing.json"))
    assert bench.recorded_traffic("stoch_b256_k8_v128256", False) is None


def test_committed_traffic_record_names_its_sources():
    # the bench uses the record only while these sources hash to its value
    # (otherwise it reports traffic null: see the gating test above)
    with open(bench.TRAFFIC_FILE) as f:
        rec = json.load(f)
    assert len(rec["kernel_source_sha256"]) == 64
    assert rec["kernel_sources"] == list(bench.DOMINANT_SOURCES)
    assert rec["dram_bytes_per_launch"] > 0


class _Done:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0

    def kill(self):
        pass

    def join(self, timeout=None):
        pass


def test_call_spread_percentiles():
    # 0.001 .. 0.101 ms: percentiles of an evenly spaced set are known exactly
    xs = [i * 1e-3 for i in range(1, 102)]
    np.random.default_rng(0).shuffle(xs)
    sp = bench.call_spread(xs)
    assert sp["samples"] == 101
    assert sp["median"] == pytest.approx(51.0)
    assert sp["p10"] == pytest.approx(11.0)
    assert sp["p90"] == pytest.approx(91.0)
    # agrees with numpy's linear interpolation on an uneven set
    ys = list(np.random.default_rng(1).gamma(2.0, 0.01, size=200))
    sp = bench.call_spread(ys)
    for key, f in (("p10", 10), ("median", 50), ("p90", 90)):
        assert sp[key] == pytest.approx(round(np.percentile(ys, f) * 1e3, 2), abs=0.006)
    assert bench.call_spread([]) == {}


def test_clock_sampler_keeps_samples_inside_the_window():
    cs = object.__new__(bench.ClockSampler)
    cs.proc, cs.thread = _Done(), _Done()
    t0 = datetime.datetime(2026, 1, 2, 3, 4, 5)

    def line(dt, mhz, reasons):
        ts = (t0 + datetime.timedelta(seconds=dt)).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        flags = ["Active" if r in reasons else "Not Active" for r in bench.ClockSampler.REASONS]
        return ", ".join([ts, str(mhz), "1965", "700.0", "0x0"] + flags)

    cs.lines = [line(-1.0, 1000, {"hw_slowdown"}),  # before the window: ignored
                line(0.2, 1965, set()), line(0.4, 1950, {"sw_power_cap"}),
                line(0.6, 1965, set()), "garbage", line(5.0, 500, {"hw_thermal_slowdown"})]
    out = cs.stop(t0.timestamp(), t0.timestamp() + 1.0)
    assert out == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                   "samples": 3, "window": "timed region"}
    # a region shorter than the sampling period: the neighbouring samples stand in
    out = cs.summarise(t0.timestamp() + 0.25, t0.timestamp() + 0.3)
    assert out["samples"] == 2 and out["sm_mhz"] == 1957.5
    assert out["window"].startswith("no sample inside")


class _FakeNvml:
    """The NVML calls the fast sampler makes, answering from a script of
    (clock, reason bits) readings."""
    NVML_CLOCK_SM = 1
    nvmlClocksEventReasonHwSlowdown = 0x8
    nvmlClocksEventReasonHwThermalSlowdown = 0x40
    nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nvmlClocksEventReasonSwPowerCap = 0x4

    def __init__(self, script):
        self.script = list(script)

    def nvmlInit(self):
        pass

    def nvmlDeviceGetHandleByUUID(self, uuid):
        assert uuid.startswith("GPU-")
        return "h"

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        if not self.script:
            raise RuntimeError("done")  # ends the sampling thread
        return self.script[0][0]

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.script.pop(0)[1]


def test_nvml_sampler_reads_clocks_and_reasons(monkeypatch):
    fake = _FakeNvml([(1965, 0), (1950, 0x4), (1965, 0x1), (1900, 0x4 | 0x8)])
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    t0 = time.time()
    s = bench.NvmlSampler("GPU-0000")
    assert s.ok
    s.thread.join(timeout=5)
    out = s.stop(t0 - 1.0, time.time() + 1.0)
    # bit 0x1 (idle) is not a reason the record keeps
    assert out["samples"] == 4 and out["sm_mhz"] == 1957.5 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["hw_slowdown", "sw_power_cap"]
    assert s.stop(t0 - 10.0, t0 - 9.0) is None  # no sample inside: the caller falls back


def test_nvml_sampler_absent(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", None)  # import fails
    s = bench.NvmlSampler("GPU-0000")
    assert not s.ok and s.stop(0.0, 1.0) is None


def test_select_workloads(monkeypatch):
    monkeypatch.setattr(bench, "STEP", list(bench.STEP))
    monkeypatch.setattr(bench, "DOMINANT", bench.DOMINANT)
    with pytest.raises(SystemExit):
        bench.select_workloads("no_such_workload")
    bench.select_workloads("tree_stoch_b64_n26_v128256")
    assert bench.STEP == ["tree_stoch_b64_n26_v128256"]
    assert bench.DOMINANT == "tree_stoch_b64_n26_v128256"


def test_reference_arm_prints_one_json_line():
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--only", "stoch_b1_k4_v32000_f32", "--steps", "2", "--warmup", "3"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"].endswith("stoch_b1_k4_v32000_f32")
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
