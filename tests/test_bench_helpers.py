"""Host-side helpers of bench.py (CPU): the DRAM-traffic lookup in a committed
ncu record, which must answer only for the kernel source it was taken on,
the name of the product kernel the library's switches select, and the
compact summary at the end of the line."""
import json
import os

import bench


def _record(tmp_path, rec):
    d = tmp_path / "profiles"
    d.mkdir()
    (d / "t.json").write_text(json.dumps(rec))
    return str(tmp_path)


def test_traffic_only_for_the_profiled_source(tmp_path, monkeypatch):
    root = _record(tmp_path, {"kernel_source_hash": "abc123", "dram_bytes_per_full_launch": 1000})
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench.profiled_traffic("abc123", "t.json") == 1000.0
    assert bench.profiled_traffic("def456", "t.json") is None      # kernel changed since
    assert bench.profiled_traffic("abc123", "missing.json") is None


def test_traffic_needs_both_keys(tmp_path, monkeypatch):
    root = _record(tmp_path, {"kernel_source_hash": "abc123"})
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench.profiled_traffic("abc123", "t.json") is None


def test_committed_traffic_record_parses():
    """The committed record names a hash and a byte count; whether the hash
    is the current one decides only whether the bench reports it."""
    path = os.path.join(bench.ROOT, "profiles", "kq_quantize_stress_traffic.json")
    rec = json.load(open(path))
    assert bench.profiled_traffic(rec["kernel_source_hash"], "kq_quantize_stress_traffic.json") > 4e8
    assert "ncu" in rec["command"]


def test_compact_summary_is_short_and_complete():
    cfgs = list(bench.CONFIG_LABELS)
    row = lambda c: dict({"config": c}, **{k: {"frac": 0.123456, "us": 12.3456}
                                           for k in bench.SUMMARY_COLS})
    variants = {"per_config": {"rows": [row(c) for c in cfgs]},
                "layers": {"rows": [{"layer": l[0], "gemm_frac": 0.7654321,
                                     "layer_speedup_over_bf16": 2.3456}
                                    for l in bench.LAYER_SHAPES]}}
    summ = bench.compact_summary(variants)
    assert set(summ["frac_of_measured_hbm"]) == set(bench.CONFIG_LABELS.values())
    assert summ["frac_of_measured_hbm"]["C4"] == [0.123] * len(bench.SUMMARY_COLS)
    assert len(json.dumps(summ)) < 1200


def test_gemm_kernel_name_follows_the_library_switches(monkeypatch):
    for var in ("KQ_GEMM_PAIR", "KQ_GEMM_PERSISTENT"):
        monkeypatch.delenv(var, raising=False)
    assert bench.gemm_kernel_name().startswith("gemm_mxf4_persistent<")
    monkeypatch.setenv("KQ_GEMM_PAIR", "1")
    assert bench.gemm_kernel_name().startswith("gemm_mxf4_pair<")
    monkeypatch.setenv("KQ_GEMM_PAIR", "00")                   # atoi("00") == 0
    assert bench.gemm_kernel_name().startswith("gemm_mxf4_persistent<")
    monkeypatch.setenv("KQ_GEMM_PERSISTENT", "0")
    assert bench.gemm_kernel_name().startswith("gemm_mxf4_kernel<")
    monkeypatch.setenv("KQ_GEMM_PERSISTENT", "x")              # atoi("x") == 0
    assert bench.gemm_kernel_name().startswith("gemm_mxf4_kernel<")


class _FakeNvml:
    """Stands in for pynvml: each query takes 2 ms (longer than a short timed
    region) and reports a fixed clock with the power-cap reason set."""
    NVML_CLOCK_SM = 0

    def nvmlInit(self):
        pass

    def nvmlDeviceGetHandleByIndex(self, i):
        return i

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        import time
        time.sleep(0.002)
        return 1890

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return 0x4


def test_clock_sampler_counts_polls_overlapping_a_short_region(monkeypatch):
    import sys
    import time
    monkeypatch.setitem(sys.modules, "pynvml", _FakeNvml())
    monkeypatch.delenv("CUDA_VISIBLE_DEVICES", raising=False)
    s = bench.ClockSampler(0)
    time.sleep(0.01)
    s.start()
    time.sleep(0.001)                  # a region shorter than one poll
    rec = s.stop()
    assert rec["source"] == "nvml"
    assert rec["samples"] >= 1 and rec["sm_mhz"] == 1890 and rec["sm_max_mhz"] == 1965
    assert rec["reasons"] == ["sw_power_cap"]
    assert rec["poll_ms"] >= 1.0 and 0.5 <= rec["region_ms"] < 50
