"""Host-side logic of bench.py (CPU only): the clock record taken during the
timed region, the roofline denominators, and the DRAM-traffic figure that is
read only while the profiled kernel source is unchanged."""
import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _line(sm, smax, hw="Not Active", thermal="Not Active", swpc="Not Active"):
    return (f"2026/01/01 00:00:00.000, 0, {sm}, {smax}, 700.0, 0x0, {hw}, {thermal}, "
            f"Not Active, {swpc}")


def test_clock_summary_keeps_the_timed_window_and_reasons():
    s = bench.ClockSampler(0)
    s.lines = [(1.0, _line(900, 1965)),                       # before the window
               (2.0, _line(1965, 1965)), (2.5, _line(1950, 1965, swpc="Active")),
               (3.0, _line(1965, 1965, hw="Active")),
               (9.0, _line(500, 1965, thermal="Active"))]     # after the window
    s.mark(1.5, 3.5)
    d = s.summary()
    assert d["samples"] == 3
    assert d["sm_mhz"] == 1965.0 and d["sm_max_mhz"] == 1965.0
    assert set(d["reasons"]) == {"hw_slowdown", "sw_power_cap"}


def test_clock_summary_without_samples():
    s = bench.ClockSampler(0)
    s.mark(0.0, 1.0)
    assert s.summary()["samples"] == 0


def test_peaks_are_measured_or_the_stated_fallback():
    hbm, bf16, kind = bench.peaks()
    if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")):
        assert kind == "measured" and hbm > 1000 and bf16 > 100
    else:
        assert (hbm, bf16, kind) == (bench.FALLBACK_HBM_GBS, bench.FALLBACK_BF16_TFLOPS, "fallback")


def test_traffic_is_read_only_for_the_profiled_source(tmp_path, monkeypatch):
    # a copy of the layout bench.read_traffic reads, with the committed figure
    src = os.path.join(ROOT, "quantized_kv_attention_split_b200", "csrc", "decode_kernel.cuh")
    prof = os.path.join(ROOT, "profiles", "decode_decode_64k_affine4_traffic.txt")
    (tmp_path / "profiles").mkdir()
    (tmp_path / "quantized_kv_attention_split_b200" / "csrc").mkdir(parents=True)
    shutil.copy(prof, tmp_path / "profiles")
    kern = tmp_path / "quantized_kv_attention_split_b200" / "csrc" / "decode_kernel.cuh"
    shutil.copy(src, kern)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    first = bench.read_traffic("decode_64k_affine4")
    if first is not None:                       # the profile matches the committed kernel
        assert first > 7e7
    kern.write_text(kern.read_text() + "\n// changed\n")
    assert bench.read_traffic("decode_64k_affine4") is None
    assert bench.read_traffic("no_such_workload") is None


def test_reference_arm_reports_the_gpu_arms_config():
    """Both arms print the same `config` object (workload_config) for the
    same workload, so their lines compare the same thing."""
    import types
    import bench
    from quantized_kv_attention_split_b200 import synthetic as S
    args = types.SimpleNamespace(workload="tiny_decode", steps=1, warmup=3, ref_seconds=1.0)
    line = bench.run_reference(args, 0, 1)
    assert line["config"] == bench.workload_config(S.WORKLOADS["tiny_decode"], 1)
    assert line["impl"] == "reference" and line["config"]["workload"] == "tiny_decode"
