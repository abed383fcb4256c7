"""Host logic of bench.py that needs no GPU: the clock record taken during the timed region.

The bench rejects its own number when the clocks seen during the timed region show a hardware
or thermal slowdown, so the parsing of the nvidia-smi samples and the choice of the samples
that fall inside the region are checked here on synthetic sample files.
"""
import os
import sys
import tempfile

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _row(sm, reasons=()):
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    flags = ["Active" if n in reasons else "Not Active" for n in names]
    active = "0x0000000000000004" if reasons else "0x0000000000000000"
    return ", ".join(["0", str(sm), "1965", "812.40", active, *flags]) + "\n"


def _sampler(lines, marks=(None, None), partial=None):
    fd, path = tempfile.mkstemp(suffix=".csv")
    with os.fdopen(fd, "w") as f:
        f.writelines(lines)
        if partial:
            f.write(partial)  # a line nvidia-smi has not finished
    clk = bench.ClockSampler(0)
    clk.path = path
    clk.marks = list(marks)
    return clk


def test_summary_keeps_the_timed_window():
    # two idle samples, the region (3 samples at 1965 MHz with a power cap), two after it
    lines = [_row(600), _row(645)] + [_row(1965, ("sw_power_cap",))] * 3 + [_row(1800), _row(700)]
    s = _sampler(lines, marks=(2, 5)).summary()
    # rows 1..5: one sample before the region, the region, one after
    assert s["samples"] == 5
    assert s["sm_mhz"] == 1965.0
    assert s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]


def test_summary_reports_thermal_slowdown_inside_the_window():
    lines = [_row(1965)] + [_row(1500, ("hw_thermal_slowdown",))] * 2 + [_row(1965)]
    s = _sampler(lines, marks=(1, 3)).summary()
    assert "hw_thermal_slowdown" in s["reasons"]


def test_summary_without_marks_uses_every_sample_and_skips_a_partial_line():
    lines = [_row(1965), _row(1960)]
    s = _sampler(lines, partial="0, 1965, 19").summary()
    assert s["samples"] == 2
    assert s["sm_mhz"] == 1962.5
    assert s["reasons"] == []


def test_summary_falls_back_when_no_sample_landed_in_the_window():
    lines = [_row(1965), _row(1965)]
    s = _sampler(lines, marks=(2, 2)).summary()
    assert s["samples"] == 2


def test_summary_without_samples_is_marked_unavailable():
    s = _sampler([]).summary()
    assert s == {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}


def test_sampler_without_nvidia_smi_degrades_to_unavailable(monkeypatch):
    # no nvidia-smi on the PATH: the sampler must not raise, and the summary says so
    monkeypatch.setenv("PATH", tempfile.gettempdir())
    clk = bench.ClockSampler(0, period_ms=5)
    with clk:
        clk.begin()
        clk.end()
    assert clk.summary()["reasons"] == ["unavailable"]


def _fake_smi(tmp_path, min_ms):
    """A stand-in nvidia-smi that refuses intervals below `min_ms` and otherwise prints one
    sample row per interval."""
    exe = tmp_path / "nvidia-smi"
    exe.write_text(
        "#!/bin/sh\n"
        "ms=0; prev=''\n"
        "for a in \"$@\"; do if [ \"$prev\" = '-lms' ]; then ms=$a; fi; prev=$a; done\n"
        f"if [ \"$ms\" -lt {min_ms} ]; then exit 2; fi\n"
        "while true; do echo '0, 1965, 1965, 700.00, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active'; "
        "sleep 0.05; done\n")
    exe.chmod(0o755)
    return str(tmp_path)


def test_sampler_records_rows_from_nvidia_smi(monkeypatch, tmp_path):
    monkeypatch.setenv("PATH", _fake_smi(tmp_path, 0) + os.pathsep + os.environ.get("PATH", ""))
    with bench.ClockSampler(0) as clk:
        clk.begin()
        clk.end()
    s = clk.summary()
    assert clk.period_ms == 20
    assert s["samples"] >= 1 and s["sm_mhz"] == 1965.0 and s["reasons"] == []


def test_sampler_falls_back_to_200_ms_when_the_interval_is_refused(monkeypatch, tmp_path):
    monkeypatch.setenv("PATH", _fake_smi(tmp_path, 200) + os.pathsep + os.environ.get("PATH", ""))
    with bench.ClockSampler(0) as clk:
        clk.begin()
        clk.end()
    s = clk.summary()
    assert clk.period_ms == 200
    assert s["samples"] >= 1 and s["sm_mhz"] == 1965.0


def test_reference_arm_reports_our_config(monkeypatch, capsys):
    import json
    import types

    class QuickSample:  # stands in for the oracle run; only the line's shape is checked here
        def run(self, budget):
            return {"value": 1.0, "cores": 4, "sample": "stand-in"}

    monkeypatch.setattr(bench, "CpuSample", QuickSample)
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    bench.run_reference(types.SimpleNamespace(steps=2, warmup=3, layers=32))
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == "GB/s" and line["higher_is_better"] is True
    assert line["config"] == bench.decode_config(32, 1)
    assert line["config"]["layer_calls_per_step"] == 672
    assert line["config"]["quantised_weight_bytes"] == 3340772224
    assert line["e2e"] == {"value": 1.0, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_algorithmic_bytes_per_launch_of_the_decode_step():
    # 0.5159 B per weight (codes 0.5, FP8 constant 1/64, fp32 group scale 4/(64*256), plus the mean),
    # x, A, B and h in bf16; averaged over the 21 launches of one layer (7 linears x M = 1, 4, 16).
    per_layer = [bench.fwd_bytes(n, k, M, bench.RANK_7B) for M in bench.DECODE_M for (_, n, k) in bench.SHAPES_7B]
    assert len(per_layer) == 21
    assert round(sum(per_layer) / 21) == 15_427_259
    # the weight part alone: codes + constants + scales + mean of a 4096 x 4096 weight
    n = k = 4096
    assert bench.weight_bytes(n, k) == n * k // 2 + n * k // 64 + 4 * ((n * k // 64 + 255) // 256) + 4
    assert bench.fwd_bytes(n, k, 1, 16) == bench.weight_bytes(n, k) + 2 * k + 2 * 16 * k + 2 * n * 16 + 2 * n


def test_traffic_record_is_reported_only_while_its_sources_are_unchanged(monkeypatch, tmp_path):
    import hashlib
    import json
    (tmp_path / "profiles").mkdir()
    src = tmp_path / "k.cu"
    src.write_bytes(b"__global__ void k() {}\n")
    rec = {"sources": ["k.cu"], "sources_sha256_16": hashlib.sha256(src.read_bytes()).hexdigest()[:16],
           "bytes_per_launch": 1234}
    (tmp_path / "profiles" / "k_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profile_traffic("k_traffic.json") == 1234
    assert bench.profile_traffic("missing.json") is None
    src.write_bytes(b"__global__ void k() { }\n")  # the kernel changed after the capture
    assert bench.profile_traffic("k_traffic.json") is None


def test_committed_traffic_records_are_consistent():
    # the records the bench quotes: their sources exist, their algorithmic bytes are the bench's own
    # figure for one decode layer, and the measured DRAM bytes are within 1 % of it (nothing re-read)
    import json
    for name, kernel in (("decode_fwd_traffic.json", "k_decode_fwd"), ("decode_bwd_traffic.json", "k_decode_bwd")):
        with open(os.path.join(bench.ROOT, "profiles", name)) as f:
            rec = json.load(f)
        assert rec["kernel"] == kernel
        assert all(os.path.exists(os.path.join(bench.ROOT, s)) for s in rec["sources"])
        assert rec["algorithmic_bytes_per_launch"] == 15_427_259
        assert rec["launches_averaged"] == 21
        assert 1.0 <= rec["bytes_per_launch"] / rec["algorithmic_bytes_per_launch"] < 1.01
