"""Host-side bookkeeping of bench.py, without a GPU: the DRAM-traffic record
written from the ncu CSV of one shrunken bandwidth-stress step, its scaling
to full-size launches, and its withdrawal once the kernel sources change;
the summary of the clock samples taken during the timed region (median SM
clock under load, throttle reasons); the physical index of a rank's GPU;
the JSON line of the oracle reference arm, which runs on the host cores."""
import csv
import json

import pytest

import bench
import synth

HEADER = ["ID", "Process ID", "Process Name", "Host Name", "Kernel Name", "Context", "Stream", "Block Size",
          "Grid Size", "Device", "CC", "Section Name", "Metric Name", "Metric Unit", "Metric Value"]


def _calls():
    """The 12 fused launches of a step, in call order, as bench names them."""
    out = []
    for dt in ("f32", "bf16"):
        for (R, C) in synth.BANDWIDTH_SHAPES:
            for q in (6, 8):
                out.append((dt, R, C, q))
    return out


def _write_csv(path, shrink, read_per_row, write_per_row, extra_kernel=True, drop=0):
    """An ncu --csv launch list: one line per (launch, metric).  Launch k of
    the step reads read_per_row(k) and writes write_per_row(k) bytes per
    captured row; values carry thousands separators as ncu prints them."""
    rows = [HEADER]
    lid = 0
    calls = _calls()[:len(_calls()) - drop]
    for k, (dt, R, C, q) in enumerate(calls):
        if extra_kernel:   # another kernel between the fused launches is skipped
            rows.append([str(lid), "1", "python", "h", "void other_kernel()", "1", "7", "(256,1,1)", "(1,1,1)",
                         "0", "10.0", "", "dram__bytes_read.sum", "byte", "123"])
            lid += 1
        r_small = R // shrink
        name = "void gq::rowquant_tma_kernel<false>(gq::TmaParams)"
        for metric, value in (("dram__bytes_read.sum", read_per_row(k) * r_small),
                              ("dram__bytes_write.sum", write_per_row(k) * r_small),
                              ("gpu__time_duration.sum", 1000.0 + k)):
            rows.append([str(lid), "1", "python", "h", name, "1", "7", "(512,1,1)", "(148,1,1)", "0", "10.0", "",
                         metric, "byte" if "bytes" in metric else "nsecond", f"{value:,.0f}"])
        lid += 1
    with open(path, "w", newline="") as f:
        csv.writer(f).writerows(rows)


@pytest.fixture
def traffic_json(tmp_path, monkeypatch):
    p = tmp_path / "rowquant_traffic.json"
    monkeypatch.setattr(bench, "TRAFFIC_PATH", str(p))
    return p


def _names():
    return [(None, None, None, f"{dt} {R}x{C} int{q}") for dt, R, C, q in _calls()]


def test_record_then_scale_to_full_size(tmp_path, traffic_json):
    shrink = 4
    rd = lambda k: 1000 + 10 * k          # bytes per row, distinct per launch
    wr = lambda k: 700 + 3 * k
    csv_path = tmp_path / "step.csv"
    _write_csv(csv_path, shrink, rd, wr)
    out = bench.record_traffic(str(csv_path), shrink)
    assert out["shrink"] == shrink and len(out["per_call"]) == 12
    assert out["kernel_source_hash"] == bench.kernel_source_hash()
    assert str(csv_path) in out["command"]
    on_disk = json.loads(traffic_json.read_text())
    assert on_disk["per_call"] == out["per_call"]
    for k, (dt, R, C, q) in enumerate(_calls()):
        rec = out["per_call"][f"{dt} {R}x{C} int{q}"]
        assert rec["rows_captured"] == R // shrink
        assert rec["dram_read_bytes"] == rd(k) * (R // shrink)
        assert rec["dram_bytes_per_row"] == pytest.approx(rd(k) + wr(k))
        # algorithmic bytes: the row read, w_hat written in the input dtype,
        # packed codes and a binary16 scale per row
        esz = 4 if dt == "f32" else 2
        prb = 3 * ((C + 3) // 4) if q == 6 else C
        assert rec["algorithmic_bytes"] == (R // shrink) * (C * 2 * esz + prb + 2)
    # full-size traffic per launch: bytes per row times each launch's full row count, averaged
    want = sum((rd(k) + wr(k)) * R for k, (_, R, _, _) in enumerate(_calls())) / 12
    got, info = bench.traffic_per_launch(bench.kernel_source_hash(), _names())
    assert got == pytest.approx(want) and info["shrink"] == shrink


def test_traffic_withdrawn_when_sources_change(tmp_path, traffic_json):
    csv_path = tmp_path / "step.csv"
    _write_csv(csv_path, 8, lambda k: 1000, lambda k: 500)
    bench.record_traffic(str(csv_path), 8)
    assert bench.traffic_per_launch(bench.kernel_source_hash(), _names())[0] is not None
    assert bench.traffic_per_launch("0" * 16, _names()) == (None, None)
    # a launch the record does not cover, or no record at all
    assert bench.traffic_per_launch(bench.kernel_source_hash(), _names() + [(0, 0, 0, "f32 8x8 int6")]) == (None, None)
    traffic_json.unlink()
    assert bench.traffic_per_launch(bench.kernel_source_hash(), _names()) == (None, None)


def test_record_refuses_an_incomplete_step(tmp_path, traffic_json):
    csv_path = tmp_path / "step.csv"
    _write_csv(csv_path, 4, lambda k: 1000, lambda k: 500, drop=1)
    with pytest.raises(AssertionError):
        bench.record_traffic(str(csv_path), 4)
    assert not traffic_json.exists()


def test_kernel_source_hash_covers_the_fused_kernel_sources():
    h = bench.kernel_source_hash()
    assert len(h) == 16 and h == bench.kernel_source_hash()
    assert "gq_rowquant_tma.cuh" in bench.FUSED_KERNEL_SOURCES


class _Exited:
    """Stands in for the nvidia-smi process of a ClockSampler."""

    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0

    def kill(self):
        pass


def _sampler_over(tmp_path, lines):
    s = bench.ClockSampler(0)
    s.path = str(tmp_path / "clocks.csv")
    with open(s.path, "w") as f:
        f.write("\n".join(lines) + "\n")
    s.proc = _Exited()
    return s


def test_clock_sampler_summary(tmp_path):
    na, act = "Not Active", "Active"
    lines = [
        f"210, 1965, 95.1, 0x0000000000000001, {na}, {na}, {na}, {na}",      # idle before the region
        f"1965, 1965, 812.0, 0x0000000000000000, {na}, {na}, {na}, {na}",
        f"1950, 1965, 990.2, 0x0000000000000004, {na}, {na}, {na}, {act}",
        f"1935, 1965, 1001.7, 0x0000000000000004, {na}, {na}, {na}, {act}",
        "garbled line",
    ]
    out = _sampler_over(tmp_path, lines).stop()
    assert out["samples"] == 4
    assert out["sm_max_mhz"] == 1965.0
    assert out["sm_mhz"] == 1950.0              # the idle 210 MHz sample is not "under load"
    assert out["reasons"] == ["sw_power_cap"]
    assert not set(out["reasons"]) & bench.REJECT


def test_clock_sampler_reports_rejecting_reasons(tmp_path):
    na, act = "Not Active", "Active"
    lines = [f"1400, 1965, 1000.0, 0x0000000000000048, {act}, {na}, {act}, {na}"]
    out = _sampler_over(tmp_path, lines).stop()
    assert out["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert set(out["reasons"]) & bench.REJECT


def test_clock_sampler_without_samples(tmp_path):
    assert _sampler_over(tmp_path, ["[N/A]"]).stop() is None
    assert bench.ClockSampler(0).stop() is None     # never started


def test_physical_gpu_index(monkeypatch):
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "3, 5,7")
    assert [bench.physical_gpu_index(r) for r in range(4)] == [3, 5, 7, 3]
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "GPU-1234abcd")
    assert bench.physical_gpu_index(0) == 0
    monkeypatch.delenv("CUDA_VISIBLE_DEVICES")
    assert bench.physical_gpu_index(2) == 2


def test_reference_arm_json_line():
    """`bench.py --impl reference` times the oracle on the host cores and
    prints one JSON line in the bench contract; it needs no GPU."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 1
    assert line["steps"] == 1 and line["warmup"] == 3 and line["higher_is_better"] is True
    assert line["value"] > 0 and line["unit"] == "GB/s" and line["ms_per_step"] > 0
    assert line["config"]["workload"].startswith("bandwidth stress")
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == line["value"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    # the minimum warm-up is enforced
    bad = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--warmup", "2"],
                         capture_output=True, text=True, timeout=120, cwd=root)
    assert bad.returncode != 0 and "--warmup must be at least 3" in bad.stderr
