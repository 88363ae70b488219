"""Host-side bookkeeping of bench.py, without a GPU: the DRAM-traffic record
written from the ncu CSV of one shrunken bandwidth-stress step, its scaling
to full-size launches, and its withdrawal once the kernel sources change."""
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
