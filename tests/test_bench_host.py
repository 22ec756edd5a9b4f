"""Host logic of bench.py on CPU: the DRAM-traffic record written from an
ncu raw export and read back against the kernel source hash, and the
median / coefficient-of-variation summary of repeated runs."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _write_raw_csv(path, rows):
    header = ["ID", "Kernel Name", "dram__bytes_read.sum", "dram__bytes_write.sum"]
    units = ["", "", "Mbyte", "Kbyte"]
    with open(path, "w") as f:
        for r in [header, units] + rows:
            f.write(",".join(f'"{c}"' for c in r) + "\n")


def test_traffic_record_round_trip(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "traffic.json"))
    csv_path = tmp_path / "raw.csv"
    _write_raw_csv(csv_path, [
        ["0", "void decode::split_i8_kernel<256, 1, 2, 0>(SplitArgs, I8Lut, float)", "822.5", "6,000"],
        ["1", "void decode::combine_kernel<__half, 256, 1>(CombineArgs)", "10.0", "1.0"],
        ["2", "void decode::split_i8_kernel<256, 1, 2, 0>(SplitArgs, I8Lut, float)", "821.5", "4,000"],
    ])
    bench.record_traffic(str(csv_path), "split_i8", 4.0, "test capture")
    rec = json.load(open(tmp_path / "traffic.json"))
    # the two matching launches average (822.5 + 6) and (821.5 + 4) MB, in bytes
    per_launch = ((822.5e6 + 6.0e6) + (821.5e6 + 4.0e6)) / 2
    assert rec["launches"] == 2
    assert rec["captured_bytes_per_launch"] == pytest.approx(per_launch)
    assert rec["traffic_bytes_per_launch"] == pytest.approx(4.0 * per_launch)
    assert rec["source_hash"] == bench.source_hash()
    assert bench.read_traffic() == pytest.approx(4.0 * per_launch)
    # a record taken on another kernel source is not used
    rec["source_hash"] = "0" * 16
    json.dump(rec, open(tmp_path / "traffic.json", "w"))
    assert bench.read_traffic() is None


def test_traffic_record_without_the_kernel_fails(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "traffic.json"))
    csv_path = tmp_path / "raw.csv"
    _write_raw_csv(csv_path, [["0", "void decode::combine_kernel<__half, 256, 1>(CombineArgs)", "10.0", "1.0"]])
    with pytest.raises(SystemExit):
        bench.record_traffic(str(csv_path), "split_i8", 4.0, "test capture")
    assert not os.path.exists(tmp_path / "traffic.json")


def test_missing_traffic_record_reads_as_none(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "absent.json"))
    assert bench.read_traffic() is None


def test_median_and_cv():
    m, cv = bench.med_cv([3.0, 1.0, 2.0])
    assert m == 2.0
    # population standard deviation of (1, 2, 3) over their mean 2
    assert cv == pytest.approx((2.0 / 3.0) ** 0.5 / 2.0)
    assert bench.med_cv([5.0]) == (5.0, 0.0)
