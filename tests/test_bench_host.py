"""Host-side pieces of bench.py's measurement: the k_fused DRAM-traffic record
(built from ncu CSV logs, read back for roofline.traffic) and its algorithmic
byte count, checked on synthetic capture files without a GPU."""
import csv
import json
import os

import pytest

import bench
import workloads


def _write_capture(path, launches):
    """An ncu --csv log with one row per (launch, metric)."""
    cols = ["ID", "Kernel Name", "Metric Name", "Metric Unit", "Metric Value"]
    with open(path, "w", newline="") as f:
        f.write("==PROF== preamble lines that are not CSV\n")
        w = csv.writer(f, quoting=csv.QUOTE_ALL)
        w.writerow(cols)
        for i, (name, rd, wr, ns) in enumerate(launches):
            w.writerow([i, name, "dram__bytes_read.sum", "Mbyte", f"{rd / 1e6:,.6f}"])
            w.writerow([i, name, "dram__bytes_write.sum", "Mbyte", f"{wr / 1e6:,.6f}"])
            w.writerow([i, name, "gpu__time_duration.sum", "ns", f"{ns}"])


@pytest.fixture()
def captures(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "traffic.json"))
    wl = workloads.LLAMA65B
    shapes = sorted({(p.n, p.k) for p in wl.projections})
    truth = {}
    paths = []
    for d in ("fwd", "bwd"):
        for (n, k) in shapes:
            rd, wr = 3_000_000 + n + 7 * k + (5 if d == "bwd" else 0), 1_000_000 + n
            path = tmp_path / f"traffic_{d}_{n}x{k}.csv"
            # the forward launched first by every case run, then the measured one (last ID)
            _write_capture(path, [("k_fused<0, 256>(FusedArgs)", 1, 1, 10), (f"k_fused<{int(d == 'bwd')}, 256>", rd, wr, 999)])
            truth[f"{d}_{n}x{k}"] = (rd, wr)
            paths.append(str(path))
    return paths, truth


def test_traffic_record_round_trip(captures):
    paths, truth = captures
    bench.write_traffic(paths)
    doc = json.load(open(bench.TRAFFIC_FILE))
    wl = workloads.LLAMA65B
    count = {}
    for p in wl.projections:
        for d in ("fwd", "bwd"):
            count[f"{d}_{p.n}x{p.k}"] = count.get(f"{d}_{p.n}x{p.k}", 0) + 1
    for key, (rd, wr) in truth.items():
        rec = doc["per_launch"][key]
        assert (rec["read"], rec["write"]) == (rd, wr), key       # the last launch of each file
        assert rec["launches_per_step"] == count[key]
        assert rec["duration_ns"] == 999
    traffic, algo = bench.fused_traffic()
    n = sum(count.values())
    assert n == 2 * len(wl.projections)
    want = sum((rd + wr) * count[k] for k, (rd, wr) in truth.items()) // n
    assert traffic == want
    assert algo == sum(doc["per_launch"][k]["algorithmic"] * count[k] for k in count) // n


def test_algorithmic_bytes_of_the_square_forward(captures):
    """fwd 8192x8192 at 8192 tokens, r = 64: X and Y in bf16, the packed weight
    (0.5 B per weight, an E4M3 byte per 64, an fp32 c2 per 16384), B [N, r] and
    the rank-r operand [M, r] in bf16."""
    paths, _ = captures
    bench.write_traffic(paths)
    doc = json.load(open(bench.TRAFFIC_FILE))
    n = k = m = 8192
    r = 64
    expect = 2 * m * k + n * k // 2 + n * k // 64 + 4 * (n * k // 16384) + 2 * n * r + 2 * m * r + 2 * m * n
    assert doc["per_launch"]["fwd_8192x8192"]["algorithmic"] == expect == 305_152_000


def test_traffic_is_null_once_the_kernel_source_changes(captures, monkeypatch):
    paths, _ = captures
    bench.write_traffic(paths)
    assert bench.fused_traffic()[0] is not None
    monkeypatch.setattr(bench, "_sources_digest", lambda paths: "0" * 64)
    assert bench.fused_traffic() == (None, None)


def test_missing_capture_is_refused(captures):
    paths, _ = captures
    with pytest.raises(SystemExit):
        bench.write_traffic(paths[:-1])
    assert not os.path.exists(bench.TRAFFIC_FILE)
