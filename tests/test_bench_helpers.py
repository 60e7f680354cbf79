"""bench.py's host helpers on the CPU: the DRAM-traffic lookup keyed by the profiled sources'
hash (a stale capture must report null, not a number), and the clock-sample summary."""
import os

import bench


def _tree(tmp_path, kernel_text, stored_hash=None):
    csrc = tmp_path / "axial_band_split_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k_a.cu").write_text(kernel_text)
    (csrc / "k_b.cuh").write_text("// header\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    return prof


def test_traffic_is_reported_only_for_the_profiled_sources(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    prof = _tree(tmp_path, "kernel v1\n")
    h = bench.kernel_source_hash(["k_a.cu", "k_b.cuh"])
    (prof / "traffic.txt").write_text(f"# comment\nsources k_a.cu k_b.cuh\nsource_hash {h}\nattn 1234\n")
    assert bench.traffic_for("attn") == 1234.0
    assert bench.traffic_for("other") is None
    # the kernel changed since the capture: no number
    (tmp_path / "axial_band_split_b200" / "csrc" / "k_a.cu").write_text("kernel v2\n")
    assert bench.traffic_for("attn") is None
    # a listed source that no longer exists, and no summary at all
    (prof / "traffic.txt").write_text(f"sources k_gone.cu\nsource_hash {h}\nattn 1234\n")
    assert bench.traffic_for("attn") is None
    os.unlink(prof / "traffic.txt")
    assert bench.traffic_for("attn") is None


def test_committed_traffic_file_names_existing_sources():
    # every source the committed summary hashes exists, so a changed kernel can be detected
    p = os.path.join(os.path.dirname(bench.__file__), "profiles", "traffic.txt")
    files = [l.split()[1:] for l in open(p) if l.startswith("sources ")][0]
    csrc = os.path.join(os.path.dirname(bench.__file__), "axial_band_split_b200", "csrc")
    assert files and all(os.path.exists(os.path.join(csrc, f)) for f in files)


def test_clock_summary(tmp_path):
    c = bench.ClockSampler(0)
    c.proc = object()                       # as if nvidia-smi had run
    c.path = str(tmp_path / "clocks.csv")
    rows = [
        "0, 1800, 1965, 700.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active, 98",
        "0, 1700, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active, 100",
        "0, 1750, 1965, 980.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active, 97",
        "0, 1965, 1965, 250.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active, 0",
        "0, 1965, 1965, 250.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active, 3",
        "garbage line",
        "0, [N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active, 0",
    ]
    open(c.path, "w").write("\n".join(rows) + "\n")
    s = c.summary()
    # the median is taken over the samples under load only; idle samples still count as samples
    assert s == {"sm_mhz": 1750.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 5,
                 "samples_under_load": 3}
    assert not os.path.exists(c.path)
    # no utilisation column, or nothing under load: the median of every sample
    s = bench.summarize_clock_lines([r.rsplit(",", 1)[0] for r in rows[:4]])
    assert s["sm_mhz"] == 1775.0 and s["samples_under_load"] == 0


def test_aggregate_is_all_ranks_units_over_the_slowest_time():
    assert bench.aggregate(11.0, 1, 10.0) == 1100.0
    assert bench.aggregate(11.0, 8, 20.0) == 4400.0
