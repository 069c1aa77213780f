"""Host-side helpers of bench.py (no GPU): the traffic lookup and the FLOP count."""

import bench
import oracle
import workloads as W


def test_recorded_traffic_sums_only_complete_current_entries(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.txt").write_text(
        "kernel=a sources=h1 dram_bytes_per_launch=100 workload=x\n"
        "kernel=b sources=h1 dram_bytes_per_launch=250 workload=x\n"
        "kernel=c sources=h0 dram_bytes_per_launch=999 workload=x\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "h1")
    assert bench.recorded_traffic(["a", "b"]) == 350
    assert bench.recorded_traffic(["a"]) == 100
    assert bench.recorded_traffic(["a", "c"]) is None          # c was taken on other sources
    assert bench.recorded_traffic(["a", "missing"]) is None


def test_pair_count_matches_oracle():
    for name in ("tiny", "dpo"):
        P, S = W.group_lengths(name)
        assert bench.pair_count(P, S) == oracle.allowed_pair_count(P, S)
