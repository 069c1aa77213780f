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


def test_shard_groups_lpt_partition():
    """Every group lands on exactly one rank, the split is deterministic, and LPT keeps the heaviest and lightest
    rank within one group's cost of each other."""
    for name in ("dpo", "grpo", "hetero"):
        P, S = W.group_lengths(name)
        costs = [bench.pair_count([p], [ss]) for p, ss in zip(P, S)]
        for world in (1, 2, 3, 4, 8):
            parts = bench.shard_groups(P, S, world)
            assert len(parts) == world
            flat = sorted(g for part in parts for g in part)
            assert flat == list(range(len(P)))
            loads = [sum(costs[g] for g in part) for part in parts]
            if len(P) >= world:
                assert max(loads) - min(loads) <= max(costs)
            assert parts == bench.shard_groups(P, S, world)
