"""Host-side helpers of bench.py (no GPU): the traffic lookup and the FLOP count."""

import bench
import oracle
import workloads as W


def test_recorded_traffic_sums_only_complete_current_entries(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.txt").write_text(
        "kernel=a sources=h1 dram_bytes_per_launch=100 workload=x\n"
        "kernel=b sources=h1 dram_bytes_per_launch=250 workload=x\n"
        "kernel=c sources=h0 dram_bytes_per_launch=999 workload=x\n"
        "kernel=a sources=h1 dram_bytes_per_launch=700 workload=y\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "h1")
    assert bench.recorded_traffic(["a", "b"], "x") == 350
    assert bench.recorded_traffic(["a"], "x") == 100
    assert bench.recorded_traffic(["a"], "y") == 700              # each workload has its own capture
    assert bench.recorded_traffic(["a", "b"], "y") is None        # b was never captured on y
    assert bench.recorded_traffic(["a"], "z") is None
    assert bench.recorded_traffic(["a", "c"], "x") is None        # c was taken on other sources
    assert bench.recorded_traffic(["a", "missing"], "x") is None


def test_committed_traffic_resolves_for_the_captured_workloads_only():
    """The committed summary serves the default line (dpo backward and forward) and the log-prob line at the full
    vocabulary; other workloads, captured nowhere, get null rather than another workload's bytes."""
    bwd = ["k_bwd_pre", "k_bwd_tc", "k_bwd_dq", "k_bwd_dq_ds", "k_bwd_convert"]
    if bench.recorded_traffic(["k_attn_fwd_tc"], "dpo") is None:
        import pytest
        pytest.skip("profiles/traffic.txt was taken on other kernel sources")
    assert bench.recorded_traffic(bwd, "dpo") > 0
    assert bench.recorded_traffic(["k_response_logprobs"], f"dpo-layout-vocab{W.LOGPROB_VOCAB}") > 0
    for other in ("grpo", "longprefix", "hetero"):
        assert bench.recorded_traffic(bwd, other) is None
        assert bench.recorded_traffic(["k_attn_fwd_tc"], other) is None


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
