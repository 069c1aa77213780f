"""The N>1 host logic of bench.py on CPU: two gloo ranks, each with its own batch of the same shape, and the
max-over-ranks step time that the whole-job value is divided by (no data-path collective exists)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import workloads as W
        P, S = W.group_lengths("dpo")
        seed = bench.rank_tensor_seed("dpo", rank)
        inp = W.make_inputs("dpo", P[:1], S[:1], seed=seed, with_dout=False)
        fake_ms = 10.0 + 5.0 * rank                 # rank 1 is the slow one
        ms = bench.max_over_ranks(fake_ms, "cpu", dist)
        _, f_fwd, f_bwd = bench.flops_of("dpo", P, S)
        val = bench.aggregate_tflops(f_fwd + f_bwd, world, ms)
        out[rank] = (seed, float(inp["q"].float()[0, 0, 0]), ms, val, tuple(inp["q"].shape))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling_and_max_time():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
        assert p.exitcode == 0
    r0, r1 = out[0], out[1]
    assert r0[0] != r1[0] and r0[1] != r1[1]          # each rank draws its own batch
    assert r0[4] == r1[4]                              # of the same shape (per-GPU work fixed)
    assert r0[2] == r1[2] == 15.0                      # both ranks see the slowest rank's time
    assert r0[3] == pytest.approx(r1[3])
    import bench
    import workloads as W
    P, S = W.group_lengths("dpo")
    _, f, b = bench.flops_of("dpo", P, S)
    assert r0[3] == pytest.approx(2 * (f + b) / 15e-3 / 1e12)


def _shard_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import workloads as W
        P, S = W.group_lengths("grpo")
        mine = bench.shard_groups(P, S, world)[rank]
        load = sum(bench.pair_count([P[g]], [S[g]]) for g in mine)
        gathered = [None] * world
        dist.all_gather_object(gathered, (mine, load))       # test-only exchange: the bench itself needs none
        fake_ms = 4.0 + load / 1e7                            # a rank's time follows its load
        ms = bench.max_over_ranks(fake_ms, "cpu", dist)
        out[rank] = (gathered, ms)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_split_one_batch_by_groups():
    """--shard groups: the ranks' groups are disjoint and together the whole batch, the LPT split is balanced to
    within one group's cost, every rank agrees on it, and the job time is the slowest rank's."""
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
        assert p.exitcode == 0
    (g0, ms0), (g1, ms1) = out[0], out[1]
    assert g0 == g1                                        # every rank computed the same split
    import bench
    import workloads as W
    P, S = W.group_lengths("grpo")
    parts = [x[0] for x in g0]
    loads = [x[1] for x in g0]
    assert sorted(parts[0] + parts[1]) == list(range(len(P)))
    assert not set(parts[0]) & set(parts[1])
    costs = [bench.pair_count([p], [ss]) for p, ss in zip(P, S)]
    assert max(loads) - min(loads) <= max(costs)
    assert ms0 == ms1 == pytest.approx(4.0 + max(loads) / 1e7)
