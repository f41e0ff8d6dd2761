"""The N > 1 host logic of bench.py (replicas only: per-rank seeds, a barrier,
the max of the step times over ranks, the whole-job rate), run as two gloo
ranks on the CPU."""
import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    from linear_attention_layer_causal_b200 import workloads as W
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank "measures" a different time; all must agree on the max
        my_ms = 10.0 + 7.0 * rank
        mx = bench.reduce_max(dist, my_ms, "cpu")
        dist.barrier()
        # per-rank inputs differ (seeded by rank) but have the workload's shapes
        inp = W.make_prefill(W.TINY, "cpu", seed=bench.rank_seed(W.TINY.seed, rank))
        first = float(inp["qkv"].float().flatten()[0])
        firsts = [None] * world
        dist.all_gather_object(firsts, first)
        out[rank] = (mx, bench.job_rate(128, world, 5, mx), firsts, tuple(inp["qkv"].shape))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_and_rate():
    world, port = 2, 29500 + os.getpid() % 2000
    # the manager's server process is spawned too: forking a process that
    # already runs threads (torch's) can deadlock the child
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, start_method="spawn")
        res = dict(out)
    assert sorted(res) == [0, 1]
    for rank, (mx, rate, firsts, shape) in res.items():
        assert mx == pytest.approx(17.0)                 # the slower rank's time
        assert rate == pytest.approx(128 * 2 * 5 / 0.017)  # all ranks' tokens / max time
        assert firsts[0] != firsts[1]                    # distinct seeded inputs
        assert shape == res[0][3]


def test_single_process_helpers():
    import importlib
    sys.path.insert(0, ROOT)
    bench = importlib.import_module("bench")
    assert bench.reduce_max(None, 3.5, "cpu") == 3.5
    assert bench.rank_seed(1001, 0) == 1001 and bench.rank_seed(1001, 1) != 1001
    assert bench.job_rate(4096, 1, 20, 10.0) == pytest.approx(4096 * 20 / 0.01)
