"""World-size-2 runs of bench.py's multi-rank host logic on CPU (gloo).

The hot path shards by request: each rank serves its own batch and there is no
data-path collective, so the job's only exchange is the MAX all-reduce of the
timed region (and of the end-to-end leg).  These tests run that logic in two
processes: the ranks draw independent batches, both see the slowest rank's
time, the whole-job throughput counts every rank's units over that time, and
a leg that holds barriers runs on every rank or on none (a MIN all-reduce).
"""
import datetime
import os
import socket

import numpy as np
import torch.distributed as dist
import torch.multiprocessing as mp

from tree_forked_decision_b200 import inputs

WORKLOAD = "tiny_fp32"
STEPS = 3


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench  # noqa: E402  (repository root is on sys.path for the tests)

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ws, r, _ = bench.dist_env()
        seed = bench.rank_seed(WORKLOAD, None, r)
        tree, a, g, _ = inputs.make_inputs(WORKLOAD, seed=seed)
        ms_local = 10.0 + 2.5 * r  # this rank's timed region, as if measured
        ms = bench.max_over_ranks(ms_local, dist, "cpu")
        value = bench.job_throughput(tree.branch_tokens, STEPS, ws, ms)
        # a leg that holds barriers runs on every rank or on none
        only_rank0 = bench.all_ranks(r == 0, dist, "cpu")
        everywhere = bench.all_ranks(True, dist, "cpu")
        np.savez(os.path.join(out_dir, f"rank{r}.npz"), ws=ws, seed=seed, q=a["q"].numpy(),
                 gk=g["k"].numpy(), ms=ms, value=value, branch=tree.branch_tokens,
                 only_rank0=only_rank0, everywhere=everywhere)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _run(tmp_path, world=2):
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    return [np.load(tmp_path / f"rank{r}.npz") for r in range(world)]


def test_two_ranks_independent_batches_and_max_time(tmp_path):
    r0, r1 = _run(tmp_path)
    assert int(r0["ws"]) == int(r1["ws"]) == 2
    # independent requests per rank: different seeds, different inputs
    assert int(r0["seed"]) != int(r1["seed"])
    assert not np.array_equal(r0["q"], r1["q"])
    assert not np.array_equal(r0["gk"], r1["gk"])
    # the job time is the slowest rank's, on every rank
    assert float(r0["ms"]) == float(r1["ms"]) == 12.5
    # whole-job throughput: both ranks' units over the slowest rank's time
    units = int(r0["branch"]) + int(r1["branch"])
    expect = units * STEPS / 0.0125
    assert abs(float(r0["value"]) - expect) <= 1e-9 * expect
    assert float(r0["value"]) == float(r1["value"])
    # leg decisions agree across ranks
    assert not bool(r0["only_rank0"]) and not bool(r1["only_rank0"])
    assert bool(r0["everywhere"]) and bool(r1["everywhere"])


def test_rank_seed_and_throughput_single_rank():
    import bench

    assert bench.rank_seed(WORKLOAD, None, 0) == inputs.WORKLOADS[WORKLOAD]["idx"]
    assert bench.rank_seed(WORKLOAD, 7, 3) == 3007
    assert bench.max_over_ranks(4.25, None, "cpu") == 4.25
    assert bench.all_ranks(True, None, "cpu") is True and bench.all_ranks(0, None, "cpu") is False
    assert bench.job_throughput(100, 2, 1, 50.0) == 4000.0
    assert bench.percentiles([5.0, 1.0, 2.0, 3.0, 4.0, 6.0, 7.0, 8.0, 9.0, 10.0]) == (5.0, 10.0)
    assert bench.percentiles([2.5]) == (2.5, 2.5)
