"""Multi-process host logic of bench.py on the CPU: two gloo ranks, each with
its own replica of the workload, timed as the max over ranks (the layer
shards over (b, h) with no collective on the data path, so the only
cross-rank step is the timing reduction)."""
import datetime
import os
import socket

import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist

    import bench
    from gated_delta_rule_153_b200.inputs import TINY, make_chunk_inputs
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        barrier, max_over_ranks = bench.rank_reducers(dist, torch.device("cpu"))
        barrier()
        ms_here = 10.0 + 5.0 * rank           # this rank's timed region
        ms_max = max_over_ranks(ms_here)
        inp = make_chunk_inputs(TINY, seed=bench.replica_seed(TINY.seed, rank))
        out.put((rank, ms_max, float(inp["q"].double().abs().sum()),
                 bench.whole_job_rate(TINY.B * TINY.T * TINY.H, world, 3, ms_max)))
        barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_as_max_and_run_independent_replicas():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, m0, q0, v0), (r1, m1, q1, v1) = res
    assert (r0, r1) == (0, 1)
    assert m0 == m1 == 15.0                  # both ranks see the slowest rank's time
    assert q0 != q1                          # each rank holds its own batch
    tokens = 1 * 64 * 1
    assert v0 == v1 == world * tokens * 3 / 0.015


def test_single_rank_rate_matches_formula():
    import bench
    assert bench.whole_job_rate(100, 1, 10, 2.0) == 100 * 10 / 0.002
    assert bench.replica_seed(5, 0) == 5 and bench.replica_seed(5, 1) != 5
