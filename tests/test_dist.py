"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2, no GPU).

Each rank runs its own step on its own seeded data (weak scaling, no data-path
collective); the job's time is the slowest rank's, and the value aggregates all ranks.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import numpy as np
    import torch.distributed as dist

    import bench
    from bit_weight_quantized_tgemm_b200 import synth

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [2.0, 3.5][rank]
        slowest = bench.max_over_ranks(local_ms, world)
        w = synth.ALL["tiny"]
        prob = (w.make() if rank == 0 else bench._reseed(w, rank).make())
        digest = float(np.asarray(prob.x, dtype=np.float64).sum())
        got = [None] * world
        dist.all_gather_object(got, digest)
        value = bench.aggregate_value(world, 1e12, slowest)
        out[rank] = (slowest, got, value)
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_distinct_data():
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    for r in range(2):
        slowest, digests, value = res[r]
        assert slowest == 3.5                      # max over ranks
        assert digests[0] != digests[1]            # each rank has its own batch
        assert value == pytest.approx(2 * 1e12 / 3.5e-3 / 1e12)
