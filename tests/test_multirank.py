"""Multi-rank host logic of bench.py on CPU: two gloo ranks, each with its
own step time and units, reduce to (sum of units) / (slowest rank's time)."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    import bench
    ms = [3.0, 5.0][rank]
    units = [131072, 131072][rank]
    value, ms_max = bench.job_throughput(ms, units, torch.device("cpu"))
    ws, r, _ = bench.dist_env()
    out[rank] = (value, ms_max, ws, r)
    torch.distributed.barrier()
    torch.distributed.destroy_process_group()


def test_two_rank_throughput_uses_max_time_and_total_units():
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
        for r in range(2):
            value, ms_max, ws, rank = out[r]
            assert ms_max == 5.0 and ws == 2 and rank == r
            assert value == pytest.approx(2 * 131072 / 5e-3)
