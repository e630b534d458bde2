"""The multi-process (N > 1) path of bench.py on CPU: two gloo ranks, max-over-ranks timing
and the whole-job value of the replicas layout (every rank runs its own layer)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        local = [10.0 + 5.0 * rank, 100.0 - rank]  # per-rank step time and e2e time (ms)
        got = bench.ranks_max(local, dist, torch.device("cpu"))
        dist.barrier()
        out[rank] = got + [bench.whole_job_ms_per_layer(got[0], world)]
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
        res = dict(out)
    for rank in range(world):
        assert res[rank][0] == 15.0 and res[rank][1] == 100.0
        assert res[rank][2] == pytest.approx(7.5)
