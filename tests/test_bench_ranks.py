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


def _reference_arm(rank, world):
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--workload", "0",
                          "--gpus", str(world), "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, env=env, timeout=300)
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    return out.returncode, [json.loads(ln) for ln in lines]


def test_reference_arm_runs_on_rank_zero_only():
    rc, lines = _reference_arm(1, 2)
    assert rc == 0 and lines == []
    rc, lines = _reference_arm(0, 2)
    assert rc == 0 and len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["dtype"] == "f64"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    # default flags sample 4 of the 16 query blocks per head, so the time is extrapolated
    assert line["extrapolated"] is True and "(extrapolated)" in line["cpu_baseline"]["sample"]
    assert line["steps"] == 1 and line["ms_per_step"] > 0
    import bench
    import argparse
    from adaptive_block_sparse_hilbert_b200 import synth
    # the reference arm prints the GPU arm's config object
    assert line["config"] == bench.bench_config(synth.WORKLOADS[0], argparse.Namespace(curve="hilbert"), 2)
