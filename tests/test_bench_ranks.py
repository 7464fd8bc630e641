"""The multi-rank path of bench.py on CPU: two gloo ranks (one process each,
rendezvous on 127.0.0.1) aggregate their step times the way the GPU bench does
over NCCL: the slowest rank's time is the job's time and the value counts
every rank's FLOP."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import torch
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, _ = bench.dist_env()
        assert (r, w) == (rank, world)
        total, value = bench.aggregate_over_ranks(10.0 + 5.0 * rank, 1e12, 4, world, torch.device("cpu"))
        out.put((rank, total, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, total, value in got:
        assert total == 15.0                                  # max over ranks
        assert value == pytest.approx(2 * 1e12 * 4 / 15e-3 / 1e12)


def test_reference_arm_runs_the_oracle_on_a_sample(tmp_path, capsys):
    """bench.py --impl reference: the oracle on the host cores, rank 0 only."""
    import json
    import sys
    import bench
    sys_argv = sys.argv
    try:
        sys.argv = ["bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0", "--m", "512"]
        assert bench.main() == 0
    finally:
        sys.argv = sys_argv
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
