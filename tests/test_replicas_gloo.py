"""The N > 1 path of bench.py on CPU: two `gloo` ranks run as replicas (no
collective on the data path); the job time is the slowest rank's, the value
the bytes of all ranks over that time, and only rank 0 runs the reference arm."""
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    my_ms = 10.0 + 5.0 * rank                       # rank 1 is the slow replica
    slowest = bench.max_over_ranks(my_ms, dist)
    value = bench.whole_job_gbs(world, 20, 1024, 4218880, slowest)
    dist.barrier()
    out[rank] = (slowest, value)
    dist.destroy_process_group()


def test_two_gloo_replicas_take_the_slowest_time():
    world, port = 2, _free_port()
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 15.0
    expect = 2 * 20 * 1024 * 4218880 / 15e-3 / 1e9
    assert abs(out[0][1] - expect) < 1e-6 and out[0][1] == out[1][1]


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        steps, warmup = 1, 0
    bench.run_reference(Args())
    assert capsys.readouterr().out == ""
