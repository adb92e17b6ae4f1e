"""The bench's multi-rank plumbing on CPU: world size 2 over gloo.

Each rank reports a different step time; the job time is the maximum over
ranks and the whole-job throughput counts every rank's tokens.
"""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    local_ms = 100.0 + 50.0 * rank
    mx = bench.reduce_max(local_ms, world, torch.device("cpu"))
    bench.barrier(world)
    out.put((rank, mx, bench.throughput(world, 32768, 10, mx)))
    dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_throughput():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, tput in res:
        assert mx == 150.0
        assert tput == pytest.approx(2 * 32768 * 10 / 0.150)
