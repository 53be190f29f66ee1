"""The N > 1 host logic of bench.py on CPU: two gloo ranks, max-over-ranks timing and the
whole-job throughput (weak scaling: every rank runs its own copy of the workload)."""
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
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    my_ms = [0.5, 0.8][rank]
    mx = bench.max_over_ranks(my_ms, world, device="cpu")
    val = bench.job_throughput(1e12, world, mx)
    out.put((rank, mx, val))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_max_and_job_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for _, mx, val in res:
        assert mx == pytest.approx(0.8)
        assert val == pytest.approx(2 * 1e12 / 0.8e-3)
