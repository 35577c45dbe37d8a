"""Multi-GPU path on the CPU: bench.py runs one independent replica per rank (the data
plane shards by sequence, so no collective touches the data path) and reports the
whole-job throughput against the slowest rank's time.  Two gloo ranks check the
reduction both ranks perform."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times_ms, units, out):
    import sys
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    import bench
    thr, ms = bench.job_throughput(units, times_ms[rank], dist)
    out.put((rank, thr, ms))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("times_ms", [(3.0, 5.0), (7.5, 2.5)])
def test_two_replicas_report_job_throughput_at_slowest_rank(times_ms):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, times_ms, 10.0, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    slow = max(times_ms)
    for rank, thr, ms in res:
        assert ms == slow
        assert abs(thr - 2 * 10.0 / (slow * 1e-3)) < 1e-6
