"""The benchmark's multi-GPU path on CPU: two gloo ranks check the
max-over-ranks timing and the whole-job throughput of independent replicas,
and that only rank 0 of the reference arm does any work."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    local_ms = [12.5, 20.0][rank]
    t_max = bench.max_over_ranks(local_ms, dist, "cpu")
    gbs = bench.replica_throughput(1e9, 10, world, t_max)
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, t_max, gbs))


def test_max_over_ranks_and_replica_throughput_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t_max, gbs in res:
        assert t_max == 20.0                      # slowest replica
        assert gbs == pytest.approx(1e9 * 10 * 2 / 0.020 / 1e9)


def test_single_process_is_its_own_max():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.replica_throughput(352403456, 1000, 1, 59.3) == pytest.approx(5942.7, rel=1e-4)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")

    class Args:
        steps, warmup = 1, 3
    assert bench.reference_arm(Args()) is None
