"""The multi-GPU bench path on CPU: two gloo ranks agree on the slowest rank's
time and on the whole-job throughput (replicas: no data-path collective)."""
import multiprocessing as mp
import os
import socket

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    import datetime

    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        mx = bench.max_over_ranks([100.0 + 7 * rank, 5.0 * (ws - rank)], device="cpu")
        v = bench.job_value(3 * 1024, dist.get_world_size(), mx[0])
        q.put((rank, mx, v))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_and_job_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    out = sorted(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, v in out:
        assert mx == [107.0, 10.0]                      # slowest rank per entry
        assert abs(v - 2 * 3 * 1024 / 0.107) < 1e-6     # all ranks' tokens / slowest time


def test_single_process_helpers():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.5, 2.0]) == [1.5, 2.0]
    assert bench.job_value(1024, 1, 1000.0) == 1024.0
