"""The multi-GPU bench runs N independent replicas: each rank times its own
steps, the job is timed as the slowest rank, and the value is the summed work
over that time.  This checks the plumbing with two gloo ranks on the CPU."""
import os
import socket
import sys

import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    t = bench.max_over_ranks(world, 10.0 * (rank + 1), device="cpu")
    v = bench.replica_value(world, step_bytes=4.0e6, ms_total=t, steps=10)
    bench.barrier(world)
    q.put((rank, t, v))
    dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, v in out:
        assert t == 20.0                       # max over ranks
        assert abs(v - 2 * 4.0e6 / 2.0 / 1e6) < 1e-12   # 2 replicas x bytes / (20 ms / 10 steps)
