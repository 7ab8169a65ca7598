"""The multi-GPU form of the bench (replicas, no data-path collective) on CPU: two gloo ranks
check the per-rank problem seeds, the max-over-ranks timing reduction and the barrier."""
import datetime
import os
import socket
import sys

import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import workloads
        w = bench.replica_workload(workloads.WORKLOADS["small_fp8"], rank, world)
        ms = bench.max_over_ranks(1.5 * (rank + 1), world)   # the slowest rank's time wins
        bench.barrier(world)
        out.put((rank, w.seed, w.shape, ms))
    finally:
        dist.destroy_process_group()


def test_two_replicas_over_gloo():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, seed0, shape0, ms0), (r1, seed1, shape1, ms1) = results
    assert (r0, r1) == (0, 1)
    assert seed0 != seed1 and shape0 == shape1      # own problem per rank, same shape
    assert ms0 == ms1 == 3.0
