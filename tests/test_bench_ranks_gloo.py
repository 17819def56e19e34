"""bench.py's multi-rank plumbing on CPU: two gloo ranks pass the barrier, every rank reads the slowest
rank's time, and the whole-job throughput is the units of all ranks over that time (weak scaling)."""
import os
import socket

import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    out = None
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world)
        import bench
        bench.barrier(world)
        ms = 10.0 + 5.0 * rank                       # rank 1 is the slow one
        ms_max = bench.max_over_ranks(ms, world, device="cpu")
        tokens_per_rank = 1000
        out = (ms_max, world * tokens_per_rank / (ms_max / 1e3))
    finally:
        q.put((rank, out))
        if dist.is_initialized():
            dist.destroy_process_group()


def test_barrier_and_max_over_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
    assert res[0] == res[1] == (15.0, 2 * 1000 / 0.015)
