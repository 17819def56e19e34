"""Sequence split, exchange step on CPU: two or four gloo ranks all-gather their fixed-size (transition,
zero-start state) summaries; every rank must receive all summaries in rank order, bit for bit."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _summaries(rank, H, dk, dv):
    g = torch.Generator().manual_seed(100 + rank)
    return torch.randn(H, dk, dk, generator=g), torch.randn(H, dk, dv, generator=g)


def _worker(rank, world, port, H, dk, dv, q):
    import torch.distributed as dist
    from kda_linear_attention_02_b200 import seqsplit
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    ok = False
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world)
        M, Z = _summaries(rank, H, dk, dv)
        M_all, Z_all = seqsplit.gather_segment_summaries(M, Z)
        ok = tuple(M_all.shape) == (world, H, dk, dk) and tuple(Z_all.shape) == (world, H, dk, dv)
        for p in range(world):
            Mp, Zp = _summaries(p, H, dk, dv)
            ok = ok and torch.equal(M_all[p], Mp) and torch.equal(Z_all[p], Zp)
    finally:
        q.put((rank, bool(ok)))          # report even when something raised, so the parent never waits out
        if dist.is_initialized():
            dist.destroy_process_group()


@pytest.mark.parametrize("world,dk,dv", [(2, 128, 128), (2, 64, 128), (4, 128, 64)])
def test_gather_segment_summaries(world, dk, dv):
    H = 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, H, dk, dv, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
    assert res == {r: True for r in range(world)}
