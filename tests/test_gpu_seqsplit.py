"""Sequence split on the GPU.

One sequence is cut into 4 unequal segments, standing for 4 ranks, all run here on one GPU with no
collective. Each segment is summarised by (cumulative transition, zero-start state). Every segment's
start state comes from the prefix scan (kda_segment_compose) of the stacked summaries, and the segment
is run from it. The concatenated outputs and the last segment's final state match the fp64 oracle and
the unsplit run. The distributed wrapper is then run in a one-rank NCCL group, where its result must
equal the plain run bit for bit.
"""
import socket

import numpy as np
import pytest
import torch

import kda_linear_attention_02_b200 as kda
import oracle
from kda_linear_attention_02_b200 import seqsplit, synth
from kda_testlib import assert_close, f32np
from test_gpu_basic import _Agg

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
BF = torch.bfloat16


def _plain(f, init):
    q, k, v, la, b = f
    T, H, D = q.shape
    o = torch.empty(T, H, D, dtype=BF, device=DEV)
    fs = torch.empty(1, H, D, D, device=DEV)
    kda.kda_chunk_fwd(q, k, v, la, b, init[None].contiguous(), synth.cu_from_lengths([T], DEV), o, fs)
    return o, fs[0]


@pytest.mark.parametrize("mu", [0.0, -6.0])
def test_four_segments_match_oracle_and_unsplit_run(mu):
    # mu = -6 (about -0.012 per step): the segments' transitions are far from zero, so every start state
    # depends on the composition of all earlier segments
    H, D = 4, 128
    seg = [1000, 1536, 1217, 1343]
    inp = synth.make_inputs([sum(seg)], H, D, D, dtype=BF, device=DEV, seed=4, with_state0=True, alpha_mu=mu,
                            alpha_sd=1.5 if mu == 0.0 else 0.5)
    f = [inp.q, inp.k, inp.v, inp.log_alpha, inp.beta]
    init = inp.state0[0]
    bounds = np.cumsum([0] + seg).tolist()
    parts = [[x[bounds[p]:bounds[p + 1]].contiguous() for x in f] for p in range(len(seg))]
    summ = [seqsplit.segment_summary(*pp) for pp in parts]
    M_all = torch.stack([m for m, _ in summ])
    Z_all = torch.stack([z for _, z in summ])
    outs, fs_last = [], None
    for p, pp in enumerate(parts):
        X = seqsplit.start_state(M_all, Z_all, p, init)
        o, fs_last = _plain(pp, X)
        outs.append(o)
    o_split = torch.cat(outs)
    o_full, fs_full = _plain(f, init)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    agg = _Agg(BF)
    for h in (0, 3):
        r = oracle.kda_seq(f32np(inp.q[:, h]), f32np(inp.k[:, h]), f32np(inp.v[:, h]), f32np(inp.log_alpha[:, h]),
                           f32np(inp.beta[:, h]), s0=init[h].double().cpu().numpy())
        agg.add("o", f32np(o_split[:, h]), r["o"], f"split outputs head {h}")
        agg.add("state", f32np(fs_last[h]), r["state"], f"split final state head {h}")
    agg.check()
    assert_close(f32np(o_split), f32np(o_full).astype(np.float64), BF, "split vs unsplit outputs")
    assert_close(f32np(fs_last), f32np(fs_full).astype(np.float64), BF, "split vs unsplit final state")


def test_distributed_wrapper_single_rank_nccl_is_the_plain_run():
    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    H, D, T = 2, 128, 777
    inp = synth.make_inputs([T], H, D, D, dtype=BF, device=DEV, seed=5, with_state0=True)
    f = [inp.q, inp.k, inp.v, inp.log_alpha, inp.beta]
    import datetime
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device(DEV), timeout=datetime.timedelta(seconds=60))
    try:
        o = torch.empty(T, H, D, dtype=BF, device=DEV)
        fs = torch.empty(H, D, D, device=DEV)
        seqsplit.sequence_split_prefill(*f, o, fs, inp.state0[0])
        torch.cuda.synchronize()
        # the same on a side stream: every step (library calls, torch copies, the collective) runs there,
        # while the current stream is kept busy with unrelated work
        side = torch.cuda.Stream(DEV)
        side.wait_stream(torch.cuda.current_stream())
        o2 = torch.full_like(o, float("nan"))
        fs2 = torch.full_like(fs, float("nan"))
        busy = torch.randn(4096, 4096, device=DEV)
        for _ in range(8):
            busy = busy @ busy.T / 4096.0
        seqsplit.sequence_split_prefill(*f, o2, fs2, inp.state0[0], stream=side)
        M, Z = seqsplit.segment_summary(*f, stream=side)
        side.synchronize()
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    o_ref, fs_ref = _plain(f, inp.state0[0])
    assert torch.equal(o, o_ref)
    assert torch.equal(fs, fs_ref)
    assert torch.equal(o2, o_ref)
    assert torch.equal(fs2, fs_ref)
    M0, Z0 = seqsplit.segment_summary(*f)
    assert torch.equal(M, M0) and torch.equal(Z, Z0)
