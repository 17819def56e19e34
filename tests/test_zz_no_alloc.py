"""kda_chunk_fwd_noalloc: the chunked forward for callers that may not allocate device memory.

A serving engine that hands all device memory to its own pool, or a program with a fixed
device-memory budget, cannot give kda_chunk_fwd a workspace; the no-allocation entry point keeps its
scratch in a fixed array inside the library instead.  This test calls it twice in a row through the
C ABI and compares every output with kda_chunk_fwd given an ordinary workspace, within the bf16
tolerances the other tests use.  It sits in a file of its own that pytest collects last.
"""
import pytest
import torch

import kda_linear_attention_02_b200 as kda
from kda_linear_attention_02_b200 import synth
from kda_testlib import assert_close, f32np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
BF = torch.bfloat16


def _outputs(inp, H, D, ckcu):
    T, N = inp.total_tokens, inp.n_seqs
    return (torch.full((T, H, D), float("nan"), dtype=BF, device=DEV),
            torch.full((N, H, D, D), float("nan"), device=DEV),
            torch.full((int(ckcu[-1]), H, D, D), float("nan"), device=DEV),
            torch.full((N, H, D, D), float("nan"), device=DEV))


def test_noalloc_matches_workspace_entry_point_twice():
    H, D, S = 8, 128, 512
    lengths = [1000, 64, 513, 0, 2048, 77]
    inp = synth.make_inputs(lengths, H, D, D, dtype=BF, device=DEV, seed=21, with_state0=True)
    ckcu = kda.kda_ckpt_offsets(inp.cu_seqlens.cpu(), S)
    ckcu_d = ckcu.to(DEV)
    ref = _outputs(inp, H, D, ckcu)
    kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.state0, inp.cu_seqlens, ref[0], ref[1],
                      ckpt_stride=S, checkpoints=ref[2], ckpt_cu=ckcu_d, final_transition=ref[3])
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    for call in range(2):
        got = _outputs(inp, H, D, ckcu)
        kda.kda_chunk_fwd_noalloc(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.state0, inp.cu_seqlens,
                                  got[0], got[1], ckpt_stride=S, checkpoints=got[2], ckpt_cu=ckcu_d,
                                  final_transition=got[3])
        torch.cuda.synchronize()
        assert kda.kda_get_device_status() == 0
        for name, a, b in zip(("o", "final_state", "checkpoints", "transition"), got, ref):
            assert_close(f32np(a), f32np(b), BF, f"no-alloc call {call}: {name}")


def test_noalloc_refuses_batches_beyond_its_scratch():
    # 16 sequences x 32 heads need more than the fixed 64 MiB for their carried states alone
    H, D = 32, 128
    inp = synth.make_inputs([64] * 16, H, D, D, dtype=BF, device=DEV, seed=2)
    o = torch.empty(inp.total_tokens, H, D, dtype=BF, device=DEV)
    with pytest.raises(kda.KDAError) as e:
        kda.kda_chunk_fwd_noalloc(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, None, inp.cu_seqlens, o)
    assert e.value.status == -6      # KDA_ERR_WORKSPACE
