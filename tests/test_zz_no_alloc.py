"""kda_chunk_fwd_noalloc: the chunked forward for callers that may not allocate device memory.

A serving engine that hands all device memory to its own pool, or a program with a fixed
device-memory budget, cannot give kda_chunk_fwd a workspace; the no-allocation entry point keeps its
scratch in a fixed array inside the library instead.  This test calls it twice in a row through the
C ABI and compares every output with kda_chunk_fwd given an ordinary workspace.  Both run the same
kernels on the same chunk grid (windowed and single-pass workspaces give identical bits), so the
comparison is exact: any difference would point at the windowing over the fixed array.  It sits in a
file of its own that pytest collects last.
"""
import pytest
import torch

import kda_linear_attention_02_b200 as kda
from kda_linear_attention_02_b200 import synth

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
            assert torch.equal(a, b), f"no-alloc call {call}: {name} differs from kda_chunk_fwd"


def test_noalloc_full_width_state_slices_over_windows():
    # 4 sequences x 32 heads = 128 chains: the state pass runs full 128-column slices (transposed products);
    # the packets (about 100 MB) exceed the 64 MiB array, so the call also runs window by window
    H, D, S = 32, 128, 512
    lengths = [700, 1300, 64, 513]
    assert kda.kda_chunk_fwd_workspace_bytes(sum(lengths), 4, H, D, D) > (64 << 20)
    inp = synth.make_inputs(lengths, H, D, D, dtype=BF, device=DEV, seed=23, with_state0=True)
    ckcu = kda.kda_ckpt_offsets(inp.cu_seqlens.cpu(), S)
    ckcu_d = ckcu.to(DEV)
    ref = _outputs(inp, H, D, ckcu)
    kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.state0, inp.cu_seqlens, ref[0], ref[1],
                      ckpt_stride=S, checkpoints=ref[2], ckpt_cu=ckcu_d, final_transition=ref[3])
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    got = _outputs(inp, H, D, ckcu)
    kda.kda_chunk_fwd_noalloc(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.state0, inp.cu_seqlens,
                              got[0], got[1], ckpt_stride=S, checkpoints=got[2], ckpt_cu=ckcu_d,
                              final_transition=got[3])
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    for name, a, b in zip(("o", "final_state", "checkpoints", "transition"), got, ref):
        assert torch.equal(a, b), f"no-alloc call: {name} differs from kda_chunk_fwd"


def test_noalloc_windows_over_the_fixed_array():
    # one 4096-token sequence at H=32: the full scratch (~172 MB of packets) exceeds the 64 MiB array while
    # its minimum (carried state + one chunk of packets) fits, so the call runs window by window and carries
    # the states across windows inside the array
    H, D, S = 32, 128, 512
    lengths = [4096]
    assert kda.kda_chunk_fwd_workspace_bytes(4096, 1, H, D, D) > (64 << 20)
    assert kda.kda_chunk_fwd_min_workspace_bytes(1, H, D, D) <= (64 << 20)
    inp = synth.make_inputs(lengths, H, D, D, dtype=BF, device=DEV, seed=22, with_state0=True)
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
            assert torch.equal(a, b), f"windowed no-alloc call {call}: {name} differs from kda_chunk_fwd"


def test_noalloc_refuses_batches_beyond_its_scratch():
    # 16 sequences x 32 heads need more than the fixed 64 MiB for their carried states alone
    H, D = 32, 128
    inp = synth.make_inputs([64] * 16, H, D, D, dtype=BF, device=DEV, seed=2)
    o = torch.empty(inp.total_tokens, H, D, dtype=BF, device=DEV)
    with pytest.raises(kda.KDAError) as e:
        kda.kda_chunk_fwd_noalloc(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, None, inp.cu_seqlens, o)
    assert e.value.status == -6      # KDA_ERR_WORKSPACE
