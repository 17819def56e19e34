"""GPU parity of the bf16 tcgen05 chunk path against the fp64 oracle (through the C ABI).

Small ragged batches cover the edge cases (length 1, 63/64/65, empty sequences, a ragged last chunk,
several tiles, checkpoints, transitions, windows); the full-size workloads are checked on sampled
(sequence, head) slices that the oracle computes exactly.
"""
import math

import pytest
import torch

import kda_linear_attention_02_b200 as kda
from kda_linear_attention_02_b200 import synth
from test_gpu_basic import _check_chunk, _run_chunk

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
BF = torch.bfloat16


@pytest.fixture(autouse=True)
def _clear_status():
    kda.kda_get_device_status()
    yield
    assert kda.kda_get_device_status() == 0, "a kernel recorded an error in the status word"


@pytest.mark.parametrize("dv", [128, 64])
def test_bf16_varlen_ragged(dv):
    lengths = [1, 63, 64, 65, 200, 0, 130, 16, 333]
    inp = synth.make_inputs(lengths, 3, 128, dv, dtype=BF, device=DEV, seed=7, with_state0=True)
    outs = _run_chunk(inp, BF, ckpt_stride=64, transition=True)
    _check_chunk(inp, BF, outs, range(len(lengths)), [0, 1, 2], ckpt_stride=64, transition=True)


@pytest.mark.parametrize("n_seqs,H,dv", [(8, 8, 128), (16, 8, 64)])
def test_bf16_64_column_state_slices(n_seqs, H, dv):
    # 64 chains at dv = 128, or 128 chains at dv = 64: the state pass runs 64-column slices (the bench
    # workload runs 128-column slices, the small ragged batches 32-column ones)
    lengths = [97, 64, 130, 1, 200, 65, 150, 33] * (n_seqs // 8)
    inp = synth.make_inputs(lengths, H, 128, dv, dtype=BF, device=DEV, seed=13, with_state0=True)
    outs = _run_chunk(inp, BF, ckpt_stride=64, transition=True)
    _check_chunk(inp, BF, outs, range(0, n_seqs, 3), [0, H - 1], ckpt_stride=64, transition=True)


def test_bf16_128_column_transposed_state_pass():
    # 8 sequences x 16 heads = 128 chains: the state pass runs full 128-column slices with transposed
    # products (state columns on the M side); ragged last chunks leave through the staged O tile's rows
    lengths = [97, 64, 130, 1, 200, 65, 150, 33]
    H = 16
    inp = synth.make_inputs(lengths, H, 128, 128, dtype=BF, device=DEV, seed=21, with_state0=True)
    outs = _run_chunk(inp, BF, ckpt_stride=64, transition=True)
    _check_chunk(inp, BF, outs, range(0, 8, 3), [0, H - 1], ckpt_stride=64, transition=True)
    # one sequence alone (16 chains) runs 32-column slices with D1 = [-W; Q gamma] S: every output element
    # sums the same products in the same order, so the two forms agree bit for bit
    o, fs, ck, ckcu, tr = outs
    cu = inp.cu_seqlens.cpu().tolist()
    for i in (2, 4):
        a, b = cu[i], cu[i + 1]
        one = synth.KDAInputs(inp.q[a:b].contiguous(), inp.k[a:b].contiguous(), inp.v[a:b].contiguous(),
                              inp.log_alpha[a:b].contiguous(), inp.beta[a:b].contiguous(),
                              synth.cu_from_lengths([b - a], DEV), inp.state0[i:i + 1].contiguous())
        o1, fs1, ck1, _, tr1 = _run_chunk(one, BF, ckpt_stride=64, transition=True)
        assert torch.equal(o1, o[a:b]) and torch.equal(fs1[0], fs[i]) and torch.equal(tr1[0], tr[i])
        c0 = int(ckcu[i])
        assert torch.equal(ck1[: (b - a) // 64], ck[c0:c0 + (b - a) // 64])


def test_bf16_transposed_state_pass_with_empty_sequences():
    # 4 sequences x 32 heads = 128 chains (128-column slices): an empty sequence keeps its start state and
    # its transition is the identity; the others match the oracle
    lengths = [0, 200, 0, 65]
    H = 32
    inp = synth.make_inputs(lengths, H, 128, 128, dtype=BF, device=DEV, seed=24, with_state0=True)
    outs = _run_chunk(inp, BF, ckpt_stride=64, transition=True)
    o, fs, ck, ckcu, tr = outs
    for i in (0, 2):
        assert torch.equal(fs[i], inp.state0[i])
        assert torch.equal(tr[i], torch.eye(128, device=DEV).expand(H, 128, 128))
    _check_chunk(inp, BF, outs, [1, 3], [0, 17, H - 1], ckpt_stride=64, transition=True)


def test_bf16_zero_state_single_sequence():
    inp = synth.make_inputs([256], 2, 128, 128, dtype=BF, device=DEV, seed=0)
    outs = _run_chunk(inp, BF, init=False)
    _check_chunk(inp, BF, outs, [0], [0, 1])


@pytest.mark.parametrize("mu,sd", [(2.0, 1.0), (6.0, 0.5)])
def test_bf16_decay_near_and_at_the_floor(mu, sd):
    # (2, 1): the long-context distribution, mean ~ -4.2; (6, 0.5): sigmoid ~ 1, i.e. -5 per step,
    # just above ln 0.0067 = -5.0057, so a 16-token tile spans nearly the full e^80 range.
    lengths = [129, 64, 300]
    inp = synth.make_inputs(lengths, 2, 128, 128, dtype=BF, device=DEV, seed=8, alpha_mu=mu, alpha_sd=sd,
                            with_state0=True)
    outs = _run_chunk(inp, BF, ckpt_stride=128, transition=True)
    _check_chunk(inp, BF, outs, range(len(lengths)), [0, 1], ckpt_stride=128, transition=True)


@pytest.mark.parametrize("mu", [-6.0, -9.0])
def test_bf16_slow_decay_carries_state(mu):
    # log_alpha = -5 sigmoid(N(mu, 0.5)): about -0.012 (mu = -6) or -0.0006 (mu = -9) per step, so the state
    # is carried across many chunks (close to linear attention with the delta rule) and every output
    # depends on the inter-chunk pass, not only those of a chunk's first tokens
    lengths = [700, 129, 1000]
    inp = synth.make_inputs(lengths, 2, 128, 128, dtype=BF, device=DEV, seed=11, alpha_mu=mu, alpha_sd=0.5,
                            with_state0=True)
    outs = _run_chunk(inp, BF, ckpt_stride=128, transition=True)
    _check_chunk(inp, BF, outs, range(len(lengths)), [0, 1], ckpt_stride=128, transition=True)


def test_bf16_floor_clamps_below_floor_decay():
    # log_alpha far below the floor (-50, -inf) must behave exactly like ln 0.0067
    lengths = [200]
    inp = synth.make_inputs(lengths, 2, 128, 128, dtype=BF, device=DEV, seed=9, with_state0=True)
    la = inp.log_alpha.clone()
    la[:, :, ::3] = -50.0
    la[:, :, 1::7] = float("-inf")
    inp.log_alpha = la
    outs = _run_chunk(inp, BF)
    _check_chunk(inp, BF, outs, [0], [0, 1])
    ref_la = la.clamp_min(math.log(0.0067))
    inp2 = synth.KDAInputs(inp.q, inp.k, inp.v, ref_la.contiguous(), inp.beta, inp.cu_seqlens, inp.state0)
    outs2 = _run_chunk(inp2, BF)
    # fp32 nearest of ln 0.0067 is what the kernel clamps to; -inf/-50 -> identical bits
    assert torch.equal(outs[0], outs2[0]) and torch.equal(outs[1], outs2[1])


def test_bf16_windows_are_bit_identical():
    lengths = [300, 5, 129, 64, 0, 700]
    inp = synth.make_inputs(lengths, 2, 128, 128, dtype=BF, device=DEV, seed=6, with_state0=True)
    full = _run_chunk(inp, BF, ckpt_stride=128, transition=True)
    N, H = len(lengths), 2
    ub = (inp.total_tokens + 63) // 64 + N                     # chunk upper bound of the workspace formula
    index = ((N + 1) * 4 + 255) // 256 * 256
    pk = (kda.kda_chunk_fwd_workspace_bytes(inp.total_tokens, N, H, 128, 128, kda.KDA_BF16) - index) // (ub * H)
    small = kda.kda_chunk_fwd_min_workspace_bytes(N, H, 128, 128, kda.KDA_BF16) + 2 * H * pk   # 3-chunk windows
    win = _run_chunk(inp, BF, ckpt_stride=128, transition=True, ws_bytes=small)
    for a, b in zip(full, win):
        if a is not None and a.dtype != torch.int32:
            assert torch.equal(a, b)


def test_bf16_transposed_state_pass_windows_are_bit_identical():
    # 8 sequences x 16 heads = 128 chains run 128-column slices with S^T in tensor memory; over 3-chunk
    # windows the state, the transition columns and the checkpoints pass from window to window through the
    # carry, in the transposed layout, and must give what one window gives
    lengths = [300, 5, 129, 64, 0, 700, 191, 1]
    N, H = len(lengths), 16
    inp = synth.make_inputs(lengths, H, 128, 128, dtype=BF, device=DEV, seed=23, with_state0=True)
    full = _run_chunk(inp, BF, ckpt_stride=128, transition=True)
    ub = (inp.total_tokens + 63) // 64 + N
    index = ((N + 1) * 4 + 255) // 256 * 256
    pk = (kda.kda_chunk_fwd_workspace_bytes(inp.total_tokens, N, H, 128, 128, kda.KDA_BF16) - index) // (ub * H)
    small = kda.kda_chunk_fwd_min_workspace_bytes(N, H, 128, 128, kda.KDA_BF16) + 2 * H * pk
    win = _run_chunk(inp, BF, ckpt_stride=128, transition=True, ws_bytes=small)
    for a, b in zip(full, win):
        if a is not None and a.dtype != torch.int32:
            assert torch.equal(a, b)
    _check_chunk(inp, BF, win, [0, 2, 5, 6, 7], [0, 9, H - 1], ckpt_stride=128, transition=True)
    assert kda.kda_get_device_status() == 0


def test_bf16_resume_from_checkpoint_matches_unsplit():
    # prefix reuse: run [0, len), take the checkpoint at b (a 512 boundary), run [b, len) from it
    lengths = [1536 + 77]
    inp = synth.make_inputs(lengths, 2, 128, 128, dtype=BF, device=DEV, seed=12, with_state0=True)
    o, fs, ck, ckcu, _ = _run_chunk(inp, BF, ckpt_stride=512)
    b = 1024
    sub = synth.KDAInputs(inp.q[b:].contiguous(), inp.k[b:].contiguous(), inp.v[b:].contiguous(),
                          inp.log_alpha[b:].contiguous(), inp.beta[b:].contiguous(),
                          synth.cu_from_lengths([lengths[0] - b], DEV), ck[1:2].contiguous())
    o2, fs2, *_ = _run_chunk(sub, BF)
    # same chunk grid and the same fp32 state -> the same arithmetic, bit for bit
    assert torch.equal(o2, o[b:]) and torch.equal(fs2, fs)


def test_bf16_empty_and_zero_token_batches():
    inp = synth.make_inputs([0, 0], 2, 128, 128, dtype=BF, device=DEV, seed=1, with_state0=True)
    o = torch.empty(0, 2, 128, dtype=BF, device=DEV)
    fs = torch.full((2, 2, 128, 128), float("nan"), device=DEV)
    tr = torch.full((2, 2, 128, 128), float("nan"), device=DEV)
    q = torch.empty(0, 2, 128, dtype=BF, device=DEV)
    kda.kda_chunk_fwd(q, q, q, torch.empty(0, 2, 128, device=DEV), torch.empty(0, 2, device=DEV), inp.state0,
                      inp.cu_seqlens, o, fs, final_transition=tr)
    torch.cuda.synchronize()
    assert torch.equal(fs, inp.state0)
    assert torch.equal(tr, torch.eye(128, device=DEV).expand(2, 2, 128, 128))


@pytest.mark.slow
def test_bf16_prefill_b4_t4096_h32_every_slice():
    # KDA prefill, B=4, T=4096, H=32, dk=dv=128, bf16, zero initial state, seed 0, fp32 checkpoints every
    # 512 tokens: the launch the benchmark times.  Every one of the 128 (sequence, head) slices -- outputs,
    # checkpoints and final states -- against the oracle (about a second of fp64 work on the host).
    inp = synth.make_inputs([4096] * 4, 32, 128, 128, dtype=BF, device=DEV, seed=0)
    outs = _run_chunk(inp, BF, init=False, ckpt_stride=512)
    _check_chunk(inp, BF, outs, range(4), range(32), ckpt_stride=512)
    o = outs[0]
    assert torch.isfinite(o.float()).all()
