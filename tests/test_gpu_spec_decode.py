"""Speculative decoding on the GPU: kda_decode_verify (outputs of every draft, state untouched) and
kda_decode_commit (state after the accepted prefix).

Pins: bit-for-bit equality with consecutive kda_recurrent_step calls on the same inputs (same per-token
arithmetic), and the fp64 oracle's sequential recurrence on sampled (sequence, head) pairs.
"""
import pytest
import torch

import kda_linear_attention_02_b200 as kda
import oracle
from kda_linear_attention_02_b200 import synth
from kda_testlib import f32np
from test_gpu_basic import _Agg

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
BF = torch.bfloat16


@pytest.fixture(autouse=True)
def _clear_status():
    kda.kda_get_device_status()
    yield


def _inputs(n, H, dk, dv, n_draft, dtype, seed):
    s0, q, k, v, la, b = synth.make_decode_inputs(n, H, dk, dv, dtype=dtype, device=DEV, seed=seed, steps=n_draft)
    return s0, (q, k, v, la, b)


def _sequential(s0, steps_in, n_steps):
    """Consecutive single decode steps: outputs [n_steps, n, H, dv] and the states after 0..n_steps steps."""
    q, k, v, la, b = steps_in
    st = s0.clone()
    outs, snaps = [], [st.clone()]
    for d in range(n_steps):
        o = torch.empty_like(v[d])
        kda.kda_recurrent_step(st, q[d], k[d], v[d], la[d], b[d], o)
        outs.append(o)
        snaps.append(st.clone())
    return torch.stack(outs), snaps


@pytest.mark.parametrize("dtype,dk,dv", [(BF, 128, 128), (torch.float32, 128, 128), (torch.float32, 64, 128),
                                         (torch.float32, 128, 64), (BF, 64, 64)])
def test_verify_and_commit_equal_sequential_steps(dtype, dk, dv):
    n, H, nd = 6, 3, 4
    s0, steps_in = _inputs(n, H, dk, dv, nd, dtype, seed=11)
    q, k, v, la, b = (synth.draft_layout(x) for x in steps_in)
    ref_o, snaps = _sequential(s0, steps_in, nd)

    state = s0.clone()
    o = torch.empty(n * nd, H, dv, dtype=dtype, device=DEV)
    kda.kda_decode_verify(state, q, k, v, la, b, o)
    torch.cuda.synchronize()
    assert torch.equal(state, s0), "verify must not write the state"
    assert torch.equal(o.view(n, nd, H, dv).transpose(0, 1), ref_o)

    acc = [0, 1, 4, 2, 3, 4]
    kda.kda_decode_commit(state, k, v, la, b, torch.tensor(acc, dtype=torch.int32, device=DEV))
    assert kda.kda_get_device_status() == 0
    for i, a in enumerate(acc):
        assert torch.equal(state[i], snaps[a][i]), f"sequence {i}, {a} accepted"


def _unaligned(x):
    """The same values one element past a 16-byte boundary (element-aligned, not 16-byte aligned)."""
    buf = torch.empty(x.numel() + 1, dtype=x.dtype, device=x.device)
    y = buf[1:].view(x.shape)
    y.copy_(x)
    return y


@pytest.mark.parametrize("nd,unaligned", [(6, False), (4, True), (7, True)])
def test_verify_and_commit_more_drafts_and_unaligned_inputs(nd, unaligned):
    # the first four drafts' inputs are copied to shared memory when q, k, v and log_alpha are 16-byte
    # aligned; later drafts, and every draft of unaligned inputs, are loaded element by element
    n, H, d = 5, 2, 128
    s0, steps_in = _inputs(n, H, d, d, nd, BF, seed=17 + nd)
    q, k, v, la, b = (synth.draft_layout(x) for x in steps_in)
    if unaligned:
        q, k, v, la = (_unaligned(x) for x in (q, k, v, la))
        assert all(x.data_ptr() % 16 != 0 for x in (q, k, v, la))
    ref_o, snaps = _sequential(s0, steps_in, nd)
    state = s0.clone()
    o = torch.empty(n * nd, H, d, dtype=BF, device=DEV)
    kda.kda_decode_verify(state, q, k, v, la, b, o)
    torch.cuda.synchronize()
    assert torch.equal(state, s0)
    assert torch.equal(o.view(n, nd, H, d).transpose(0, 1), ref_o)
    acc = [nd, 0, 1, nd - 1, min(5, nd)][:n]
    kda.kda_decode_commit(state, k, v, la, b, torch.tensor(acc, dtype=torch.int32, device=DEV))
    assert kda.kda_get_device_status() == 0
    for i, a in enumerate(acc):
        assert torch.equal(state[i], snaps[a][i]), f"sequence {i}, {a} accepted"


def test_single_draft_is_one_decode_step():
    n, H, d = 4, 2, 128
    s0, steps_in = _inputs(n, H, d, d, 1, BF, seed=5)
    q, k, v, la, b = (synth.draft_layout(x) for x in steps_in)
    ref_o, snaps = _sequential(s0, steps_in, 1)
    state = s0.clone()
    o = torch.empty(n, H, d, dtype=BF, device=DEV)
    kda.kda_decode_verify(state, q, k, v, la, b, o)
    assert torch.equal(o, ref_o[0])
    kda.kda_decode_commit(state, k, v, la, b, torch.ones(n, dtype=torch.int32, device=DEV))
    assert torch.equal(state, snaps[1])


@pytest.mark.parametrize("dtype", [BF, torch.float32])
def test_verify_and_commit_against_oracle(dtype):
    n, H, d, nd = 8, 4, 128, 6
    s0, steps_in = _inputs(n, H, d, d, nd, dtype, seed=2)
    q, k, v, la, b = (synth.draft_layout(x) for x in steps_in)
    state = s0.clone()
    o = torch.empty(n * nd, H, d, dtype=dtype, device=DEV)
    kda.kda_decode_verify(state, q, k, v, la, b, o)
    acc = [nd, 0, 3, 1, 5, 2, nd, 4]
    kda.kda_decode_commit(state, k, v, la, b, torch.tensor(acc, dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    agg = _Agg(dtype)
    o4 = o.view(n, nd, H, d)
    for i, h in [(0, 0), (1, 3), (2, 1), (4, 2), (6, 3), (7, 0)]:
        rows = slice(i * nd, (i + 1) * nd)
        r = oracle.kda_seq(f32np(q[rows, h]), f32np(k[rows, h]), f32np(v[rows, h]), f32np(la[rows, h]),
                           f32np(b[rows, h]), s0=s0[i, h].double().cpu().numpy(), marks=list(range(1, nd + 1)))
        agg.add("o", f32np(o4[i, :, h]), r["o"], f"draft outputs ({i},{h})")
        want = s0[i, h].double().cpu().numpy() if acc[i] == 0 else r["marks"][acc[i] - 1]
        agg.add("state", f32np(state[i, h]), want, f"committed state ({i},{h}), {acc[i]} accepted")
    agg.check()


def test_out_of_range_accept_count_is_reported_and_leaves_state():
    n, H, d, nd = 4, 2, 128, 4
    s0, steps_in = _inputs(n, H, d, d, nd, BF, seed=7)
    q, k, v, la, b = (synth.draft_layout(x) for x in steps_in)
    _, snaps = _sequential(s0, steps_in, nd)
    state = s0.clone()
    kda.kda_decode_commit(state, k, v, la, b, torch.tensor([2, -1, nd + 1, 0], dtype=torch.int32, device=DEV))
    assert kda.kda_get_device_status() == -7
    assert torch.equal(state[0], snaps[2][0])
    assert torch.equal(state[1:], s0[1:])
