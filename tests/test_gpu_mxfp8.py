"""GPU parity of the MXFP8-input chunk path (kda_chunk_fwd_mxfp8) against the fp64 oracle.

q, k and v are quantised to MXFP8 (E4M3 codes, one E8M0 scale per 32 channels) by the input generator.
The oracle decodes the same bytes with its own MX decode and runs the sequential recurrence on the
decoded values.  The channels are skewed block by block before quantisation so that neighbouring
32-channel blocks get different shared scales: a scale applied to the wrong block fails the comparison.
Two properties hold at any size: the MXFP8 path equals the bf16 path run on the decoded values given as
bf16, bit for bit (the decode is exact); and adding a constant to every scale code of q and v scales the
outputs by the matching power of two, exactly.
"""
import numpy as np
import pytest
import torch

import kda_linear_attention_02_b200 as kda
import oracle
from kda_linear_attention_02_b200 import synth
from kda_testlib import f32np, oracle_slices
from test_gpu_basic import _Agg, _check_chunk, _run_chunk

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
BF = torch.bfloat16


@pytest.fixture(autouse=True)
def _clear_status():
    kda.kda_get_device_status()
    yield
    assert kda.kda_get_device_status() == 0, "a kernel recorded an error in the status word"


def _skew(x, factors):
    """Multiply 32-channel block b of the last axis by factors[b]."""
    f = torch.tensor(factors, dtype=torch.float32, device=x.device).repeat_interleave(32)
    return x.float() * f[: x.shape[-1]]


def _mx_inputs(lengths, H, dv, seed, skew=True, **kw):
    inp = synth.make_inputs(lengths, H, 128, dv, dtype=BF, device=DEV, seed=seed, **kw)
    q, k, v = inp.q.float(), inp.k.float(), inp.v.float()
    if skew:
        # different magnitudes per block with the inputs' overall scale kept: q and k stay unit vectors
        # and v keeps unit-order entries, so the outputs stay on the scale the absolute bound is set for
        q = _skew(q, [1.0, 4.0, 0.25, 2.0])
        q = q / q.norm(dim=-1, keepdim=True).clamp_min(1e-6)
        k = _skew(k, [1.0, 2.0, 4.0, 8.0])
        k = k / k.norm(dim=-1, keepdim=True).clamp_min(1e-6)
        v = _skew(v, [0.5, 1.0, 0.25, 0.125])
    mx = (*synth.mxfp8_quantize(q), *synth.mxfp8_quantize(k), *synth.mxfp8_quantize(v))
    if skew and inp.total_tokens:
        for sc in (mx[1], mx[3], mx[5]):
            assert bool((sc[..., 1:] != sc[..., :-1]).float().mean() > 0.5), "blocks should get different scales"
    return inp, mx


def _oracle_inputs(inp, mx):
    """The packed inputs with q, k, v replaced by the oracle's decode of the MXFP8 bytes (fp32, exact)."""
    qc, qs, kc, ks, vc, vs = (t.cpu().numpy() for t in mx)
    dec = [torch.from_numpy(oracle.mxfp8_decode(c, s).astype(np.float32)) for c, s in ((qc, qs), (kc, ks), (vc, vs))]
    return synth.KDAInputs(dec[0], dec[1], dec[2], inp.log_alpha.cpu(), inp.beta.cpu(), inp.cu_seqlens.cpu(),
                           None if inp.state0 is None else inp.state0.cpu())


def _torch_decoded_bf16(mx):
    """The decoded values as bf16 through torch's float8 conversions (exact), for the bf16 path."""
    out = []
    for c, s in ((mx[0], mx[1]), (mx[2], mx[3]), (mx[4], mx[5])):
        e = c.view(torch.float8_e4m3fn).float()
        x = s.view(torch.float8_e8m0fnu).float().repeat_interleave(32, dim=-1)
        out.append((e * x).to(BF).contiguous())
    return out


def _run_mx(inp, mx, *, ckpt_stride=0, transition=False, ws_bytes=None, init=True):
    T, H, dk = inp.q.shape
    dv = inp.v.shape[-1]
    n = inp.n_seqs
    o = torch.full((T, H, dv), float("nan"), dtype=BF, device=DEV)
    fs = torch.full((n, H, dk, dv), float("nan"), device=DEV)
    tr = torch.full((n, H, dk, dk), float("nan"), device=DEV) if transition else None
    ck = ckcu = None
    if ckpt_stride:
        ckcu_h = kda.kda_ckpt_offsets(inp.cu_seqlens.cpu(), ckpt_stride)
        ck = torch.full((max(1, int(ckcu_h[-1])), H, dk, dv), float("nan"), device=DEV)
        ckcu = ckcu_h.to(DEV)
    ws = None if ws_bytes is None else torch.empty(ws_bytes, dtype=torch.uint8, device=DEV)
    qc, qs, kc, ks, vc, vs = mx
    kda.kda_chunk_fwd_mxfp8(qc, qs, kc, ks, vc, vs, inp.log_alpha, inp.beta, inp.state0 if init else None,
                            inp.cu_seqlens, o, fs, ckpt_stride=ckpt_stride, checkpoints=ck, ckpt_cu=ckcu,
                            final_transition=tr, workspace=ws)
    torch.cuda.synchronize()
    return o, fs, ck, ckcu, tr


@pytest.mark.parametrize("dv", [128, 64])
def test_mxfp8_varlen_ragged(dv):
    lengths = [1, 63, 64, 65, 200, 0, 130, 16, 333]
    inp, mx = _mx_inputs(lengths, 3, dv, seed=21, with_state0=True)
    outs = _run_mx(inp, mx, ckpt_stride=64, transition=True)
    _check_chunk(_oracle_inputs(inp, mx), BF, outs, range(len(lengths)), [0, 1, 2], ckpt_stride=64,
                 transition=True)


@pytest.mark.parametrize("dv", [128, 64])
def test_mxfp8_equals_bf16_path_on_decoded_inputs(dv):
    lengths = [700, 1, 64, 129, 0, 333]
    inp, mx = _mx_inputs(lengths, 4, dv, seed=22, with_state0=True)
    a = _run_mx(inp, mx, ckpt_stride=128, transition=True)
    q, k, v = _torch_decoded_bf16(mx)
    dec = synth.KDAInputs(q, k, v, inp.log_alpha, inp.beta, inp.cu_seqlens, inp.state0)
    b = _run_chunk(dec, BF, ckpt_stride=128, transition=True)
    for x, y, what in zip(a, b, ("o", "final_state", "checkpoints", "ckpt_cu", "transition")):
        assert torch.equal(x, y), f"{what} differs from the bf16 path on the decoded inputs"


def test_mxfp8_scale_codes_scale_the_outputs_exactly():
    lengths = [300, 65]
    inp, mx = _mx_inputs(lengths, 2, 128, seed=23, with_state0=False)
    base = _run_mx(inp, mx, init=False)
    qc, qs, kc, ks, vc, vs = mx
    a, b = -9, 7   # q x 2^-9, v x 2^7: o x 2^-2, the state x 2^7
    assert int(qs.min()) + a >= 1 and int(vs.max()) + b <= 254
    moved = _run_mx(inp, (qc, (qs.int() + a).to(torch.uint8), kc, ks, vc, (vs.int() + b).to(torch.uint8)),
                    init=False)
    assert torch.equal(moved[0].float(), base[0].float() * 2.0 ** (a + b))
    assert torch.equal(moved[1], base[1] * 2.0 ** b)


def test_mxfp8_windows_are_bit_identical():
    lengths = [300, 5, 129, 64, 0, 700]
    N, H = len(lengths), 2
    inp, mx = _mx_inputs(lengths, H, 128, seed=24, with_state0=True)
    full = _run_mx(inp, mx, ckpt_stride=128, transition=True)
    ub = (inp.total_tokens + 63) // 64 + N
    index = ((N + 1) * 4 + 255) // 256 * 256
    pk = (kda.kda_chunk_fwd_workspace_bytes(inp.total_tokens, N, H, 128, 128, kda.KDA_MXFP8) - index) // (ub * H)
    small = kda.kda_chunk_fwd_min_workspace_bytes(N, H, 128, 128, kda.KDA_MXFP8) + 2 * H * pk
    win = _run_mx(inp, mx, ckpt_stride=128, transition=True, ws_bytes=small)
    for x, y in zip(full, win):
        assert torch.equal(x, y)


def test_mxfp8_prefill_workload_sampled():
    # the prefill workload (B=4, T=4096, H=32, dk=dv=128, checkpoints every 512) with MXFP8 q, k, v, in the
    # launch configuration the benchmark times; sampled (sequence, head) slices against the oracle
    lengths = [4096] * 4
    inp, mx = _mx_inputs(lengths, 32, 128, seed=0, skew=False)
    outs = _run_mx(inp, mx, ckpt_stride=512, init=False)
    o, fs, ck, ckcu, _ = outs
    dec = _oracle_inputs(inp, mx)
    seqs, heads = [0, 3], [0, 17, 31]
    res = oracle_slices(dec, seqs, heads, ckpt_stride=512, s0=None)
    cu = inp.cu_seqlens.cpu().tolist()
    ckcu = ckcu.cpu().tolist()
    agg = _Agg(BF)
    for (i, h), r in res.items():
        agg.add("o", f32np(o[cu[i]:cu[i + 1], h]), r["o"], f"o seq {i} head {h}")
        agg.add("final_state", f32np(fs[i, h]), r["state"], f"final state seq {i} head {h}")
        for j in range(len(r["marks"])):
            agg.add("checkpoints", f32np(ck[ckcu[i] + j, h]), r["marks"][j], f"ckpt {j} seq {i} head {h}")
    agg.check()


# ---------------------------------------------------------------------------- decode step with MXFP8 inputs

def _mx_decode_inputs(n, H, dk, dv, steps, seed):
    s0, q, k, v, la, b = synth.make_decode_inputs(n, H, dk, dv, dtype=BF, device=DEV, seed=seed, steps=steps)
    f = [0.5, 1.0, 0.25, 0.125]
    qs_ = _skew(q, [1.0, 4.0, 0.25, 2.0])
    qs_ = qs_ / qs_.norm(dim=-1, keepdim=True).clamp_min(1e-6)
    ks_ = _skew(k, [1.0, 2.0, 4.0, 8.0])
    ks_ = ks_ / ks_.norm(dim=-1, keepdim=True).clamp_min(1e-6)
    mx = (*synth.mxfp8_quantize(qs_), *synth.mxfp8_quantize(ks_), *synth.mxfp8_quantize(_skew(v, f)))
    return s0, mx, la, b


@pytest.mark.parametrize("dk,dv", [(128, 128), (128, 64), (64, 128), (64, 64)])
def test_mxfp8_decode_steps_vs_oracle(dk, dv):
    n, H, steps = 5, 3, 6
    s0, mx, la, b = _mx_decode_inputs(n, H, dk, dv, steps, seed=31)
    state = s0.clone()
    outs = []
    for t in range(steps):
        o = torch.full((n, H, dv), float("nan"), dtype=BF, device=DEV)
        kda.kda_recurrent_step_mxfp8(state, *(x[t] for x in mx), la[t], b[t], o)
        outs.append(o)
    torch.cuda.synchronize()
    dec = [oracle.mxfp8_decode(mx[j].cpu().numpy(), mx[j + 1].cpu().numpy()) for j in (0, 2, 4)]
    agg = _Agg(BF)
    for i in range(n):
        for h in range(H):
            r = oracle.kda_seq(dec[0][:, i, h], dec[1][:, i, h], dec[2][:, i, h], f32np(la[:, i, h]),
                               f32np(b[:, i, h]), s0=s0[i, h].double().cpu().numpy())
            o = np.stack([f32np(outs[t][i, h]) for t in range(steps)])
            agg.add("o", o, r["o"], f"decode o seq {i} head {h}", per_slice_rel=False)
            agg.add("state", f32np(state[i, h]), r["state"], f"decode state seq {i} head {h}")
    agg.check()


def test_mxfp8_decode_equals_bf16_decode_on_decoded_inputs():
    n, H, dk, dv, steps = 7, 4, 128, 128, 4
    s0, mx, la, b = _mx_decode_inputs(n, H, dk, dv, steps, seed=32)
    q, k, v = _torch_decoded_bf16(mx)
    sa, sb = s0.clone(), s0.clone()
    for t in range(steps):
        oa = torch.empty(n, H, dv, dtype=BF, device=DEV)
        ob = torch.empty(n, H, dv, dtype=BF, device=DEV)
        kda.kda_recurrent_step_mxfp8(sa, *(x[t] for x in mx), la[t], b[t], oa)
        kda.kda_recurrent_step(sb, q[t], k[t], v[t], la[t], b[t], ob)
        torch.cuda.synchronize()
        assert torch.equal(oa, ob), f"step {t}: o differs from the bf16 decode on the decoded inputs"
    assert torch.equal(sa, sb)


def test_mxfp8_nan_codes_read_as_nan():
    # OCP MX v1.0: the E4M3 codes S.1111.111 are NaN.  One such code in v of token 70, head 1 makes that
    # head's outputs NaN from the chunk holding it on (the chunk's products take 0 x NaN = NaN, and the state
    # carries it), in the chunk path and in the decode step; the other heads are unchanged
    lengths = [200]
    inp, mx = _mx_inputs(lengths, 3, 128, seed=41, skew=False, with_state0=True)
    base = _run_mx(inp, mx)
    vc = mx[4].clone()
    vc[70, 1, 5] = 0x7F
    bad = _run_mx(inp, (mx[0], mx[1], mx[2], mx[3], vc, mx[5]))
    assert torch.equal(bad[0][:, 0], base[0][:, 0]) and torch.equal(bad[0][:, 2], base[0][:, 2])
    assert torch.equal(bad[0][:64, 1], base[0][:64, 1])
    assert bool(torch.isnan(bad[0][64:, 1].float()).any(dim=-1).all()), "every output from token 64 on has a NaN"
    assert bool(torch.isnan(bad[1][0, 1]).any())
    n, H, steps = 3, 2, 2
    s0, dmx, la, b = _mx_decode_inputs(n, H, 128, 128, steps, seed=42)
    dvc = dmx[4].clone()
    dvc[0, 1, 0, 9] = 0xFF   # step 0, sequence 1, head 0
    state = s0.clone()
    o = torch.empty(n, H, 128, dtype=BF, device=DEV)
    kda.kda_recurrent_step_mxfp8(state, dmx[0][0], dmx[1][0], dmx[2][0], dmx[3][0], dvc[0], dmx[5][0], la[0], b[0], o)
    torch.cuda.synchronize()
    assert bool(torch.isnan(o[1, 0].float()).any()) and bool(torch.isnan(state[1, 0]).any())
    assert not bool(torch.isnan(o[0]).any()) and not bool(torch.isnan(state[0]).any())
