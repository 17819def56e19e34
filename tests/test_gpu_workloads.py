"""Full-size workloads on the GPU, checked against the fp64 oracle on sampled slices.

  * long-context prefill: B=1, T=1,048,576, H=32, dk=dv=128, bf16, log_alpha = -5 sigmoid(N(2,1)) (near
    the floor), random fp32 initial state ~ N(0, 0.02), fp32 checkpoints every 512 tokens;
  * decode: 256 sequences x 32 heads of 128 x 128 fp32 state, 1024 consecutive steps, with bf16 and with
    MXFP8 q, k, v;
  * varlen: 64 sequences with lengths uniform in [1024, 65536] (seed 1) packed by cu_seqlens,
    processed through a windowed workspace; half the sequences resumed from a checkpoint at a
    512-token boundary; every sequence split into 8 segments whose transitions and zero-start states
    are composed by kda_segment_compose.
"""
import gc

import pytest
import torch

import kda_linear_attention_02_b200 as kda
import oracle
from kda_linear_attention_02_b200 import synth
from kda_testlib import assert_close, f32np, oracle_slices
from test_gpu_basic import _Agg

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
DEV = "cuda:0"
BF = torch.bfloat16


@pytest.fixture(autouse=True)
def _clear_status():
    kda.kda_get_device_status()
    yield
    assert kda.kda_get_device_status() == 0, "a kernel recorded an error in the status word"
    gc.collect()
    torch.cuda.empty_cache()


def test_long_context_1m_tokens():
    T, H, D, S = 1 << 20, 32, 128, 512
    inp = synth.make_inputs([T], H, D, D, dtype=BF, device=DEV, seed=0, alpha_mu=2.0, alpha_sd=1.0,
                            with_state0=True)
    ckcu_h = kda.kda_ckpt_offsets(inp.cu_seqlens.cpu(), S)
    assert ckcu_h.tolist() == [0, T // S]
    ck = torch.empty(T // S, H, D, D, device=DEV)
    o = torch.empty(T, H, D, dtype=BF, device=DEV)
    fs = torch.empty(1, H, D, D, device=DEV)
    kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.state0, inp.cu_seqlens, o, fs,
                      ckpt_stride=S, checkpoints=ck, ckpt_cu=ckcu_h.to(DEV))
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    # sampled heads: outputs and checkpoints over a 64K-token prefix (they depend only on the prefix)
    P = 1 << 16
    heads = [0, 17, 31]
    res = oracle_slices(inp, [0], heads, marks_fn=lambda i, L: list(range(S, P + 1, S)),
                        tok_range=lambda i: (0, P))
    agg = _Agg(BF)
    for (i, h), r in res.items():
        agg.add("o", f32np(o[:P, h]), r["o"], f"o head {h}")
        for j in range(P // S):
            agg.add("ckpt", f32np(ck[j, h]), r["marks"][j], f"ckpt {j} head {h}")
    agg.check()
    # one head over the whole million tokens: final state and the last checkpoint
    r = oracle_slices(inp, [0], [5], want_o=False)[(0, 5)]
    assert_close(f32np(fs[0, 5]), r["state"], BF, "final state head 5 after 2^20 tokens")
    assert torch.equal(ck[-1], fs[0])            # stride divides the length: last checkpoint == final state
    assert torch.isfinite(o.float()).all()


def test_decode_256x32_1024_steps():
    n, H, D, steps = 256, 32, 128, 1024
    s0, q, k, v, la, b = synth.make_decode_inputs(n, H, D, D, dtype=BF, device=DEV, seed=3, steps=steps)
    state = s0.clone()
    pairs = [(0, 0), (13, 7), (255, 31), (128, 16), (77, 3), (200, 29)]
    outs = torch.empty(steps, len(pairs), D, dtype=BF, device=DEV)
    o = torch.empty(n, H, D, dtype=BF, device=DEV)
    idx_n = torch.tensor([p[0] for p in pairs], device=DEV)
    idx_h = torch.tensor([p[1] for p in pairs], device=DEV)
    for t_ in range(steps):
        kda.kda_recurrent_step(state, q[t_], k[t_], v[t_], la[t_], b[t_], o)
        outs[t_] = o[idx_n, idx_h]
    torch.cuda.synchronize()
    agg = _Agg(BF)
    for pi, (i, h) in enumerate(pairs):
        r = oracle.kda_seq(f32np(q[:, i, h]), f32np(k[:, i, h]), f32np(v[:, i, h]), f32np(la[:, i, h]),
                           f32np(b[:, i, h]), s0=s0[i, h].double().cpu().numpy())
        agg.add("o", f32np(outs[:, pi]), r["o"], f"decode o ({i},{h})")
        agg.add("state", f32np(state[i, h]), r["state"], f"decode state ({i},{h})")
    agg.check()
    assert torch.isfinite(state).all()


def test_decode_256x32_1024_steps_mxfp8():
    # the decode workload with MXFP8 q, k, v, as the benchmark times it; the oracle decodes the same bytes
    n, H, D, steps = 256, 32, 128, 1024
    s0, q, k, v, la, b = synth.make_decode_inputs(n, H, D, D, dtype=BF, device=DEV, seed=4, steps=steps)
    mx = (*synth.mxfp8_quantize(q), *synth.mxfp8_quantize(k), *synth.mxfp8_quantize(v))
    del q, k, v
    state = s0.clone()
    pairs = [(0, 0), (91, 12), (255, 31)]
    outs = torch.empty(steps, len(pairs), D, dtype=BF, device=DEV)
    o = torch.empty(n, H, D, dtype=BF, device=DEV)
    idx_n = torch.tensor([p[0] for p in pairs], device=DEV)
    idx_h = torch.tensor([p[1] for p in pairs], device=DEV)
    for t_ in range(steps):
        kda.kda_recurrent_step_mxfp8(state, *(x[t_] for x in mx), la[t_], b[t_], o)
        outs[t_] = o[idx_n, idx_h]
    torch.cuda.synchronize()
    agg = _Agg(BF)
    for pi, (i, h) in enumerate(pairs):
        dec = [oracle.mxfp8_decode(mx[j][:, i, h].cpu().numpy(), mx[j + 1][:, i, h].cpu().numpy()) for j in (0, 2, 4)]
        r = oracle.kda_seq(dec[0], dec[1], dec[2], f32np(la[:, i, h]), f32np(b[:, i, h]),
                           s0=s0[i, h].double().cpu().numpy())
        agg.add("o", f32np(outs[:, pi]), r["o"], f"MXFP8 decode o ({i},{h})")
        agg.add("state", f32np(state[i, h]), r["state"], f"MXFP8 decode state ({i},{h})")
    agg.check()
    assert torch.isfinite(state).all()


def test_varlen_resume_and_segments():
    H, D, S = 32, 128, 512
    lengths = synth.varlen_lengths(64, 1024, 65536, 1)
    N = len(lengths)
    inp = synth.make_inputs(lengths, H, D, D, dtype=BF, device=DEV, seed=0)
    T = inp.total_tokens
    cu = inp.cu_seqlens.cpu().tolist()
    ckcu_h = kda.kda_ckpt_offsets(cu, S)
    ck = torch.empty(int(ckcu_h[-1]), H, D, D, device=DEV)
    o = torch.empty(T, H, D, dtype=BF, device=DEV)
    fs = torch.empty(N, H, D, D, device=DEV)
    ws = torch.empty(16 << 30, dtype=torch.uint8, device=DEV)      # windowed: the full batch needs ~86 GB
    assert ws.numel() < kda.kda_chunk_fwd_workspace_bytes(T, N, H, D, D)
    kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, None, inp.cu_seqlens, o, fs,
                      ckpt_stride=S, checkpoints=ck, ckpt_cu=ckcu_h.to(DEV), workspace=ws)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0

    # segment boundaries (chunk aligned): b_s = 64 * floor(s * len / (8 * 64)), s = 0..7, b_8 = len
    seg_bounds = [[64 * ((s * L) // (8 * 64)) for s in range(8)] + [L] for L in lengths]
    sample = [0, 1, 30, 63]
    heads = [0, 21]

    def marks(i, L):
        m = set(range(S, L + 1, S)) | set(seg_bounds[i][1:8])
        return sorted(m)

    res = oracle_slices(inp, sample, heads, marks_fn=marks)
    agg = _Agg(BF)
    for (i, h), r in res.items():
        a, z = cu[i], cu[i + 1]
        mk = marks(i, z - a)
        agg.add("o", f32np(o[a:z, h]), r["o"], f"o seq {i} head {h}")
        agg.add("final", f32np(fs[i, h]), r["state"], f"final seq {i} head {h}")
        nck = (z - a) // S
        assert int(ckcu_h[i + 1] - ckcu_h[i]) == nck
        for j in range(nck):
            agg.add("ckpt", f32np(ck[int(ckcu_h[i]) + j, h]), r["marks"][mk.index((j + 1) * S)],
                    f"ckpt {j} seq {i}")
    agg.check()

    # prefix reuse: even sequences resume at b_i = 512 * floor(len_i / 1024) from the stored checkpoint
    even = list(range(0, N, 2))
    b_res = [S * (lengths[i] // 1024) for i in even]
    sub_len = [lengths[i] - b for i, b in zip(even, b_res)]
    rows = torch.cat([torch.arange(cu[i] + b, cu[i + 1], device=DEV) for i, b in zip(even, b_res)])
    init = torch.stack([ck[int(ckcu_h[i]) + b // S - 1] for i, b in zip(even, b_res)])
    sub = synth.KDAInputs(inp.q[rows].contiguous(), inp.k[rows].contiguous(), inp.v[rows].contiguous(),
                          inp.log_alpha[rows].contiguous(), inp.beta[rows].contiguous(),
                          synth.cu_from_lengths(sub_len, DEV), init.contiguous())
    o2 = torch.empty(sub.total_tokens, H, D, dtype=BF, device=DEV)
    fs2 = torch.empty(len(even), H, D, D, device=DEV)
    kda.kda_chunk_fwd(sub.q, sub.k, sub.v, sub.log_alpha, sub.beta, sub.state0, sub.cu_seqlens, o2, fs2,
                      workspace=ws)
    torch.cuda.synchronize()
    # the suffix chunk grid coincides with the unsplit run's: same arithmetic, bit for bit
    assert torch.equal(fs2, fs[even])
    assert torch.equal(o2, o[rows])
    del sub, o2, fs2, rows, init
    gc.collect()
    torch.cuda.empty_cache()

    # sequence split: 8 segments per sequence from a zero state with transitions, then the prefix scan
    seg_len = [bb[s + 1] - bb[s] for bb in seg_bounds for s in range(8)]
    assert min(seg_len) > 0
    seg_cu_tok = synth.cu_from_lengths(seg_len, DEV)
    Zs = torch.empty(len(seg_len), H, D, D, device=DEV)
    Ms = torch.empty(len(seg_len), H, D, D, device=DEV)
    kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, None, seg_cu_tok, o, Zs,
                      final_transition=Ms, workspace=ws)
    starts = torch.empty_like(Zs)
    ends = torch.empty(N, H, D, D, device=DEV)
    kda.kda_segment_compose(Ms, Zs, synth.cu_from_lengths([8] * N, DEV), None, starts, ends)
    torch.cuda.synchronize()
    agg = _Agg(BF)
    for (i, h), r in res.items():
        mk = marks(i, lengths[i])
        agg.add("end", f32np(ends[i, h]), r["state"], f"composed end seq {i} head {h}")
        for s in range(1, 8):
            agg.add("start", f32np(starts[8 * i + s, h]), r["marks"][mk.index(seg_bounds[i][s])],
                    f"segment {s} start seq {i} head {h}")
        assert not torch.any(torch.isnan(starts[8 * i, h]))
        assert torch.count_nonzero(starts[8 * i, h]) == 0          # zero initial state
    agg.check()
    # a plain sum of zero-start states is not the final state (the reason for the transitions)
    plain = Zs.view(N, 8, H, D, D).sum(1)
    rel = float((plain - fs).norm() / fs.norm())
    assert rel > 0.05
