"""Decode continues a prefill: kda_chunk_fwd over the first T tokens of each sequence, then n
kda_recurrent_step calls from its final state, gives the outputs and final state of the oracle's run
over all T + n tokens (bf16 and fp32 inputs)."""
import numpy as np
import pytest
import torch

import kda_linear_attention_02_b200 as kda
from kda_linear_attention_02_b200 import synth
from kda_testlib import f32np, oracle_slices
from test_gpu_basic import _Agg, _run_chunk

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(autouse=True)
def _clear_status():
    kda.kda_get_device_status()
    yield
    assert kda.kda_get_device_status() == 0, "a kernel recorded an error in the status word"


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_prefill_then_decode_continues_the_sequence(dtype, d):
    T, n_dec, N, H = 200, 5, 2, 2
    inp = synth.make_inputs([T + n_dec] * N, H, d, d, dtype=dtype, device=DEV, seed=41, with_state0=True)
    cu = inp.cu_seqlens.cpu().tolist()
    rows = torch.cat([torch.arange(cu[i], cu[i] + T) for i in range(N)]).to(DEV)
    pre = synth.KDAInputs(*(x[rows].contiguous() for x in (inp.q, inp.k, inp.v, inp.log_alpha, inp.beta)),
                          synth.cu_from_lengths([T] * N, DEV), inp.state0)
    _, fs, _, _, _ = _run_chunk(pre, dtype)
    state = fs.clone()
    outs = []
    for j in range(n_dec):
        tok = torch.tensor([cu[i] + T + j for i in range(N)], device=DEV)
        o = torch.full((N, H, d), float("nan"), dtype=dtype, device=DEV)
        kda.kda_recurrent_step(state, *(x[tok].contiguous() for x in (inp.q, inp.k, inp.v, inp.log_alpha,
                                                                       inp.beta)), o)
        outs.append(o)
    torch.cuda.synchronize()
    res = oracle_slices(inp, range(N), range(H))
    agg = _Agg(dtype)
    for (i, h), r in res.items():
        o_dec = np.stack([f32np(outs[j][i, h]) for j in range(n_dec)])
        agg.add("o", o_dec, r["o"][T:], f"decoded o seq {i} head {h}", per_slice_rel=False)
        agg.add("state", f32np(state[i, h]), r["state"], f"state seq {i} head {h}")
    agg.check()
