"""Prefix reuse end to end on the GPU.

A first prompt is prefilled with checkpoints every 512 tokens.  The checkpoints the prefix directory
plans for it are copied into a slot pool.  A second prompt sharing its first 5000 tokens looks up the
deepest checkpointed block end inside the shared prefix and resumes there from the slot's state.  Its
outputs and final state equal a full run of the second prompt bit for bit: the chunk grid of the resumed
run coincides with the full run's, so the arithmetic is the same.
"""
import numpy as np
import pytest
import torch

import kda_linear_attention_02_b200 as kda
from kda_linear_attention_02_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
BF = torch.bfloat16


def _cat(a, b, n_a):
    fields = []
    for x, y in zip((a.q, a.k, a.v, a.log_alpha, a.beta), (b.q, b.k, b.v, b.log_alpha, b.beta)):
        fields.append(torch.cat([x[:n_a], y]).contiguous())
    return fields


def _run(fields, init=None, ckpt=0):
    q, k, v, la, b = fields
    T, H, D = q.shape
    cu = synth.cu_from_lengths([T], DEV)
    o = torch.empty(T, H, D, dtype=BF, device=DEV)
    fs = torch.empty(1, H, D, D, device=DEV)
    ck = ckcu = None
    if ckpt:
        ckcu_h = kda.kda_ckpt_offsets([0, T], ckpt)
        ck = torch.empty(int(ckcu_h[-1]), H, D, D, device=DEV)
        ckcu = ckcu_h.to(DEV)
    kda.kda_chunk_fwd(q, k, v, la, b, init, cu, o, fs, ckpt_stride=ckpt, checkpoints=ck, ckpt_cu=ckcu)
    return o, fs, ck


def test_resume_from_looked_up_checkpoint_is_bit_exact():
    H, D, BLK = 4, 128, kda.KDA_PREFIX_BLOCK
    L1, shared, L2 = 6000, 5000, 7000
    rng = np.random.default_rng(0)
    tok1 = rng.integers(0, 150_000, size=L1, dtype=np.int32)
    tok2 = np.concatenate([tok1[:shared], rng.integers(0, 150_000, size=L2 - shared, dtype=np.int32)])
    in1 = synth.make_inputs([L1], H, D, D, dtype=BF, device=DEV, seed=0)
    tail = synth.make_inputs([L2 - shared], H, D, D, dtype=BF, device=DEV, seed=1)
    f1 = [in1.q, in1.k, in1.v, in1.log_alpha, in1.beta]
    f2 = _cat(in1, tail, shared)                     # the same projected inputs on the shared tokens

    # request 1: prefill with checkpoints every 512 tokens, then record its planned checkpoints
    _, _, ck1 = _run(f1, ckpt=BLK)
    cache = kda.kda_prefix_cache_create(1000, 8, 2)   # unit 2 blocks = 1024 tokens
    try:
        h1 = kda.kda_prefix_block_hashes(tok1)
        assert len(h1) == L1 // BLK
        assert kda.kda_prefix_cache_lookup(cache, h1) == (0, 0, -1)
        ends = kda.kda_prefix_cache_plan(cache, len(h1), 0)
        assert ends == [2, 4, 6, 8, 10, 11]
        slots = kda.kda_prefix_cache_insert(cache, h1, ends)
        pool = torch.empty(8, H, D, D, device=DEV)
        for e, s in zip(ends, slots):
            pool[s] = ck1[e - 1]                      # checkpoint j holds the state after (j + 1) * 512 tokens
        # the copies run on the current stream, before every later reader: the slots may be committed
        kda.kda_prefix_cache_commit(cache, slots)

        # request 2: 9 full blocks are shared; the deepest checkpoint inside them ends block 8
        h2 = kda.kda_prefix_block_hashes(tok2)
        m, r, s = kda.kda_prefix_cache_lookup(cache, h2)
        assert (m, r, s) == (shared // BLK, 8, slots[ends.index(8)])
        start = r * BLK
        o_sub, fs_sub, _ = _run([x[start:].contiguous() for x in f2], init=pool[s:s + 1].contiguous())
        o_full, fs_full, _ = _run(f2)
        torch.cuda.synchronize()
        assert kda.kda_get_device_status() == 0
        assert torch.equal(o_sub, o_full[start:])
        assert torch.equal(fs_sub, fs_full)
        kda.kda_prefix_cache_release(cache, s)        # the resumed prefill has read the slot
    finally:
        kda.kda_prefix_cache_destroy(cache)
