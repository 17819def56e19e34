"""Sequence split across ranks (orkas.ai "Kimi K3 architecture" post, section "비용은 서빙 스택에서
돌아옵니다", sequence-split item).

KDA applies token-dependent transitions to its incoming state, so per-rank states computed from zero
cannot simply be summed.  Each rank's token segment is summarised by two composable quantities: its
cumulative transition M (dk x dk) and its final state from a zero start Z (dk x dv).  One fixed-size
all-gather of (M, Z) and an exclusive prefix scan X_{p+1} = M_p X_p + Z_p give every rank its start
state, and the rank then runs its segment from that state.  The all-gather moves H * dk * (dk + dv)
fp32 per rank (128 KiB per head at dk = dv = 128), independent of the sequence length.

All arithmetic runs in libkda's kernels (kda_chunk_fwd with the transition output, and
kda_segment_compose); this module only sequences the calls and the one collective.  The three steps
are also exposed one by one, so a caller can overlap the collective with other work.

Streams: every function takes an optional CUDA ``stream``.  When one is given, all of the function's
work -- the library calls, the small torch copies and concatenations around them, and the allocations
of its temporaries -- is issued on that stream, and the tensors it returns are ready in that stream's
order; a caller that reads them on another stream must make that stream wait first.
"""
from __future__ import annotations

import contextlib

import torch

from . import kda_chunk_fwd, kda_segment_compose


def _on(stream):
    """Issue everything inside on `stream` (torch ops, allocations, library calls), or on the current
    stream when it is None."""
    return contextlib.nullcontext() if stream is None else torch.cuda.stream(stream)


def segment_summary(q, k, v, log_alpha, beta, *, workspace=None, stream=None):
    """(M, Z) of one token segment [T, H, .] from a zero state: M [H, dk, dk], Z [H, dk, dv] fp32."""
    with _on(stream):
        return _segment_summary(q, k, v, log_alpha, beta, workspace)


def _segment_summary(q, k, v, log_alpha, beta, workspace):
    T, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    cu = torch.tensor([0, T], dtype=torch.int32, device=dev)
    scratch_o = torch.empty(T, H, dv, dtype=q.dtype, device=dev)   # outputs of the zero-start pass: unused
    M = torch.empty(1, H, dk, dk, dtype=torch.float32, device=dev)
    Z = torch.empty(1, H, dk, dv, dtype=torch.float32, device=dev)
    kda_chunk_fwd(q, k, v, log_alpha, beta, None, cu, scratch_o, Z, final_transition=M, workspace=workspace)
    return M[0], Z[0]


def gather_segment_summaries(M, Z, group=None, *, stream=None):
    """All-gather every rank's (M, Z), ordered by rank: ([W, H, dk, dk], [W, H, dk, dv])."""
    with _on(stream):
        return _gather(M, Z, group)


def _gather(M, Z, group):
    import torch.distributed as dist

    world = dist.get_world_size(group)
    dk = M.shape[-1]
    packed = torch.cat([M, Z], dim=-1).contiguous()                 # [H, dk, dk + dv]: one message
    H = packed.shape[0]
    # concatenated along the first dimension (the form every backend accepts), then viewed per rank
    out = torch.empty((world * H,) + tuple(packed.shape[1:]), dtype=packed.dtype, device=packed.device)
    dist.all_gather_into_tensor(out, packed, group=group)
    out = out.view((world,) + tuple(packed.shape))
    return out[..., :dk].contiguous(), out[..., dk:].contiguous()


def start_state(M_all, Z_all, rank, init=None, *, stream=None):
    """Start state of segment `rank` from the gathered summaries and the sequence's initial state
    ([H, dk, dv] or None for zero), by kda_segment_compose: [H, dk, dv] fp32."""
    with _on(stream):
        return _start_state(M_all, Z_all, rank, init)


def _start_state(M_all, Z_all, rank, init):
    W = M_all.shape[0]
    dev = Z_all.device
    seg_cu = torch.tensor([0, W], dtype=torch.int32, device=dev)
    starts = torch.empty_like(Z_all)
    kda_segment_compose(M_all, Z_all, seg_cu, None if init is None else init[None].contiguous(), starts)
    return starts[rank]


def sequence_split_prefill(q, k, v, log_alpha, beta, o, final_state=None, initial_state=None, *, group=None,
                           workspace=None, stream=None):
    """Chunked prefill of one sequence whose tokens are split across the ranks of `group`, each rank
    holding a contiguous segment [T_p, H, .] in rank order.  Writes this rank's outputs o [T_p, H, dv]
    and, when given, its segment's final state [H, dk, dv] (on the last rank: the sequence's final
    state).  initial_state [H, dk, dv] is the sequence's initial state (same on every rank) or None.
    With `stream`, every step (the collective included) is issued on it."""
    import torch.distributed as dist

    with _on(stream):
        rank = dist.get_rank(group)
        M, Z = _segment_summary(q, k, v, log_alpha, beta, workspace)
        M_all, Z_all = _gather(M, Z, group)
        X = _start_state(M_all, Z_all, rank, initial_state)
        T, H, dk = q.shape
        dv = v.shape[-1]
        cu = torch.tensor([0, T], dtype=torch.int32, device=q.device)
        fs = torch.empty(1, H, dk, dv, dtype=torch.float32, device=q.device)
        kda_chunk_fwd(q, k, v, log_alpha, beta, X[None].contiguous(), cu, o, fs, workspace=workspace)
        if final_state is not None:
            final_state.copy_(fs[0])
    return o
