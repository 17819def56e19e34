"""Shared helpers for the tests: parity metrics and oracle runs on slices of packed inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle

# Tolerances (whole tensor, fp64 accumulation of the error norms).
BF16_REL_FRO = 1e-2      # relative Frobenius error, bf16 inputs with fp32 accumulation
BF16_MAX_ABS = 5e-2      # max absolute error, bf16
F32_REL_FRO = 1e-4       # relative Frobenius error, fp32 inputs
F32_MAX_ABS = 5e-4       # max absolute error, fp32


def tol(dtype):
    return (BF16_REL_FRO, BF16_MAX_ABS) if dtype == torch.bfloat16 else (F32_REL_FRO, F32_MAX_ABS)


# Denominator floor of the relative Frobenius error.  A reference whose norm is below this is made of
# values under fp32's normal range (e.g. the transition of a long, strongly decaying sequence, ~1e-68)
# that no fp32 result can represent; there the error is taken in absolute terms.
REL_FLOOR = 1e-30


def rel_fro(x, ref) -> float:
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    den = max(float(np.linalg.norm(ref)), REL_FLOOR)
    return float(np.linalg.norm(x - ref) / den)


def max_abs(x, ref) -> float:
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.max(np.abs(x - ref))) if x.size else 0.0


def assert_close(x, ref, dtype, what):
    rf, ma = tol(dtype)
    r, m = rel_fro(x, ref), max_abs(x, ref)
    assert np.all(np.isfinite(np.asarray(x, np.float64))), f"{what}: non-finite values"
    assert r <= rf and m <= ma, f"{what}: rel_fro={r:.3e} (<= {rf}) max_abs={m:.3e} (<= {ma})"
    return r, m


def f32np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def oracle_slices(inp, seqs, heads, *, ckpt_stride=0, marks_fn=None, want_transition=False, want_o=True,
                  s0=None, tok_range=None):
    """Run the oracle on (sequence, head) slices of a packed KDAInputs (tensors may live on the GPU).

    Returns {(i, h): result-dict}.  marks_fn(i, length) -> list of token counts (overrides the
    checkpoint marks).  tok_range(i) -> (a, b) restricts sequence i to tokens [a, b) of it.
    s0: [N,H,dk,dv] tensor or None (defaults to inp.state0).
    """
    cu = inp.cu_seqlens.cpu().tolist()
    s0 = inp.state0 if s0 is None else s0
    jobs = []
    for i in seqs:
        a, b = cu[i], cu[i + 1]
        if tok_range is not None:
            ra, rb = tok_range(i)
            a, b = a + ra, a + rb
        L = b - a
        for h in heads:
            kw = dict(q=f32np(inp.q[a:b, h]), k=f32np(inp.k[a:b, h]), v=f32np(inp.v[a:b, h]),
                      log_alpha=f32np(inp.log_alpha[a:b, h]), beta=f32np(inp.beta[a:b, h]),
                      s0=None if s0 is None else s0[i, h].double().cpu().numpy(),
                      want_o=want_o, want_transition=want_transition)
            if marks_fn is not None:
                kw["marks"] = marks_fn(i, L)
            elif ckpt_stride:
                kw["marks"] = [j * ckpt_stride for j in range(1, L // ckpt_stride + 1)]
            jobs.append(((i, h), kw))
    return oracle.run_slices(jobs)
