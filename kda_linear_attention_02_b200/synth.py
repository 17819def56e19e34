"""Seeded synthetic inputs for the KDA operator (shared by the tests, the smoke check and the bench).

This module draws random numbers and nothing else: it holds none of the operator's arithmetic (the
decay floor, the recurrence and the chunk algebra live in the CUDA library and, independently, in the
oracle).  Both sides receive the same bytes.

Recipe (per workload, all draws from one ``torch.Generator`` seeded with ``seed`` on ``device``, in
the order q, k, v, beta-logits, alpha-logits, initial state):
  q, k        ~ N(0, 1), L2-normalised over the key dimension per (token, head) in fp32, then cast
  v           ~ N(0, 1), cast
  beta        = sigmoid(N(0, 1))                                      fp32 [tokens, H]
  log_alpha   = -5 * sigmoid(N(mu, sd))                              fp32 [tokens, H, dk]
                (mu, sd) = (0, 1.5) by default; (2, 1) for the long-context workload
  state0      ~ N(0, 0.02**2) (standard deviation 0.02) when asked   fp32 [N, H, dk, dv]
Varlen lengths: torch.randint(lo, hi + 1, (n,)) from a CPU generator seeded with ``len_seed``.
Large tensors are drawn in token slabs so that no fp32 temporary exceeds ``slab_bytes``.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass
class KDAInputs:
    q: torch.Tensor            # [T_tot, H, dk]
    k: torch.Tensor            # [T_tot, H, dk]
    v: torch.Tensor            # [T_tot, H, dv]
    log_alpha: torch.Tensor    # [T_tot, H, dk] fp32
    beta: torch.Tensor         # [T_tot, H] fp32
    cu_seqlens: torch.Tensor   # [N+1] int32 (same device)
    state0: torch.Tensor | None  # [N, H, dk, dv] fp32 or None

    @property
    def n_seqs(self) -> int:
        return self.cu_seqlens.numel() - 1

    @property
    def total_tokens(self) -> int:
        return self.q.shape[0]


def varlen_lengths(n: int, lo: int, hi: int, len_seed: int) -> list[int]:
    g = torch.Generator("cpu")
    g.manual_seed(len_seed)
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g)]


def cu_from_lengths(lengths, device="cpu") -> torch.Tensor:
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    return torch.tensor(cu, dtype=torch.int32, device=device)


def _draw(shape, gen, device, mean=0.0, std=1.0, slab_rows=None):
    out = torch.empty(shape, dtype=torch.float32, device=device)
    rows = shape[0]
    step = max(1, rows if slab_rows is None else slab_rows)
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        out[r0:r1].normal_(mean, std, generator=gen)
    return out


def make_inputs(lengths, H, dk, dv, *, dtype=torch.bfloat16, device="cpu", seed=0,
                alpha_mu=0.0, alpha_sd=1.5, with_state0=False, state_sd=0.02,
                slab_bytes=1 << 30) -> KDAInputs:
    """Draw one packed batch of KDA inputs; see the module docstring for the recipe."""
    T = int(sum(lengths))
    gen = torch.Generator(device)
    gen.manual_seed(seed)
    slab = max(1, slab_bytes // max(1, H * max(dk, dv) * 4))

    def unit_rows(x):
        # L2-normalise over the last dim slab by slab, in fp32
        for r0 in range(0, x.shape[0], slab):
            s = x[r0:r0 + slab]
            s.div_(s.norm(dim=-1, keepdim=True).clamp_min(1e-12))
        return x

    def cast(x):
        if dtype == torch.float32:
            return x
        out = torch.empty(x.shape, dtype=dtype, device=device)
        for r0 in range(0, x.shape[0], slab):
            out[r0:r0 + slab].copy_(x[r0:r0 + slab])
        return out

    q = cast(unit_rows(_draw((T, H, dk), gen, device, slab_rows=slab)))
    k = cast(unit_rows(_draw((T, H, dk), gen, device, slab_rows=slab)))
    v = cast(_draw((T, H, dv), gen, device, slab_rows=slab))
    beta = torch.sigmoid(_draw((T, H), gen, device))
    la = _draw((T, H, dk), gen, device, mean=alpha_mu, std=alpha_sd, slab_rows=slab)
    for r0 in range(0, T, slab):
        s = la[r0:r0 + slab]
        s.sigmoid_().mul_(-5.0)
    state0 = None
    if with_state0:
        state0 = _draw((len(lengths), H, dk, dv), gen, device, std=state_sd)
    return KDAInputs(q=q, k=k, v=v, log_alpha=la, beta=beta,
                     cu_seqlens=cu_from_lengths(lengths, device), state0=state0)


def make_decode_inputs(n, H, dk, dv, *, dtype=torch.bfloat16, device="cpu", seed=0,
                       steps=1, state_sd=0.02, alpha_mu=0.0, alpha_sd=1.5):
    """Decode workload: a state per (sequence, head) and ``steps`` single-token inputs.

    Returns (state0 [n,H,dk,dv] fp32, q,k [steps,n,H,dk], v [steps,n,H,dv], log_alpha [steps,n,H,dk],
    beta [steps,n,H]); same distributions as the prefill recipe, (mu, sd) = (0, 1.5) unless given.
    """
    gen = torch.Generator(device)
    gen.manual_seed(seed)
    q = _draw((steps, n, H, dk), gen, device)
    q = (q / q.norm(dim=-1, keepdim=True).clamp_min(1e-12)).to(dtype)
    k = _draw((steps, n, H, dk), gen, device)
    k = (k / k.norm(dim=-1, keepdim=True).clamp_min(1e-12)).to(dtype)
    v = _draw((steps, n, H, dv), gen, device).to(dtype)
    beta = torch.sigmoid(_draw((steps, n, H), gen, device))
    la = -5.0 * torch.sigmoid(_draw((steps, n, H, dk), gen, device, mean=alpha_mu, std=alpha_sd))
    state0 = _draw((n, H, dk, dv), gen, device, std=state_sd)
    return state0, q, k, v, la, beta


def draft_layout(x):
    """[n_draft, n, H, ...] per-step decode inputs -> the token-major draft layout [n * n_draft, H, ...]
    (sequence i's drafts at rows i * n_draft ..) of kda_decode_verify / kda_decode_commit."""
    return x.transpose(0, 1).contiguous().reshape(x.shape[0] * x.shape[1], *x.shape[2:])


def mxfp8_quantize(x: torch.Tensor, block: int = 32):
    """Quantise x [..., d] to MXFP8 for use as an input: (E4M3 codes uint8 [..., d], E8M0 scales uint8
    [..., d / block]).

    The scale choice is the one the OCP Microscaling Formats v1.0 specification suggests: per block of
    `block` consecutive elements, shared exponent floor(log2(amax)) - 8 (8 = largest exponent of E4M3),
    elements divided by 2^shared and rounded to E4M3, saturating at +-448.  An all-zero block gets scale
    1.0.  Rounding and the code bytes come from torch's float8 conversion.
    """
    xf = x.float()
    d = xf.shape[-1]
    if d % block:
        raise ValueError("the last axis must be a multiple of the block")
    xb = xf.reshape(*xf.shape[:-1], d // block, block)
    amax = xb.abs().amax(dim=-1)
    _, e = torch.frexp(amax)                   # amax = m 2^e, m in [0.5, 1): floor(log2 amax) = e - 1
    shared = torch.where(amax > 0, e - 1 - 8, torch.zeros_like(e)).clamp(-127, 127)
    elems = torch.ldexp(xb, -shared.unsqueeze(-1).to(xf.dtype)).clamp(-448.0, 448.0)
    codes = elems.to(torch.float8_e4m3fn).view(torch.uint8).reshape(xf.shape)
    scales = (shared + 127).to(torch.uint8)
    return codes.contiguous(), scales.contiguous()
