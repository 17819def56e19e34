#!/usr/bin/env python
"""bench.py -- KDA operator throughput on B200: chunked prefill tokens/s (headline) and recurrent
decode steps/s, each against its HBM roofline, plus end-to-end and CPU-oracle baselines.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One timed step = one kda_chunk_fwd call over the prefill workload (B=4 sequences x T=4096 tokens,
H=32 heads, dk=dv=128, bf16 q/k/v, fp32 log_alpha/beta, zero initial state, fp32 final state and
fp32 state checkpoints every 512 tokens): the per-chunk decay prep, the intra-chunk tcgen05 pass,
the inter-chunk tcgen05 state pass and the checkpoint writes.  The decode workload (256 sequences x
32 heads of 128 x 128 fp32 state, 1024 consecutive kda_recurrent_step calls) and a segment compose
are timed alongside and reported under "decode" and "compose", with speculative decoding under
"speculative" and the prefill with MXFP8 q/k/v under "mxfp8".  Inputs are seeded synthetic data
drawn on the device; every input and output set is larger than the 126 MB L2, so no flush is needed.

Under torchrun (N > 1) every rank runs its own batch on its own GPU (weak scaling, no data-path
collective); the step time is the max over ranks (one NCCL all-reduce of a scalar outside the timed
region).  --impl reference times the fp64 CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "KDA prefill tokens/s (H=32,d=128,bf16) & decode steps/s; % of TC/HBM roofline"
B, T, H, D = 4, 4096, 32, 128
CKPT = 512
DEC_N, DEC_STEPS = 256, 1024
SPEC_ND, SPEC_POOL, SPEC_ROUNDS = 4, 16, 256   # drafts per round, distinct draft sets, timed rounds
# Algorithmic bytes per (token, head) of the prefill path.  Reads: q, k, v bf16 (3 x 256 B),
# log_alpha fp32 (512 B), beta fp32 (4 B).  Writes: o bf16 (256 B), the 512-token checkpoint
# (128 x 128 x 4 B / 512 = 128 B) and the final state (64 KiB per 4096 tokens = 16 B).
PREFILL_READ_B = 3 * 256 + 512 + 4
PREFILL_WRITE_B = 256 + 128 + 16
# The same with MXFP8 q, k, v: 1-byte E4M3 codes plus one E8M0 scale byte per 32 channels.
PREFILL_READ_MX_B = 3 * 128 + 3 * 4 + 512 + 4
# Decode bytes per (sequence, head) step: state read + write (2 x 64 KiB), q/k/v bf16, log_alpha,
# beta, o bf16.
DECODE_B = 2 * D * D * 4 + 3 * D * 2 + D * 4 + 4 + D * 2
DECODE_MX_B = 2 * D * D * 4 + 3 * D + 3 * D // 32 + D * 4 + 4 + D * 2


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), float(j.get("bf16_tflops_sustained", j["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


class Clocks:
    """nvidia-smi sampler (read-only queries) running while the measured work runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.path = tempfile.mktemp(prefix="kda_clocks_", suffix=".csv")
        self.f = open(self.path, "w")
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                       "-lms", "100", "-i", str(index)], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    def stop(self):
        if self.p is not None:
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except Exception:
                self.p.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            c = [x.strip() for x in line.split(",")]
            if len(c) < 9:
                continue
            try:
                sm.append(float(c[1]))
                mx.append(float(c[2]))
            except ValueError:
                continue
            for n, v in zip(names, c[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def captured_traffic(kernel):
    """DRAM bytes per launch of `kernel` from the committed ncu summary (profiles/traffic.txt), or None
    when the kernel's sources changed since that capture (their SHA-256 no longer matches)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    srcs = [os.path.join(ROOT, "kda_linear_attention_02_b200", "csrc", f) for f in ("kda_chunk_bf16.cu", "kda_device.cuh")]
    digest = hashlib.sha256()
    for f in srcs:
        with open(f, "rb") as fh:
            digest.update(fh.read())
    now = digest.hexdigest()[:16]
    for line in open(path):
        parts = line.split()
        if len(parts) == 3 and not line.startswith("#") and parts[0] == kernel:
            return int(parts[1]) if parts[2] == now else None
    return None


def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def max_over_ranks(x, world, device="cuda"):
    """Largest value of x over the ranks (the slowest rank's time), one all-reduce."""
    import torch
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def cpu_oracle_sample(inp, budget_s=12.0, max_slices=None, ckpt=CKPT):
    """Times the fp64 oracle (as it stands) on whole (sequence, head) slices of the workload,
    as many as fit the time budget (estimated from one calibration slice).  Like the GPU step it
    produces the outputs, the final state and the state after every `ckpt` tokens (0 = none)."""
    import oracle
    cu = inp.cu_seqlens.cpu().tolist()
    nseq = len(cu) - 1
    Hh = inp.q.shape[1]

    def job(i, h):
        a, b = cu[i], cu[i + 1]
        f = lambda t: t.float().cpu().numpy()
        marks = list(range(ckpt, b - a + 1, ckpt)) if ckpt else None
        s0 = None if inp.state0 is None else inp.state0[i, h].double().cpu().numpy()
        return dict(q=f(inp.q[a:b, h]), k=f(inp.k[a:b, h]), v=f(inp.v[a:b, h]),
                    log_alpha=f(inp.log_alpha[a:b, h]), beta=f(inp.beta[a:b, h]), s0=s0, marks=marks,
                    want_o=True)

    threads = oracle.threads_used()
    t0 = time.perf_counter()
    oracle.kda_seq(**job(0, 0))
    one = time.perf_counter() - t0
    n = max(1, min(nseq * Hh, int(budget_s * threads / max(one, 1e-3))))
    if max_slices:
        n = min(n, max_slices)
    keys = [(i, h) for i in range(nseq) for h in range(Hh)][:n]
    jobs = [(key, job(*key)) for key in keys]
    t0 = time.perf_counter()
    oracle.run_slices(jobs, threads)
    dt = time.perf_counter() - t0
    toks = sum(cu[i + 1] - cu[i] for i, _ in keys)
    return {"value": toks / Hh / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} of {nseq * Hh} (sequence, head) slices x {cu[1] - cu[0]} tokens, fp64, "
                      f"{dt:.1f} s on {threads} threads; tokens/s = token-heads/s / {Hh}"}


def cpu_oracle_decode_sample(s0, q, k, v, la, b, budget_s=6.0, max_slices=512):
    """Times the fp64 oracle (as it stands) on the decode workload: whole (sequence, head) slices, each
    one head's state carried through all the steps, as many as fit the time budget; steps/s of the whole
    workload is extrapolated from the sample.  q, k, v, la: [steps, n, H, d]; b: [steps, n, H]."""
    import oracle
    steps, n, Hh = b.shape

    def job(i, h):
        f = lambda t: t.float().cpu().numpy()
        return dict(q=f(q[:, i, h]), k=f(k[:, i, h]), v=f(v[:, i, h]), log_alpha=f(la[:, i, h]), beta=f(b[:, i, h]),
                    s0=s0[i, h].double().cpu().numpy(), want_o=True)

    threads = oracle.threads_used()
    t0 = time.perf_counter()
    oracle.kda_seq(**job(0, 0))
    one = time.perf_counter() - t0
    m = max(1, min(n * Hh, max_slices, int(budget_s * threads / max(one, 1e-3))))
    keys = [(i, h) for i in range(n) for h in range(Hh)][:m]
    jobs = [(key, job(*key)) for key in keys]
    t0 = time.perf_counter()
    oracle.run_slices(jobs, threads)
    dt = time.perf_counter() - t0
    whole_s = dt * (n * Hh) / m
    return {"value": steps / whole_s, "unit": "steps/s", "cores": threads, "kind": "oracle",
            "sample": f"{m} of {n * Hh} (sequence, head) slices x {steps} steps, fp64, {dt:.1f} s on {threads} "
                      f"threads; steps/s of the whole workload extrapolated from the sample"}


def host_slices(inp, keys, ckpt=0, tok_limit=None):
    """Host copies of whole (sequence, head) slices of a device workload, as oracle jobs (taken before
    the device inputs are freed, timed later).  tok_limit keeps only each slice's first tokens."""
    cu = inp.cu_seqlens.cpu().tolist()
    jobs = []
    for i, h in keys:
        a, b = cu[i], cu[i + 1]
        if tok_limit is not None:
            b = min(b, a + tok_limit)
        f = lambda t: t.float().cpu().numpy()
        marks = list(range(ckpt, b - a + 1, ckpt)) if ckpt else None
        s0 = None if inp.state0 is None else inp.state0[i, h].double().cpu().numpy()
        jobs.append(((i, h), dict(q=f(inp.q[a:b, h]), k=f(inp.k[a:b, h]), v=f(inp.v[a:b, h]),
                                  log_alpha=f(inp.log_alpha[a:b, h]), beta=f(inp.beta[a:b, h]), s0=s0,
                                  marks=marks, want_o=True)))
    return jobs


def cpu_oracle_jobs(jobs, heads, total_token_heads, what):
    """Times the fp64 oracle (as it stands) on prepared slice jobs and extrapolates the workload's
    tokens/s (token-heads/s of the sample / heads)."""
    import oracle
    threads = oracle.threads_used()
    t0 = time.perf_counter()
    oracle.run_slices(jobs, threads)
    dt = time.perf_counter() - t0
    th = sum(j[1]["q"].shape[0] for j in jobs)
    return {"value": th / dt / heads, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{what}: {len(jobs)} (sequence, head) slices, {th} token-heads of {total_token_heads} "
                      f"({100.0 * th / total_token_heads:.3g} %), fp64, {dt:.1f} s on {threads} threads; "
                      f"tokens/s = token-heads/s / {heads}, extrapolated from the sample"}


def timed_calls(fn, steps, warmup, stream):
    """Average device time (ms) of `steps` calls of fn after `warmup` calls, CUDA events on `stream`."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def prefill_roofline(token_heads, ms, hbm, extra_bytes=0, read_b=PREFILL_READ_B, out_b=256):
    """HBM roofline of one chunked-prefill call: q, k, v, log_alpha, beta in, o out (per token-head),
    plus `extra_bytes` (checkpoints, initial and final states) per call."""
    alg = (read_b + out_b) * token_heads + extra_bytes
    gbs = alg / (ms / 1e3) / 1e9
    return {"bound": "hbm", "kernel": "kda_chunk_fwd (whole call)", "achieved": round(gbs, 1), "peak": hbm,
            "unit": "GB/s", "frac": round(gbs / hbm, 4), "alg_bytes_per_launch": int(alg),
            "ideal_ms": round(alg / (hbm * 1e9) * 1e3, 4)}


# The tcgen05 products of one (chunk, head) item and one chunk step, as the kernels issue them:
# (phase, N, K, B MN-major, products of that shape per unit).  M = 128 throughout.
# (name, N, K, B MN-major, A MN-major, products per unit); M = 128.  The state products are those of the
# 128-column slices the prefill workload runs: products 1 and 3 transposed (state columns on the M side).
MMA_PHASES = [
    ("prep A: [K e^(g-b); Q e^(g-b)] x 160 anchored key rows, per 64-channel half", 160, 64, False, False, 2),
    ("prep B, K part: [X; X] diag(beta) x -(K gamma)^T", 128, 64, False, False, 1),
    ("prep B, V part: [X; X] diag(beta) x V (MN-major)", 128, 64, True, False, 1),
    ("state 1: S^T [-W; Q gamma]^T (S the MN-major A operand)", 128, 128, False, True, 1),
    ("state 2: Kdec^T U' (U'^T the K-major B operand)", 128, 64, False, False, 1),
    ("state 3: U'^T Aqk^T (N = 64 tokens)", 64, 64, False, False, 1),
]


def mma_phase_rates(kda, tc_tflops, n_sms, sm_mhz):
    """SM cycles per product for each tcgen05 phase shape, back to back and one at a time, as FLOP per
    cycle per SM and as a fraction of the measured bf16 peak expressed per SM cycle."""
    import torch
    peak_fc = tc_tflops * 1e12 / (n_sms * sm_mhz * 1e6)
    rows = []
    for name, n, k, mn, amn, per_unit in MMA_PHASES:
        cyc = kda.kda_selftest_mma_rate(n, k, b_mn_major=mn, a_mn_major=amn, reps=512)
        torch.cuda.synchronize()
        c = cyc.cpu()
        ok = c[:, 0] > 0
        b2b, single = float(c[ok, 0].mean()), float(c[ok, 1].mean())
        fl = 2.0 * 128 * n * k
        rows.append({"phase": name, "M": 128, "N": n, "K": k, "b_mn_major": mn, "a_mn_major": amn, "per_unit": per_unit,
                     "cycles_back_to_back": round(b2b, 1), "cycles_single": round(single, 1),
                     "flop_per_cycle_sm_back_to_back": round(fl / b2b, 1),
                     "flop_per_cycle_sm_single": round(fl / single, 1),
                     "frac_back_to_back": round(fl / b2b / peak_fc, 4), "frac_single": round(fl / single / peak_fc, 4)})
    return {"peak_flop_per_cycle_sm": round(peak_fc, 1),
            "peak_basis": f"measured bf16 peak {tc_tflops} TFLOP/s / {n_sms} SMs / {sm_mhz} MHz",
            "how": "kda_selftest_mma_rate: one CTA per SM, 512 products of each shape timed with the SM clock, "
                   "back to back (one commit at the end) and one at a time (commit and wait per product)",
            "phases": rows}


def run_workload_legs(kda, synth, dev, stream, hbm, want_cpu):
    """The other configurations of the operator, each timed as whole kda_chunk_fwd calls: the fp32
    workload (B=1, T=256, H=2, dk=dv=64), the long-context prefill (B=1, T=2^20, H=32, checkpoints every
    512, initial state) and the varlen batch (64 sequences, lengths U[1024, 65536] seed 1, checkpoints,
    a resumed batch, 8 segments per sequence composed).  Returns (legs, oracle jobs for later timing)."""
    import gc
    import torch
    legs, cpu_jobs = {}, {}
    Dd = D

    # ---------------- fp32: B=1, T=256, H=2, dk=dv=64, zero initial state, seed 0
    inp = synth.make_inputs([256], 2, 64, 64, dtype=torch.float32, device=dev, seed=0)
    o = torch.empty(256, 2, 64, device=dev)
    fs = torch.empty(1, 2, 64, 64, device=dev)
    ws = torch.empty(kda.kda_chunk_fwd_workspace_bytes(256, 1, 2, 64, 64, kda.KDA_F32), dtype=torch.uint8,
                     device=dev)
    f = lambda: kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, None, inp.cu_seqlens, o, fs,
                                  workspace=ws)
    ms = timed_calls(f, 200, 20, stream)
    # fp32 q, k, v (3 x 64 x 4 B), log_alpha (64 x 4 B), beta, o (64 x 4 B); final state 16 KiB per head
    rl = prefill_roofline(512, ms, hbm, extra_bytes=2 * 64 * 64 * 4, read_b=3 * 256 + 256 + 4, out_b=256)
    rl["note"] = "512 token-heads per call: launch- and latency-bound, far below any bandwidth limit"
    legs["fp32"] = {"workload": "KDA chunked forward B=1 T=256 H=2 dk=dv=64 fp32, zero initial state, seed 0",
                    "value": 256 / (ms / 1e3), "unit": "tokens/s", "ms_per_call": round(ms, 5), "dtype": "f32",
                    "roofline": rl}
    if want_cpu:
        cpu_jobs["fp32"] = (host_slices(inp, [(0, 0), (0, 1)]), 2, 512, "the whole workload")
    del inp, o, fs, ws

    # ---------------- long context: B=1, T=2^20, H=32, bf16, log_alpha = -5 sigmoid(N(2, 1)), state ~ N(0, 0.02)
    TL = 1 << 20
    inp = synth.make_inputs([TL], H, Dd, Dd, dtype=torch.bfloat16, device=dev, seed=0, alpha_mu=2.0, alpha_sd=1.0,
                            with_state0=True)
    ckcu_h = kda.kda_ckpt_offsets(inp.cu_seqlens.cpu(), CKPT)
    ck = torch.empty(int(ckcu_h[-1]), H, Dd, Dd, device=dev)
    ckcu = ckcu_h.to(dev)
    o = torch.empty(TL, H, Dd, dtype=torch.bfloat16, device=dev)
    fs = torch.empty(1, H, Dd, Dd, device=dev)
    ws = torch.empty(kda.kda_chunk_fwd_workspace_bytes(TL, 1, H, Dd, Dd, kda.KDA_BF16), dtype=torch.uint8, device=dev)
    f = lambda: kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, inp.state0, inp.cu_seqlens, o, fs,
                                  ckpt_stride=CKPT, checkpoints=ck, ckpt_cu=ckcu, workspace=ws)
    ms = timed_calls(f, 3, 3, stream)
    kda.kda_profile_begin(2)
    for _ in range(2):
        f()
    torch.cuda.synchronize()
    _, lp, ls, ln = kda.kda_profile_end()
    th = TL * H
    st_b = Dd * Dd * 4 * H
    rl = prefill_roofline(th, ms, hbm, extra_bytes=int(ckcu_h[-1]) * st_b + 2 * st_b)
    legs["long_context"] = {
        "workload": "KDA prefill B=1 T=1048576 H=32 dk=dv=128 bf16, log_alpha = -5 sigmoid(N(2,1)), initial state "
                    "~ N(0, 0.02), fp32 checkpoints every 512 tokens, full workspace",
        "value": TL / (ms / 1e3), "unit": "tokens/s", "ms_per_call": round(ms, 4), "dtype": "bf16",
        "roofline": rl, "kernels": {"prep_bf16_kernel": {"ms": round(lp / ln, 4)},
                                    "state_bf16_kernel": {"ms": round(ls / ln, 4)}}}
    if want_cpu:
        keys = [(0, h) for h in range(0, H, 2)]
        cpu_jobs["long_context"] = (host_slices(inp, keys, ckpt=CKPT, tok_limit=1 << 15), H, th,
                                    "first 32768 tokens of every second head, with the 512-token checkpoints")
    del inp, o, fs, ws, ck, ckcu, f
    gc.collect()
    torch.cuda.empty_cache()

    # ---------------- varlen: 64 sequences, lengths U[1024, 65536] (seed 1), H=32, bf16, checkpoints every 512
    lengths = synth.varlen_lengths(64, 1024, 65536, 1)
    N = len(lengths)
    inp = synth.make_inputs(lengths, H, Dd, Dd, dtype=torch.bfloat16, device=dev, seed=0)
    TV = inp.total_tokens
    ckcu_h = kda.kda_ckpt_offsets(inp.cu_seqlens.cpu(), CKPT)
    ck = torch.empty(int(ckcu_h[-1]), H, Dd, Dd, device=dev)
    ckcu = ckcu_h.to(dev)
    o = torch.empty(TV, H, Dd, dtype=torch.bfloat16, device=dev)
    fs = torch.empty(N, H, Dd, Dd, device=dev)
    full_ws = kda.kda_chunk_fwd_workspace_bytes(TV, N, H, Dd, Dd, kda.KDA_BF16)
    free_b, _ = torch.cuda.mem_get_info(dev)
    ws_b = int(min(full_ws, max(kda.kda_chunk_fwd_min_workspace_bytes(N, H, Dd, Dd), free_b - (16 << 30))))
    ws = torch.empty(ws_b, dtype=torch.uint8, device=dev)
    f = lambda: kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, None, inp.cu_seqlens, o, fs,
                                  ckpt_stride=CKPT, checkpoints=ck, ckpt_cu=ckcu, workspace=ws)
    ms = timed_calls(f, 3, 3, stream)
    th = TV * H
    rl = prefill_roofline(th, ms, hbm, extra_bytes=int(ckcu_h[-1]) * st_b + N * st_b)
    varlen = {"workload": f"KDA varlen prefill: 64 sequences, lengths U[1024, 65536] (seed 1, {TV} tokens), packed, "
                          "H=32 dk=dv=128 bf16, zero initial state, fp32 checkpoints every 512 tokens",
              "value": TV / (ms / 1e3), "unit": "tokens/s", "ms_per_call": round(ms, 4), "dtype": "bf16",
              "workspace_bytes": ws_b, "windowed": ws_b < full_ws, "roofline": rl}
    if want_cpu:
        keys = [(i, h) for i in range(0, N, 8) for h in (0, 16)]
        cpu_jobs["varlen"] = (host_slices(inp, keys, ckpt=CKPT), H, th,
                              "whole sequences 0, 8, .., 56 at heads 0 and 16, with the 512-token checkpoints")
    # 8 segments per sequence (b_s = 64 floor(s len / 512)) from a zero state with their transitions, then the
    # prefix scan over the segments' (transition, zero-start state)
    seg_len = []
    for L in lengths:
        bb = [64 * ((s_ * L) // 512) for s_ in range(8)] + [L]
        seg_len += [bb[s_ + 1] - bb[s_] for s_ in range(8)]
    seg_cu = synth.cu_from_lengths(seg_len, dev)
    Zs = torch.empty(len(seg_len), H, Dd, Dd, device=dev)
    Ms = torch.empty(len(seg_len), H, Dd, Dd, device=dev)
    g = lambda: kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, None, seg_cu, o, Zs,
                                  final_transition=Ms, workspace=ws)
    seg_ms = timed_calls(g, 2, 1, stream)
    starts = torch.empty_like(Zs)
    ends = torch.empty(N, H, Dd, Dd, device=dev)
    scu = synth.cu_from_lengths([8] * N, dev)
    h_ = lambda: kda.kda_segment_compose(Ms, Zs, scu, None, starts, ends)
    comp_ms = timed_calls(h_, 3, 1, stream)
    varlen["segments"] = {"what": "kda_chunk_fwd over the 512 segments from zero with their transitions, then "
                                  "kda_segment_compose", "chunk_fwd_ms": round(seg_ms, 4),
                          "compose_ms": round(comp_ms, 4)}
    # resumed batch: the even sequences restart at b_i = 512 floor(len_i / 1024) from their stored checkpoint, the
    # odd ones run whole (their token inputs drawn afresh with those lengths; the states come from the run above)
    even = list(range(0, N, 2))
    b_res = {i: CKPT * (lengths[i] // 1024) for i in even}
    init = torch.zeros(N, H, Dd, Dd, device=dev)
    for i in even:
        if b_res[i] > 0:
            init[i] = ck[int(ckcu_h[i]) + b_res[i] // CKPT - 1]
    rlen = [lengths[i] - b_res.get(i, 0) for i in range(N)]
    del inp, o, fs, ck, ckcu, Zs, Ms, starts, ends, f, g, h_
    gc.collect()
    torch.cuda.empty_cache()
    rin = synth.make_inputs(rlen, H, Dd, Dd, dtype=torch.bfloat16, device=dev, seed=1)
    TR = rin.total_tokens
    rck_h = kda.kda_ckpt_offsets(rin.cu_seqlens.cpu(), CKPT)
    rck = torch.empty(max(1, int(rck_h[-1])), H, Dd, Dd, device=dev)
    rckcu = rck_h.to(dev)
    ro = torch.empty(TR, H, Dd, dtype=torch.bfloat16, device=dev)
    rfs = torch.empty(N, H, Dd, Dd, device=dev)
    f = lambda: kda.kda_chunk_fwd(rin.q, rin.k, rin.v, rin.log_alpha, rin.beta, init, rin.cu_seqlens, ro, rfs,
                                  ckpt_stride=CKPT, checkpoints=rck, ckpt_cu=rckcu, workspace=ws)
    rms = timed_calls(f, 3, 3, stream)
    varlen["resume"] = {"what": "the batch with the even sequences resumed at 512 floor(len / 1024) from their "
                                "checkpoints (odd ones whole)", "tokens": TR, "ms_per_call": round(rms, 4),
                        "value": TR / (rms / 1e3), "unit": "tokens/s",
                        "roofline": prefill_roofline(TR * H, rms, hbm,
                                                     extra_bytes=int(rck_h[-1]) * st_b + 2 * N * st_b)}
    legs["varlen"] = varlen
    del rin, ro, rfs, rck, rckcu, init, ws, f
    gc.collect()
    torch.cuda.empty_cache()
    return legs, cpu_jobs


def run_ours(args):
    import torch
    import kda_linear_attention_02_b200 as kda
    from kda_linear_attention_02_b200 import synth

    rank, world, local = dist_setup(args)
    dev = torch.device("cuda", torch.cuda.current_device())
    hbm, tc, tc_sus, peak_kind = peaks()
    stream = torch.cuda.current_stream()

    # ------------------------------------------------------------------ prefill workload
    inp = synth.make_inputs([T] * B, H, D, D, dtype=torch.bfloat16, device=dev, seed=rank)
    ckcu_h = kda.kda_ckpt_offsets(inp.cu_seqlens.cpu(), CKPT)
    ckcu = ckcu_h.to(dev)
    ck = torch.empty(int(ckcu_h[-1]), H, D, D, device=dev)
    o = torch.empty(B * T, H, D, dtype=torch.bfloat16, device=dev)
    fs = torch.empty(B, H, D, D, device=dev)
    ws = torch.empty(kda.kda_chunk_fwd_workspace_bytes(B * T, B, H, D, D, kda.KDA_BF16), dtype=torch.uint8,
                     device=dev)

    def step():
        kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, None, inp.cu_seqlens, o, fs,
                          ckpt_stride=CKPT, checkpoints=ck, ckpt_cu=ckcu, workspace=ws)

    clocks = Clocks(dev.index if world == 1 else local)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    # The timed steps run without per-kernel events: an event recorded between two kernels serialises
    # them, while the library lets each kernel's blocks start as the previous kernel drains.
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = e0.elapsed_time(e1) / args.steps
    # per-kernel durations: the same steps once more, with CUDA events around each kernel
    prof_steps = min(args.steps, 50)
    kda.kda_profile_begin(prof_steps)
    for _ in range(prof_steps):
        step()
    torch.cuda.synchronize()
    ms_idx, ms_prep, ms_state, ncalls = kda.kda_profile_end()
    barrier(world)
    ms_max = max_over_ranks(ms, world)
    st = kda.kda_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status {kda.kda_status_string(st)}")
    tokens_job = B * T * world
    value = tokens_job / (ms_max / 1e3)

    # per-kernel roofline (live CUDA events on the launching stream, averaged over the timed calls)
    th = B * T * H
    prep_ms, state_ms, idx_ms = ms_prep / ncalls, ms_state / ncalls, ms_idx / ncalls
    prep_bytes, state_bytes = PREFILL_READ_B * th, PREFILL_WRITE_B * th
    kernels = {
        "kda_chunk_index": {"ms": idx_ms},
        "prep_bf16_kernel": {"ms": prep_ms, "alg_bytes": prep_bytes,
                             "achieved_gbs": prep_bytes / (prep_ms / 1e3) / 1e9},
        "state_bf16_kernel": {"ms": state_ms, "alg_bytes": state_bytes,
                              "achieved_gbs": state_bytes / (state_ms / 1e3) / 1e9},
    }
    dom = "prep_bf16_kernel" if prep_ms >= state_ms else "state_bf16_kernel"
    ach = kernels[dom]["achieved_gbs"]
    whole_bytes = (PREFILL_READ_B + PREFILL_WRITE_B) * th
    whole_gbs = whole_bytes / (ms / 1e3) / 1e9
    traffic = captured_traffic(dom)
    roofline = {"bound": "hbm", "kernel": dom, "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(ach / hbm, 4), "traffic": traffic, "peak_kind": peak_kind,
                "alg_bytes_per_launch": kernels[dom]["alg_bytes"],
                "whole_step": {"alg_bytes": whole_bytes, "achieved_gbs": round(whole_gbs, 1),
                               "frac": round(whole_gbs / hbm, 4)},
                "kernels": {k: {kk: (round(vv, 4) if isinstance(vv, float) else vv) for kk, vv in v.items()}
                            for k, v in kernels.items()},
                "kernel_timing": f"CUDA events around each kernel over {prof_steps} further steps of the same "
                                 "workload (the timed steps run without them)"}

    # ------------------------------------------------------------------ end to end from host buffers
    pin = lambda t: torch.empty(t.shape, dtype=t.dtype, pin_memory=True).copy_(t.cpu())
    hq, hk, hv, hla, hb = pin(inp.q), pin(inp.k), pin(inp.v), pin(inp.log_alpha), pin(inp.beta)
    ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    hfs = torch.empty(fs.shape, dtype=fs.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hla, hb))
    d2h = ho.numel() * ho.element_size() + hfs.numel() * hfs.element_size()
    e2e_steps = max(2, min(args.steps, 20))   # about 13 ms each (PCIe-bound)
    # Pipelined through the public C ABI: step i's inputs go up on one stream while step i - 1 computes and
    # its o and final state come down on a third; two device buffer sets alternate, ordered by events.
    # Every step still uploads its own inputs and downloads its own results inside the timed region.
    bufs = [(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, o, fs)]
    bufs.append(tuple(torch.empty_like(t) for t in bufs[0]))
    ws2 = ws
    s_up, s_cmp, s_dn = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = {k_: [torch.cuda.Event() for _ in range(2)] for k_ in ("up", "cmp", "dn")}
    ho2 = [ho, torch.empty_like(ho, pin_memory=True)]
    hfs2 = [hfs, torch.empty_like(hfs, pin_memory=True)]
    first_use = [True, True]

    def e2e_step(i):
        b = i % 2
        q_, k_, v_, la_, b_, o_, fs_ = bufs[b]
        with torch.cuda.stream(s_up):
            if not first_use[b]:
                s_up.wait_event(ev["cmp"][b])          # step i - 2 has finished reading this input set
            for d_, h_ in ((q_, hq), (k_, hk), (v_, hv), (la_, hla), (b_, hb)):
                d_.copy_(h_, non_blocking=True)
            ev["up"][b].record(s_up)
        s_cmp.wait_event(ev["up"][b])
        if not first_use[b]:
            s_cmp.wait_event(ev["dn"][b])              # step i - 2's results have left this output set
        kda.kda_chunk_fwd(q_, k_, v_, la_, b_, None, inp.cu_seqlens, o_, fs_, ckpt_stride=CKPT, checkpoints=ck,
                          ckpt_cu=ckcu, workspace=ws2, stream=s_cmp)
        ev["cmp"][b].record(s_cmp)
        with torch.cuda.stream(s_dn):
            s_dn.wait_event(ev["cmp"][b])
            ho2[b].copy_(o_, non_blocking=True)
            hfs2[b].copy_(fs_, non_blocking=True)
            ev["dn"][b].record(s_dn)
        first_use[b] = False

    def drain():
        for st in (s_up, s_cmp, s_dn):
            st.synchronize()

    for i in range(2):
        e2e_step(i)
    drain()
    barrier(world)
    e0.record(s_cmp)
    s_up.wait_event(e0)
    s_dn.wait_event(e0)
    for i in range(e2e_steps):
        e2e_step(i)
    s_cmp.wait_stream(s_up)
    s_cmp.wait_stream(s_dn)
    e1.record(s_cmp)
    drain()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world)
    e2e = {"value": tokens_job / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 3)}
    del hq, hk, hv, hla, hb, ho, hfs, ho2, hfs2, bufs

    # ------------------------------------------------------------------ the prefill with MXFP8 q, k, v
    # The same workload, its q, k, v quantised to MXFP8 (E4M3 codes, one E8M0 scale per 32 channels).
    mx = (*synth.mxfp8_quantize(inp.q), *synth.mxfp8_quantize(inp.k), *synth.mxfp8_quantize(inp.v))

    def mx_step():
        kda.kda_chunk_fwd_mxfp8(*mx, inp.log_alpha, inp.beta, None, inp.cu_seqlens, o, fs, ckpt_stride=CKPT,
                                checkpoints=ck, ckpt_cu=ckcu, workspace=ws)

    mx_steps = max(3, min(args.steps, 50))
    for _ in range(3):
        mx_step()
    torch.cuda.synchronize()
    barrier(world)
    e0.record(stream)
    for _ in range(mx_steps):
        mx_step()
    e1.record(stream)
    torch.cuda.synchronize()
    mx_ms = max_over_ranks(e0.elapsed_time(e1) / mx_steps, world)
    kda.kda_profile_begin(mx_steps)
    for _ in range(mx_steps):
        mx_step()
    torch.cuda.synchronize()
    _, mx_prep, mx_state, mx_n = kda.kda_profile_end()
    barrier(world)
    mx_prep_ms = mx_prep / mx_n
    mx_prep_gbs = PREFILL_READ_MX_B * th / (mx_prep_ms / 1e3) / 1e9
    mxfp8 = {"workload": "the prefill workload with q, k, v in MXFP8 (E4M3 codes, E8M0 scale per 32 channels)",
             "value": tokens_job / (mx_ms / 1e3), "unit": "tokens/s", "ms_per_step": round(mx_ms, 5),
             "kernels": {"prep_bf16_kernel<MX>": {"ms": round(mx_prep_ms, 4)},
                         "state_bf16_kernel": {"ms": round(mx_state / mx_n, 4)}},
             "roofline": {"bound": "hbm", "kernel": "prep_bf16_kernel (MXFP8 inputs)",
                          "achieved": round(mx_prep_gbs, 1), "peak": hbm, "unit": "GB/s",
                          "frac": round(mx_prep_gbs / hbm, 4), "alg_bytes_per_launch": PREFILL_READ_MX_B * th}}
    st = kda.kda_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status {kda.kda_status_string(st)}")
    del mx

    # ------------------------------------------------------------------ decode workload
    s0, dq, dk_, dv_, dla, db = synth.make_decode_inputs(DEC_N, H, D, D, dtype=torch.bfloat16, device=dev,
                                                         seed=100 + rank, steps=DEC_STEPS)
    state = s0.clone()
    do = torch.empty(DEC_N, H, D, dtype=torch.bfloat16, device=dev)
    for t_ in range(3):
        kda.kda_recurrent_step(state, dq[t_], dk_[t_], dv_[t_], dla[t_], db[t_], do)
    state.copy_(s0)
    torch.cuda.synchronize()
    barrier(world)
    e0.record(stream)
    for t_ in range(DEC_STEPS):
        kda.kda_recurrent_step(state, dq[t_], dk_[t_], dv_[t_], dla[t_], db[t_], do)
    e1.record(stream)
    torch.cuda.synchronize()
    dec_ms = max_over_ranks(e0.elapsed_time(e1), world)
    step_ms = dec_ms / DEC_STEPS
    dec_bytes = DECODE_B * DEC_N * H
    dec_gbs = dec_bytes / (step_ms / 1e3) / 1e9
    decode = {"metric": "KDA decode steps/s (256 seqs x H=32, 128x128 fp32 state, 1024 steps)",
              "value": world * DEC_STEPS / (dec_ms / 1e3), "unit": "steps/s",
              "tokens_per_s": DEC_N * world * DEC_STEPS / (dec_ms / 1e3), "ms_per_step": round(step_ms, 5),
              "roofline": {"bound": "hbm", "kernel": "decode_step_kernel", "achieved": round(dec_gbs, 1),
                           "peak": hbm, "unit": "GB/s", "frac": round(dec_gbs / hbm, 4),
                           "alg_bytes_per_launch": dec_bytes}}
    # kept for the oracle's decode timing, which runs after the clock sampling has stopped
    dec_in = (s0, dq, dk_, dv_, dla, db) if rank == 0 and world == 1 and not args.no_cpu_baseline else None
    # the same decode loop with MXFP8 q, k, v (1-byte codes + one scale byte per 32 channels)
    mxd = (*synth.mxfp8_quantize(dq), *synth.mxfp8_quantize(dk_), *synth.mxfp8_quantize(dv_))
    del dq, dk_, dv_
    state.copy_(s0)
    for t_ in range(3):
        kda.kda_recurrent_step_mxfp8(state, *(x[t_] for x in mxd), dla[t_], db[t_], do)
    state.copy_(s0)
    torch.cuda.synchronize()
    barrier(world)
    e0.record(stream)
    for t_ in range(DEC_STEPS):
        kda.kda_recurrent_step_mxfp8(state, *(x[t_] for x in mxd), dla[t_], db[t_], do)
    e1.record(stream)
    torch.cuda.synchronize()
    mxd_ms = max_over_ranks(e0.elapsed_time(e1), world) / DEC_STEPS
    mxd_bytes = DECODE_MX_B * DEC_N * H
    decode["mxfp8"] = {"value": world / (mxd_ms / 1e3), "unit": "steps/s", "ms_per_step": round(mxd_ms, 5),
                       "roofline": {"bound": "hbm", "kernel": "decode_step_kernel (MXFP8 inputs)",
                                    "achieved": round(mxd_bytes / (mxd_ms / 1e3) / 1e9, 1), "peak": hbm,
                                    "unit": "GB/s", "frac": round(mxd_bytes / (mxd_ms / 1e3) / 1e9 / hbm, 4),
                                    "alg_bytes_per_launch": mxd_bytes}}
    del s0, mxd, dla, db, state, do

    # ------------------------------------------------------------------ speculative decoding
    # The decode workload's 256 sequences x 32 heads; each round verifies 4 drafts per sequence
    # (kda_decode_verify) and commits an accepted prefix drawn uniformly from 0..4 (kda_decode_commit).
    # A pool of 16 seeded draft sets (673 MB, larger than L2) is cycled through.
    gen = torch.Generator("cpu").manual_seed(300 + rank)
    s0, sq, sk, sv, sla, sb = synth.make_decode_inputs(DEC_N, H, D, D, dtype=torch.bfloat16, device=dev,
                                                       seed=200 + rank, steps=SPEC_ND * SPEC_POOL)
    pool = []
    for r in range(SPEC_POOL):
        sl = slice(r * SPEC_ND, (r + 1) * SPEC_ND)
        acc_h = torch.randint(0, SPEC_ND + 1, (DEC_N,), generator=gen, dtype=torch.int32)
        pool.append(tuple(synth.draft_layout(x[sl]) for x in (sq, sk, sv, sla, sb)) + (acc_h.to(dev), acc_h))
    del sq, sk, sv, sla, sb
    state = s0.clone()
    so = torch.empty(DEC_N * SPEC_ND, H, D, dtype=torch.bfloat16, device=dev)

    def spec_round(r):
        q_, k_, v_, la_, b_, acc_d, _ = pool[r % SPEC_POOL]
        kda.kda_decode_verify(state, q_, k_, v_, la_, b_, so)
        kda.kda_decode_commit(state, k_, v_, la_, b_, acc_d)

    for r in range(3):
        spec_round(r)
    state.copy_(s0)
    torch.cuda.synchronize()
    barrier(world)
    e0.record(stream)
    for r in range(SPEC_ROUNDS):
        spec_round(r)
    e1.record(stream)
    torch.cuda.synchronize()
    spec_ms = max_over_ranks(e0.elapsed_time(e1), world) / SPEC_ROUNDS
    # algorithmic bytes per round: verify reads the state once and every draft's q, k, v (bf16), log_alpha
    # and beta, and writes its output; commit reads and writes the state of the sequences that accepted
    # at least one draft, reading the accepted drafts' k, v, log_alpha, beta.
    st_b = D * D * 4
    ver_b = DEC_N * H * (st_b + SPEC_ND * (3 * D * 2 + D * 4 + 4 + D * 2))
    com_b = sum(H * sum((2 * st_b + int(a) * (2 * D * 2 + D * 4 + 4)) for a in p[6].tolist() if a > 0)
                for p in pool) / SPEC_POOL
    acc_mean = sum(float(p[6].float().mean()) for p in pool) / SPEC_POOL
    spec_gbs = (ver_b + com_b) / (spec_ms / 1e3) / 1e9
    speculative = {"workload": f"{DEC_N} seqs x H={H}, {D}x{D} fp32 state, {SPEC_ND} drafts per round, accepted "
                               f"counts uniform in 0..{SPEC_ND}", "rounds_per_s": world / (spec_ms / 1e3),
                   "accepted_tokens_per_s": world * DEC_N * acc_mean / (spec_ms / 1e3),
                   "ms_per_round": round(spec_ms, 5), "mean_accepted": round(acc_mean, 3),
                   "roofline": {"bound": "hbm", "kernel": "decode_multi_kernel (verify + commit)",
                                "achieved": round(spec_gbs, 1), "peak": hbm, "unit": "GB/s",
                                "frac": round(spec_gbs / hbm, 4), "alg_bytes_per_round": int(ver_b + com_b)}}
    del s0, pool, state, so

    # ------------------------------------------------------------------ segment compose (64 seqs x 8 segments)
    nseg = 8
    M = torch.randn(64 * nseg, H, D, D, device=dev) * (1.0 / D ** 0.5)
    Z = torch.randn(64 * nseg, H, D, D, device=dev)
    seg_cu = synth.cu_from_lengths([nseg] * 64, dev)
    starts = torch.empty_like(Z)
    ends = torch.empty(64, H, D, D, device=dev)
    comp_ms = timed_calls(lambda: kda.kda_segment_compose(M, Z, seg_cu, None, starts, ends), 5, 3, stream)
    comp_bytes = 64 * nseg * H * 3 * D * D * 4
    compose = {"workload": "64 sequences x 8 segments x H=32, dk=dv=128 fp32", "ms": round(comp_ms, 4),
               "achieved_gbs": round(comp_bytes / (comp_ms / 1e3) / 1e9, 1)}
    del M, Z, starts, ends
    props = torch.cuda.get_device_properties(dev)
    mma = mma_phase_rates(kda, tc, props.multi_processor_count, 1965.0)
    legs, leg_jobs = {}, {}
    if not args.no_workloads:
        legs, leg_jobs = run_workload_legs(kda, synth, dev, stream, hbm,
                                           rank == 0 and world == 1 and not args.no_cpu_baseline)
    clk = clocks.stop()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_sample(inp)
    if dec_in is not None:
        decode["cpu_baseline"] = cpu_oracle_decode_sample(*dec_in)
        dec_in = None
    for name, (jobs, heads, total, what) in leg_jobs.items():
        legs[name]["cpu_baseline"] = cpu_oracle_jobs(jobs, heads, total, what)
    leg_jobs = None

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_max, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "KDA prefill B=4 T=4096 H=32 dk=dv=128 bf16, zero initial state, fp32 final "
                                   "state, fp32 checkpoints every 512 tokens",
                       "global_batch": B * world, "seq_len": T, "heads": H, "dk": D, "dv": D, "ckpt_stride": CKPT,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": "inputs and outputs larger than L2 (1.1 GB per step), no flush"},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clk,
            "gpu_launches": 4 * args.steps, "mma_phases": mma, "decode": decode, "speculative": speculative, "compose": compose, "mxfp8": mxfp8,
        }
        line.update(legs)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_reference(args):
    """fp64 CPU oracle, as it stands, on the host cores: each step is a bounded sample of the same
    prefill workload (whole (sequence, head) slices)."""
    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    from kda_linear_attention_02_b200 import synth
    import oracle
    oracle.build()
    inp = synth.make_inputs([T] * B, H, D, D, dtype=torch.bfloat16, device="cpu", seed=0)
    per_step_slices = oracle.threads_used()          # one slice per host thread per step
    samples = []
    for it in range(args.warmup + args.steps):
        r = cpu_oracle_sample(inp, budget_s=1e9, max_slices=per_step_slices)
        if it >= args.warmup:
            samples.append(r)
    val = statistics.median(s["value"] for s in samples)
    ms = per_step_slices * T / H / val * 1e3
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "KDA prefill B=4 T=4096 H=32 dk=dv=128 bf16, zero initial state, fp32 final "
                                   "state, fp32 checkpoints every 512 tokens",
                       "global_batch": B, "seq_len": T, "heads": H, "dk": D, "dv": D, "ckpt_stride": CKPT},
            "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": samples[0]["cores"], "kind": "oracle",
                             "sample": f"each step: {per_step_slices} (sequence, head) slices x {T} tokens"},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the fp32, long-context and varlen workloads (timed after the headline)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
