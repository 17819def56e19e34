"""Pins for the fp64 oracle: it is checked against things other than itself.

Each pin is chosen so that a plausible slip in the oracle (a dropped term, a wrong sign, decay on the
value axis instead of the key axis, o read from S_{t-1} instead of S_t, a wrong floor) fails one:
  * a hand-worked scalar example (tests/golden/kda_scalar_hand_example.txt);
  * the dk = dv = 1 closed form on random inputs;
  * brute force: explicit dense products of the per-step maps for T <= 16 (a different algorithm);
  * the delta rule's exactness (beta = 1, |k| = 1 writes v exactly: q = k reads it back);
  * the contraction bound of the cumulative transition;
  * reductions: literal beta = 0, channel-wise gated linear attention and causal linear attention
    (erase-free limit beta -> 0), and the scalar-gate (Gated DeltaNet) special case;
  * the decay floor facts printed on the orkas.ai page (tests/golden/decay_floor_facts.txt);
  * segment composition (transition + zero-start state, then a prefix scan) reproduces the unsplit
    run, while a plain sum of zero-start states does not;
  * the fp64 chunk form (tests/chunk_reference.py) reproduces the sequential loop;
  * the MXFP8 input decode: every E4M3 and E8M0 code against torch's own float8 conversions (an
    independent library routine), the format facts of the OCP MX v1.0 specification
    (tests/golden/mxfp8_format_facts.txt), and the block structure of the shared scales.
"""
import math
import os

import numpy as np
import pytest
import torch

from chunk_reference import blocked_unit_lower_inverse, chunk_forward

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_inputs(rng, T, dk, dv, unit=True, la_lo=-3.0, la_hi=-0.01):
    q = rng.standard_normal((T, dk)).astype(np.float32)
    k = rng.standard_normal((T, dk)).astype(np.float32)
    if unit:
        q /= np.linalg.norm(q, axis=1, keepdims=True)
        k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv)).astype(np.float32)
    la = rng.uniform(la_lo, la_hi, (T, dk)).astype(np.float32)
    b = rng.uniform(0.05, 0.95, T).astype(np.float32)
    return q, k, v, la, b


def _rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


def test_hand_example_scalar(oracle_mod):
    rows = []
    s0 = None
    for line in open(os.path.join(GOLDEN, "kda_scalar_hand_example.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith("s0"):
            s0 = float(line.split()[1])
            continue
        rows.append([float(x) for x in line.split()])
    rows = np.array(rows)
    T = len(rows)
    la = np.log(rows[:, 1]).reshape(T, 1)
    out = oracle_mod.kda_seq(rows[:, 5:6], rows[:, 3:4], rows[:, 4:5], la, rows[:, 2],
                             s0=np.array([[s0]]), marks=list(range(1, T + 1)))
    # ln(1/2) reaches the operator as fp32 (relative rounding <= 2^-24), so alpha carries a relative
    # error of about 4e-8 per step; everything else in the example is exact in binary.
    np.testing.assert_allclose(out["marks"][:, 0, 0], rows[:, 6], rtol=2e-7, atol=0)
    np.testing.assert_allclose(out["o"][:, 0], rows[:, 7], rtol=2e-7, atol=0)


def test_scalar_closed_form(oracle_mod):
    rng = np.random.default_rng(1)
    T = 40
    q, k, v, la, b = _rand_inputs(rng, T, 1, 1, unit=False)
    s0 = 0.7
    out = oracle_mod.kda_seq(q, k, v, la, b, s0=np.array([[s0]]))
    q, k, v, la, b = (x.astype(np.float64) for x in (q, k, v, la, b))
    f = (1.0 - b * k[:, 0] ** 2) * np.exp(la[:, 0])          # per-step factor
    for t in range(T):
        s = np.prod(f[:t + 1]) * s0
        for j in range(t + 1):
            s += np.prod(f[j + 1:t + 1]) * b[j] * k[j, 0] * v[j, 0]
        assert abs(out["o"][t, 0] - s * q[t, 0]) <= 1e-12 * max(1.0, abs(s))


@pytest.mark.parametrize("T,dk,dv", [(1, 4, 4), (7, 5, 3), (16, 8, 6), (16, 3, 9)])
def test_brute_force_dense_products(oracle_mod, T, dk, dv):
    rng = np.random.default_rng(T * 100 + dk * 10 + dv)
    q, k, v, la, b = _rand_inputs(rng, T, dk, dv)
    s0 = rng.standard_normal((dk, dv))
    out = oracle_mod.kda_seq(q, k, v, la, b, s0=s0, marks=list(range(1, T + 1)),
                             want_transition=True)
    q, k, v, la, b = (x.astype(np.float64) for x in (q, k, v, la, b))
    A = [(np.eye(dk) - b[t] * np.outer(k[t], k[t])) @ np.diag(np.exp(la[t])) for t in range(T)]

    def P(a, z):           # A_z ... A_a  (empty product = I), 0-based inclusive
        m = np.eye(dk)
        for t in range(a, z + 1):
            m = A[t] @ m
        return m

    for t in range(T):
        S = P(0, t) @ s0
        for j in range(t + 1):
            S = S + P(j + 1, t) @ (b[j] * np.outer(k[j], v[j]))
        np.testing.assert_allclose(out["marks"][t], S, rtol=0, atol=1e-12)
        np.testing.assert_allclose(out["o"][t], S.T @ q[t], rtol=0, atol=1e-12)
    np.testing.assert_allclose(out["transition"], P(0, T - 1), rtol=0, atol=1e-12)
    np.testing.assert_allclose(out["state"], out["marks"][-1], rtol=0, atol=0)


def test_delta_rule_writes_value_exactly(oracle_mod):
    rng = np.random.default_rng(3)
    T, dk, dv = 50, 16, 12
    q, k, v, la, b = _rand_inputs(rng, T, dk, dv)
    b[:] = 1.0
    out = oracle_mod.kda_seq(k, k, v, la, b, s0=rng.standard_normal((dk, dv)))
    # |k| = 1 to fp32 rounding; the readback equals v up to that rounding
    np.testing.assert_allclose(out["o"], v.astype(np.float64), rtol=0, atol=1e-5)


def test_transition_is_a_contraction(oracle_mod):
    rng = np.random.default_rng(4)
    T, dk, dv = 64, 12, 4
    q, k, v, la, b = _rand_inputs(rng, T, dk, dv)
    b = rng.uniform(0.0, 2.0, T).astype(np.float32)
    out = oracle_mod.kda_seq(q, k, v, la, b, want_transition=True)
    kn = np.linalg.norm(k.astype(np.float64), axis=1)
    slack = 1e-6 * T + np.max(np.abs(kn - 1.0)) * 4 * T
    assert np.linalg.norm(out["transition"], 2) <= 1.0 + slack
    # and the state map is affine: M s0 + Z equals the run from s0
    s0 = rng.standard_normal((dk, dv))
    z = oracle_mod.kda_seq(q, k, v, la, b)["state"]
    full = oracle_mod.kda_seq(q, k, v, la, b, s0=s0)["state"]
    np.testing.assert_allclose(out["transition"] @ s0 + z, full, rtol=0, atol=1e-12)


def test_literal_beta_zero(oracle_mod):
    rng = np.random.default_rng(5)
    T, dk, dv = 30, 8, 5
    q, k, v, la, b = _rand_inputs(rng, T, dk, dv)
    b[:] = 0.0
    s0 = rng.standard_normal((dk, dv))
    out = oracle_mod.kda_seq(q, k, v, la, b, s0=s0)
    G = np.cumsum(la.astype(np.float64), axis=0)
    ref = (np.exp(G) * q.astype(np.float64)) @ s0
    np.testing.assert_allclose(out["o"], ref, rtol=1e-12, atol=1e-14)
    # alpha == 1 as well: the state never moves
    out1 = oracle_mod.kda_seq(q, k, v, np.zeros_like(la), b, s0=s0)
    np.testing.assert_allclose(out1["o"], q.astype(np.float64) @ s0, rtol=1e-13, atol=1e-14)


def test_erase_free_limit_is_gated_linear_attention(oracle_mod):
    rng = np.random.default_rng(6)
    T, dk, dv = 40, 8, 6
    q, k, v, la, _ = _rand_inputs(rng, T, dk, dv)
    eps = 1e-9
    b = np.full(T, eps, np.float32)
    out = oracle_mod.kda_seq(q, k, v, la, b)
    q64, k64, v64 = (x.astype(np.float64) for x in (q, k, v))
    G = np.cumsum(la.astype(np.float64), axis=0)
    gla = np.zeros((T, dv))
    for t in range(T):
        for s in range(t + 1):
            gla[t] += (q64[t] * np.exp(G[t] - G[s])) @ k64[s] * v64[s]
    beps = float(np.float32(eps))
    assert _rel(out["o"] / beps, gla) < 1e-6
    # alpha == 1: causal linear attention tril(Q K^T) V
    out1 = oracle_mod.kda_seq(q, k, v, np.zeros_like(la), b)
    lin = np.tril(q64 @ k64.T) @ v64
    assert _rel(out1["o"] / beps, lin) < 1e-6


def test_scalar_gate_reduces_to_gated_deltanet(oracle_mod):
    rng = np.random.default_rng(7)
    T, dk, dv = 33, 10, 7
    q, k, v, _, b = _rand_inputs(rng, T, dk, dv)
    gate = rng.uniform(-2.0, -0.05, T).astype(np.float32)
    la = np.repeat(gate[:, None], dk, axis=1)
    s0 = rng.standard_normal((dk, dv))
    out = oracle_mod.kda_seq(q, k, v, la, b, s0=s0)
    # Gated DeltaNet: one scalar gate per head and token
    S = s0.copy()
    for t in range(T):
        kt, vt, qt = (x[t].astype(np.float64) for x in (k, v, q))
        S = math.exp(float(gate[t])) * S
        S = S - float(b[t]) * np.outer(kt, kt @ S) + float(b[t]) * np.outer(kt, vt)
        np.testing.assert_allclose(out["o"][t], S.T @ qt, rtol=0, atol=1e-12)


def test_decay_floor_facts(oracle_mod):
    facts = {}
    for line in open(os.path.join(GOLDEN, "decay_floor_facts.txt")):
        if line.strip() and not line.startswith("#"):
            key, val = line.split()
            facts[key] = float(val)
    lf = oracle_mod.decay_floor()
    assert lf == math.log(facts["retain_floor"])
    assert abs(lf - (-5.005647752585217)) < 1e-12
    tile_min = facts["tile_tokens"] * lf                    # -80.09
    assert facts["tile_log_decay_bound"] - 0.1 < tile_min < facts["tile_log_decay_bound"]
    inv = math.exp(-tile_min)
    assert inv < 1.1 * facts["inverse_bound_printed"] * math.exp(0.1)   # e^80.09 = 6.06e34
    assert abs(math.exp(80) / facts["inverse_bound_printed"] - 1) < 0.01
    bf16_max = torch.finfo(torch.bfloat16).max
    assert abs(bf16_max / facts["bf16_max_printed"] - 1) < 0.01
    assert inv < bf16_max and 128 * inv < torch.finfo(torch.float32).max


def test_floor_clamps_log_decay(oracle_mod):
    rng = np.random.default_rng(8)
    T, dk, dv = 20, 6, 5
    q, k, v, la, b = _rand_inputs(rng, T, dk, dv)
    lf = oracle_mod.decay_floor()
    la_f = la.copy(); la_f[:, ::2] = np.float32(lf)
    la_inf = la.copy(); la_inf[:, ::2] = -np.inf
    la_m6 = la.copy(); la_m6[:, ::2] = -6.0
    la_nan = la.copy(); la_nan[:, ::2] = np.nan
    ref = oracle_mod.kda_seq(q, k, v, la_f, b)["o"]
    fl32 = float(np.float32(lf))
    # fp32 rounding of the floor constant vs the double one: tiny difference only
    for lx in (la_inf, la_m6, la_nan):
        o = oracle_mod.kda_seq(q, k, v, lx, b)["o"]
        assert _rel(o, ref) < 1e-6 * (1 + abs(fl32 - lf) * 1e6)
    # above the floor nothing changes
    o_above = oracle_mod.kda_seq(q, k, v, la, b)["o"]
    assert _rel(o_above, ref) > 1e-3


def test_segment_composition(oracle_mod):
    rng = np.random.default_rng(9)
    T, dk, dv = 97, 8, 6
    q, k, v, la, b = _rand_inputs(rng, T, dk, dv)
    s0 = rng.standard_normal((dk, dv))
    bounds = [0, 13, 40, 41, 90, T]
    full = oracle_mod.kda_seq(q, k, v, la, b, s0=s0, marks=bounds[1:])
    Ms, Zs = [], []
    for a, z in zip(bounds[:-1], bounds[1:]):
        r = oracle_mod.kda_seq(q[a:z], k[a:z], v[a:z], la[a:z], b[a:z], want_transition=True,
                               want_o=False)
        Ms.append(r["transition"]); Zs.append(r["state"])
    starts, end = oracle_mod.segment_compose(np.array(Ms), np.array(Zs), s0)
    np.testing.assert_allclose(end, full["state"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(starts[0], s0, rtol=0, atol=0)
    for si in range(1, len(bounds) - 1):
        np.testing.assert_allclose(starts[si], full["marks"][si - 1], rtol=0, atol=1e-12)
    # re-running each segment from its composed start state gives the unsplit outputs
    for si, (a, z) in enumerate(zip(bounds[:-1], bounds[1:])):
        o = oracle_mod.kda_seq(q[a:z], k[a:z], v[a:z], la[a:z], b[a:z], s0=starts[si])["o"]
        np.testing.assert_allclose(o, full["o"][a:z], rtol=0, atol=1e-12)
    # a plain sum of zero-start states is wrong for KDA (token-dependent transitions)
    plain = sum(Zs)
    assert _rel(plain, full["state"]) > 0.05


def test_blocked_inverse_matches_dense():
    rng = np.random.default_rng(10)
    for n in (16, 37, 64):
        A = np.tril(rng.uniform(-0.5, 0.5, (n, n)), -1)
        X = blocked_unit_lower_inverse(A, 16)
        np.testing.assert_allclose(X, np.linalg.inv(np.eye(n) + A), rtol=0, atol=1e-10)


@pytest.mark.parametrize("C", [16, 64, 200])
@pytest.mark.parametrize("la_range", [(-3.0, -0.01), (-5.5, -4.9)])
def test_chunk_form_matches_oracle(oracle_mod, C, la_range):
    rng = np.random.default_rng(11 + C)
    T, dk, dv = 200, 16, 12
    q, k, v, la, b = _rand_inputs(rng, T, dk, dv, la_lo=la_range[0], la_hi=la_range[1])
    s0 = rng.standard_normal((dk, dv))
    ref = oracle_mod.kda_seq(q, k, v, la, b, s0=s0, want_transition=True)
    O, S, M = chunk_forward(q, k, v, la, b, s0, C=C, want_transition=True)
    np.testing.assert_allclose(O, ref["o"], rtol=0, atol=1e-10)
    np.testing.assert_allclose(S, ref["state"], rtol=0, atol=1e-10)
    np.testing.assert_allclose(M, ref["transition"], rtol=0, atol=1e-10)


def test_tile_anchor_bound_at_the_floor():
    # 16 steps at the floor in one tile: the largest inverse factor is exp(80.09) < bf16 max
    lam = np.full((64, 4), math.log(0.0067))
    g = np.cumsum(lam, axis=0)
    worst = 0.0
    for i0 in range(0, 64, 16):
        b = g[i0 - 1] if i0 else np.zeros(4)
        worst = max(worst, float(np.max(b - g[i0:i0 + 16])))
    assert abs(worst - (-16 * math.log(0.0067))) < 1e-9
    assert math.exp(worst) < torch.finfo(torch.bfloat16).max


def test_e4m3_codes_match_library(oracle_mod):
    codes = torch.arange(256, dtype=torch.uint8)
    lib = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = np.array([oracle_mod.e4m3_value(c) for c in range(256)])
    np.testing.assert_array_equal(np.isnan(mine), np.isnan(lib))
    ok = ~np.isnan(lib)
    np.testing.assert_array_equal(mine[ok], lib[ok])
    np.testing.assert_array_equal(np.signbit(mine[ok]), np.signbit(lib[ok]))


def test_e8m0_codes_match_library(oracle_mod):
    codes = torch.arange(256, dtype=torch.uint8)
    lib = codes.view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    mine = np.array([oracle_mod.e8m0_value(c) for c in range(256)])
    np.testing.assert_array_equal(np.isnan(mine), np.isnan(lib))
    ok = ~np.isnan(lib)
    np.testing.assert_array_equal(mine[ok], lib[ok])


def test_mxfp8_format_facts(oracle_mod):
    block = None
    for line in open(os.path.join(GOLDEN, "mxfp8_format_facts.txt")):
        if not line.strip() or line.startswith("#"):
            continue
        kind, code, val = line.split()
        if kind == "block":
            block = int(val)
            continue
        got = (oracle_mod.e4m3_value if kind == "e4m3" else oracle_mod.e8m0_value)(int(code, 16))
        want = float(val)
        if math.isnan(want):
            assert math.isnan(got), (kind, code)
        else:
            assert got == want and math.copysign(1, got) == math.copysign(1, want), (kind, code, got)
    # one shared scale per 32 elements: a row of ones with four different scales decodes block by block
    assert block == 32
    codes = np.full((2, 128), 0x38, np.uint8)
    scales = np.array([[127, 128, 126, 130], [0, 254, 127, 120]], np.uint8)
    out = oracle_mod.mxfp8_decode(codes, scales, block)
    for r in range(2):
        for i in range(128):
            assert out[r, i] == 2.0 ** (int(scales[r, i // block]) - 127)


def test_mxfp8_decode_is_scale_times_element(oracle_mod):
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 256, (3, 7, 64)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x3A           # no NaN codes
    scales = rng.integers(100, 140, (3, 7, 2)).astype(np.uint8)
    out = oracle_mod.mxfp8_decode(codes, scales)
    elem = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    scl = torch.from_numpy(scales).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    np.testing.assert_array_equal(out, elem * np.repeat(scl, 32, axis=-1))


def test_resuming_from_a_state_continues_the_sequence(oracle_mod):
    # T tokens, then n more from the state they leave, is the run over T + n tokens: outputs, states and
    # transition (the step map is applied token by token, so the split point changes nothing)
    rng = np.random.default_rng(17)
    T, n, dk, dv = 23, 9, 6, 5
    q, k, v, la, b = _rand_inputs(rng, T + n, dk, dv)
    s0 = rng.standard_normal((dk, dv))
    full = oracle_mod.kda_seq(q, k, v, la, b, s0=s0, marks=[T], want_transition=True)
    head = oracle_mod.kda_seq(q[:T], k[:T], v[:T], la[:T], b[:T], s0=s0, want_transition=True)
    tail = oracle_mod.kda_seq(q[T:], k[T:], v[T:], la[T:], b[T:], s0=head["state"], want_transition=True)
    np.testing.assert_array_equal(full["marks"][0], head["state"])
    np.testing.assert_allclose(np.concatenate([head["o"], tail["o"]]), full["o"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(tail["state"], full["state"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(tail["transition"] @ head["transition"], full["transition"], rtol=0, atol=1e-12)
