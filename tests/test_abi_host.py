"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every entry point that
include/kda.h declares, computes the checkpoint table, sizes its workspace, and rejects bad
arguments before launching anything."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import kda_linear_attention_02_b200 as kda
from kda_linear_attention_02_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kda._load()


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "kda.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    syms = _declared_symbols()
    assert len(syms) >= 10
    for s in syms:
        assert hasattr(lib, s), f"libkda.so does not export {s}"
    # and nothing else leaks out besides the declared entry points
    assert ctypes.CDLL(kda.lib_path()).kda_version() != 0


def test_version_and_status_strings(lib):
    assert "sm_100a" in kda.kda_version()
    assert kda.kda_status_string(0) == "KDA_OK"
    assert kda.kda_status_string(-5) == "KDA_ERR_TIMEOUT"
    assert kda.kda_status_string(-7) == "KDA_ERR_DEVICE_INPUT"


def _brute_ckpt_cu(cu, stride):
    out = [0]
    for i in range(len(cu) - 1):
        L = cu[i + 1] - cu[i]
        out.append(out[-1] + sum(1 for j in range(1, L + 1) if j % stride == 0))
    return out


@pytest.mark.parametrize("stride", [64, 512, 1024])
def test_ckpt_offsets_bit_exact(lib, stride):
    from kda_linear_attention_02_b200 import synth
    lengths = synth.varlen_lengths(64, 1024, 65536, 1) + [0, 511, 512, 513, 1]
    cu = synth.cu_from_lengths(lengths).tolist()
    got = kda.kda_ckpt_offsets(cu, stride).tolist()
    assert got == _brute_ckpt_cu(cu, stride)


def test_ckpt_offsets_rejects_bad_tables(lib):
    with pytest.raises(kda.KDAError):
        kda.kda_ckpt_offsets([0, 10, 5], 64)
    with pytest.raises(kda.KDAError):
        kda.kda_ckpt_offsets([1, 10], 64)
    with pytest.raises(kda.KDAError):
        kda.kda_ckpt_offsets([0, 10], 0)


def test_varlen_lengths_recipe():
    from kda_linear_attention_02_b200 import synth
    L = synth.varlen_lengths(64, 1024, 65536, 1)
    assert len(L) == 64 and min(L) >= 1024 and max(L) <= 65536
    assert L == synth.varlen_lengths(64, 1024, 65536, 1)


def test_workspace_sizes(lib):
    full = kda.kda_chunk_fwd_workspace_bytes(4 * 4096, 4, 32, 128, 128, kda.KDA_BF16)
    mini = kda.kda_chunk_fwd_min_workspace_bytes(4, 32, 128, 128, kda.KDA_BF16)
    assert full > mini > 0
    assert kda.kda_chunk_fwd_workspace_bytes(100, 1, 2, 64, 64, kda.KDA_F32) > 0
    # unsupported combinations report 0
    assert kda.kda_chunk_fwd_workspace_bytes(100, 1, 2, 96, 64, kda.KDA_F32) == 0
    assert kda.kda_chunk_fwd_workspace_bytes(100, 1, 2, 64, 64, kda.KDA_BF16) == 0


def test_workspace_layout_matches_the_documented_one(lib):
    # workspace = chunk index (n + 1 int32, rounded to 256 B) + per chunk of the bound ceil(T / 64) + n:
    # H packet slots and one 8-byte chunk-table entry; the windowed minimum holds the carried states
    # [n, H, dk, dv + dk] fp32 (rounded to 256 B) and one chunk's worth.  A bf16 packet slot at dk = dv = 128
    # is 74,752 bytes.
    r256 = lambda x: (x + 255) // 256 * 256
    for n, H in [(1, 1), (4, 32), (7, 3)]:
        index = r256((n + 1) * 4)
        per_chunk = kda.kda_chunk_fwd_workspace_bytes(64 * 10, n, H, 128, 128, kda.KDA_BF16) - \
            kda.kda_chunk_fwd_workspace_bytes(64 * 9, n, H, 128, 128, kda.KDA_BF16)
        assert per_chunk == H * 74752 + 8
        for T in (0, 1, 64, 65, 4096, 100000):
            ub = (T + 63) // 64 + n
            assert kda.kda_chunk_fwd_workspace_bytes(T, n, H, 128, 128, kda.KDA_BF16) == index + ub * per_chunk
            assert kda.kda_chunk_fwd_workspace_bytes(T, n, H, 128, 128, kda.KDA_MXFP8) == index + ub * per_chunk
        carry = r256(n * H * 128 * (128 + 128) * 4)
        assert kda.kda_chunk_fwd_min_workspace_bytes(n, H, 128, 128, kda.KDA_BF16) == index + carry + per_chunk
        for dt, dk, dv in [(kda.KDA_BF16, 128, 64), (kda.KDA_F32, 64, 64), (kda.KDA_F32, 128, 128), (kda.KDA_F32, 64, 128)]:
            pc = kda.kda_chunk_fwd_workspace_bytes(640, n, H, dk, dv, dt) - kda.kda_chunk_fwd_workspace_bytes(576, n, H, dk, dv, dt)
            assert pc > 8 and (pc - 8) % H == 0
            assert kda.kda_chunk_fwd_min_workspace_bytes(n, H, dk, dv, dt) == index + r256(n * H * dk * (dv + dk) * 4) + pc


def _call_chunk(lib, **over):
    """Raw C call with fake (never dereferenced) pointers: all of these must fail on the host."""
    a = dict(q=0x1000, k=0x2000, v=0x3000, la=0x4000, b=0x5000, s0=None, cu=0x6000, n=2, T=100, H=4, dk=128,
             dv=128, dt=0, stride=0, o=0x7000, fs=None, ck=None, ckcu=None, tr=None, ws=0x10000, wsb=1 << 30)
    a.update(over)
    vp = ctypes.c_void_p
    return lib.kda_chunk_fwd(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["la"]), vp(a["b"]), vp(a["s0"]),
                             vp(a["cu"]), a["n"], a["T"], a["H"], a["dk"], a["dv"], a["dt"], a["stride"], vp(a["o"]),
                             vp(a["fs"]), vp(a["ck"]), vp(a["ckcu"]), vp(a["tr"]), vp(a["ws"]), a["wsb"], None)


def test_chunk_fwd_host_argument_errors(lib):
    assert _call_chunk(lib, H=0) == -1
    assert _call_chunk(lib, n=-1) == -1
    assert _call_chunk(lib, T=-5) == -1
    assert _call_chunk(lib, dt=7) == -1
    assert _call_chunk(lib, dk=96) == -3
    assert _call_chunk(lib, dk=64, dt=0) == -3            # bf16 path needs dk = 128
    assert _call_chunk(lib, stride=100, ck=0x8000, ckcu=0x9000) == -1   # not a multiple of 64
    assert _call_chunk(lib, stride=512) == -1             # checkpoints missing
    assert _call_chunk(lib, q=None) == -1
    assert _call_chunk(lib, cu=None) == -1
    assert _call_chunk(lib, ws=None) == -1
    assert _call_chunk(lib, q=0x1004) == -2               # misaligned
    assert _call_chunk(lib, ws=0x10010) == -2             # workspace must be 256-byte aligned
    assert _call_chunk(lib, wsb=100) == -6                # workspace too small
    assert _call_chunk(lib, n=0) == 0                     # empty batch: nothing to do


def test_decode_and_compose_host_argument_errors(lib):
    vp = ctypes.c_void_p
    ok = [vp(0x1000)] * 6
    assert lib.kda_recurrent_step(*ok, 1, 0, 128, 128, 0, vp(0x2000), None) == -1
    assert lib.kda_recurrent_step(*ok, 1, 1, 96, 128, 0, vp(0x2000), None) == -3
    assert lib.kda_recurrent_step(vp(0x1004), *ok[1:], 1, 1, 128, 128, 0, vp(0x2000), None) == -2
    assert lib.kda_recurrent_step(*ok, 0, 1, 128, 128, 0, vp(0x2000), None) == 0
    assert lib.kda_segment_compose(vp(0x1000), vp(0x2000), None, None, 1, 1, 1, 128, 128, vp(0x3000), None,
                                   None) == -1
    assert lib.kda_segment_compose(vp(0x1000), vp(0x2000), vp(0x4000), None, 1, 1, 1, 128, 80, vp(0x3000), None,
                                   None) == -3
    assert lib.kda_selftest_umma(vp(0x1000), vp(0x2000), vp(0x3000), 20, 0, None) == -1
    assert lib.kda_selftest_umma(vp(0x1000), vp(0x2000), vp(0x3000), 48, 1, None) == -1   # MN-major: n % 32
    assert lib.kda_selftest_umma(vp(0x1000), vp(0x2000), vp(0x3000), 64, 16, None) == -1  # unknown flag bit
    assert lib.kda_selftest_umma(vp(0x1000), vp(0x2000), vp(0x3000), 64, 10, None) == -1  # A in TMEM with M = 64
    assert lib.kda_selftest_umma(vp(0x1000), vp(0x2000), vp(0x3000), 64, 6, None) == -1   # A both in TMEM and MN-major
    # tensor-core rate diagnostic: shape limits and the cycles buffer are checked before any launch
    assert lib.kda_selftest_mma_rate(8, 64, 0, 16, vp(0x1000), 1, None) == -1       # n below 16
    assert lib.kda_selftest_mma_rate(160, 96, 0, 16, vp(0x1000), 1, None) == -1     # k not 64 or 128
    assert lib.kda_selftest_mma_rate(96, 64, 1, 16, vp(0x1000), 1, None) == -1      # MN-major needs n % 64 == 0
    assert lib.kda_selftest_mma_rate(128, 64, 2, 16, vp(0x1000), 1, None) == -1     # no A from TMEM here
    assert lib.kda_selftest_mma_rate(128, 64, 16, 16, vp(0x1000), 1, None) == -1    # unknown flag bit
    assert lib.kda_selftest_mma_rate(128, 64, 0, 0, vp(0x1000), 1, None) == -1      # no repetitions
    assert lib.kda_selftest_mma_rate(128, 64, 0, 16, None, 1, None) == -1
    assert lib.kda_selftest_mma_rate(128, 64, 0, 16, vp(0x1002), 1, None) == -2     # unaligned buffer


def test_speculative_decode_host_argument_errors(lib):
    vp = ctypes.c_void_p
    st, q, k, v, la, b, o, acc = (vp(0x1000 * (i + 1)) for i in range(8))
    # verify: (state, q, k, v, la, beta, n, n_draft, H, dk, dv, dtype, o, stream)
    assert lib.kda_decode_verify(st, q, k, v, la, b, 2, 0, 4, 128, 128, 0, o, None) == -1      # no drafts
    assert lib.kda_decode_verify(st, q, k, v, la, b, 2, 3, 0, 128, 128, 0, o, None) == -1      # no heads
    assert lib.kda_decode_verify(st, q, k, v, la, b, 2, 3, 4, 96, 128, 0, o, None) == -3       # dk
    assert lib.kda_decode_verify(st, q, k, v, la, b, 2, 3, 4, 128, 128, 5, o, None) == -1      # dtype
    assert lib.kda_decode_verify(vp(0x1004), q, k, v, la, b, 2, 3, 4, 128, 128, 0, o, None) == -2
    assert lib.kda_decode_verify(st, None, k, v, la, b, 2, 3, 4, 128, 128, 0, o, None) == -1
    assert lib.kda_decode_verify(st, q, k, v, la, b, 0, 3, 4, 128, 128, 0, o, None) == 0       # empty batch
    # commit: (state, k, v, la, beta, n_accept, n, n_draft, H, dk, dv, dtype, stream)
    assert lib.kda_decode_commit(st, k, v, la, b, None, 2, 3, 4, 128, 128, 0, None) == -1      # no counts
    assert lib.kda_decode_commit(st, k, v, la, b, acc, 2, -1, 4, 128, 128, 0, None) == -1
    assert lib.kda_decode_commit(st, k, v, la, b, vp(0x1002), 2, 3, 4, 128, 128, 0, None) == -2
    assert lib.kda_decode_commit(st, k, v, la, b, acc, 2, 3, 4, 64, 80, 1, None) == -3
    assert lib.kda_decode_commit(st, k, v, la, b, acc, 0, 3, 4, 128, 128, 0, None) == 0


def test_draft_layout_is_token_major_per_sequence():
    from kda_linear_attention_02_b200 import synth
    x = torch.arange(3 * 2 * 5).reshape(3, 2, 5)        # [n_draft=3, n=2, H=5]
    y = synth.draft_layout(x)
    assert y.shape == (6, 5)
    for i in range(2):
        for d in range(3):
            assert torch.equal(y[i * 3 + d], x[d, i])


def test_binding_checks_shapes_on_cpu_tensors(lib):
    q = torch.zeros(64, 2, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        kda.kda_chunk_fwd(q, q, q[:, :1], torch.zeros(64, 2, 128), torch.zeros(64, 2),
                          None, torch.tensor([0, 64], dtype=torch.int32), q)


def _call_mx(lib, **over):
    """kda_chunk_fwd_mxfp8 with fake (never dereferenced) pointers: all of these must fail on the host."""
    a = dict(q=0x1000, qs=0x1100, k=0x2000, ks=0x2100, v=0x3000, vs=0x3100, la=0x4000, b=0x5000, s0=None,
             cu=0x6000, n=2, T=100, H=4, dk=128, dv=128, stride=0, o=0x7000, fs=None, ck=None, ckcu=None, tr=None,
             ws=0x10000, wsb=1 << 30)
    a.update(over)
    vp = ctypes.c_void_p
    return lib.kda_chunk_fwd_mxfp8(vp(a["q"]), vp(a["qs"]), vp(a["k"]), vp(a["ks"]), vp(a["v"]), vp(a["vs"]),
                                   vp(a["la"]), vp(a["b"]), vp(a["s0"]), vp(a["cu"]), a["n"], a["T"], a["H"],
                                   a["dk"], a["dv"], a["stride"], vp(a["o"]), vp(a["fs"]), vp(a["ck"]),
                                   vp(a["ckcu"]), vp(a["tr"]), vp(a["ws"]), a["wsb"], None)


def test_mxfp8_chunk_fwd_host_argument_errors(lib):
    assert _call_mx(lib, dk=64) == -3                     # dk = 128 only, as the bf16 path
    assert _call_mx(lib, dv=96) == -3
    assert _call_mx(lib, qs=None) == -1                   # every scale array is required
    assert _call_mx(lib, vs=None) == -1
    assert _call_mx(lib, ks=0x2102) == -2                 # q/k scales: whole 4-byte rows
    assert _call_mx(lib, dv=64, vs=0x3101) == -2
    assert _call_mx(lib, q=0x1008) == -2                  # codes move by TMA: 16-byte aligned
    assert _call_mx(lib, H=0) == -1
    assert _call_mx(lib, wsb=100) == -6
    assert _call_mx(lib, n=0) == 0
    # kda_chunk_fwd cannot take MXFP8 (no scales); the workspace queries size it like bf16
    assert _call_chunk(lib, dt=2) == -1
    assert kda.kda_chunk_fwd_workspace_bytes(4096, 1, 32, 128, 128, kda.KDA_MXFP8) == \
        kda.kda_chunk_fwd_workspace_bytes(4096, 1, 32, 128, 128, kda.KDA_BF16)
    assert kda.kda_chunk_fwd_workspace_bytes(4096, 1, 32, 64, 64, kda.KDA_MXFP8) == 0


def test_mxfp8_quantizer_recipe():
    import oracle
    from kda_linear_attention_02_b200 import synth
    g = torch.Generator().manual_seed(3)
    x = torch.randn(7, 3, 128, generator=g) * torch.tensor([1e-3, 1.0, 40.0, 1e4]).repeat_interleave(32)
    x[0, 0, 32:64] = 0.0
    codes, scales = synth.mxfp8_quantize(x)
    assert codes.dtype == torch.uint8 and scales.shape == (7, 3, 4)
    assert int(scales[0, 0, 1]) == 127                    # an all-zero block gets scale 1.0
    dec = oracle.mxfp8_decode(codes.numpy(), scales.numpy())
    amax = x.reshape(7, 3, 4, 32).abs().amax(-1).numpy()
    # the largest element of a block lands in [256, 448] (or saturates at 448) after its scale
    X = 2.0 ** (scales.numpy().astype(np.int64) - 127)
    top = amax / X
    nz = amax > 0
    assert np.all((top[nz] >= 256) & (top[nz] < 512))
    # E4M3 rounding: relative error at most 2^-4 where the scaled value is a normal E4M3 number below
    # the largest one; above 448 it saturates to 448
    Xe = np.repeat(X, 32, axis=-1)
    xs = np.abs(x.numpy()) / Xe
    normal = (xs >= 2.0 ** -6) & (xs <= 448)
    err = np.abs(dec - x.numpy())[normal] / np.abs(x.numpy())[normal]
    assert err.max() <= 2.0 ** -4 + 1e-12
    sat = xs > 448
    assert np.all(np.abs(dec[sat]) == 448 * Xe[sat])


def test_mxfp8_decode_host_argument_errors(lib):
    vp = ctypes.c_void_p
    st, q, qs, k, ks, v, vs, la, b, o = (vp(0x1000 * (i + 1)) for i in range(10))
    call = lambda *a, **kw: lib.kda_recurrent_step_mxfp8(*a)
    assert call(st, q, qs, k, ks, v, vs, la, b, 2, 0, 128, 128, o, None) == -1        # no heads
    assert call(st, q, qs, k, ks, v, vs, la, b, 2, 4, 96, 128, o, None) == -3         # dk
    assert call(st, q, None, k, ks, v, vs, la, b, 2, 4, 128, 128, o, None) == -1      # a scale array missing
    assert call(vp(0x1004), q, qs, k, ks, v, vs, la, b, 2, 4, 128, 128, o, None) == -2
    assert call(st, q, qs, k, ks, v, vs, la, b, 2, 4, 128, 128, vp(0xA001), None) == -2   # o is bf16
    assert call(st, q, qs, k, ks, v, vs, la, b, 0, 4, 128, 128, o, None) == 0         # empty batch
