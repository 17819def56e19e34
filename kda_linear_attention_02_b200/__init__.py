"""kda_linear_attention_02_b200 -- Kimi Delta Attention (KDA) on one NVIDIA B200.

A thin Python binding over the C ABI of ``libkda.so`` (see ``include/kda.h``).  Every function here
has the name of the C entry point it calls and only marshals arguments: it checks shapes, dtypes
and devices of torch tensors, turns them into raw pointers and passes the current CUDA stream.  All
of the operator's arithmetic runs in the library's CUDA kernels; there is no fallback.  If the
library has not been built the import of any entry point fails loudly.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "KDA_BF16", "KDA_F32", "KDA_MXFP8", "KDA_CHUNK", "KDAError", "lib_path",
    "kda_chunk_fwd_workspace_bytes", "kda_chunk_fwd_min_workspace_bytes", "kda_chunk_fwd", "kda_chunk_fwd_mxfp8",
    "kda_chunk_fwd_noalloc",
    "kda_recurrent_step", "kda_recurrent_step_mxfp8", "kda_decode_verify", "kda_decode_commit", "kda_segment_compose", "kda_ckpt_offsets", "kda_get_device_status",
    "kda_status_string", "kda_version", "kda_profile_begin", "kda_profile_end", "kda_selftest_wait_timeout",
    "kda_selftest_umma", "KDA_SELFTEST_B_MN_MAJOR", "KDA_SELFTEST_A_TMEM", "kda_selftest_mma_rate", "KDA_PREFIX_BLOCK", "kda_prefix_block_hashes", "kda_prefix_cache_create",
    "kda_prefix_cache_destroy", "kda_prefix_cache_lookup", "kda_prefix_cache_plan", "kda_prefix_cache_insert",
    "kda_prefix_cache_commit", "kda_prefix_cache_abort", "kda_prefix_cache_release", "kda_prefix_cache_stats",
    "KDA_PREFIX_NO_SLOT", "KDA_PREFIX_STORED",
]

KDA_BF16 = 0
KDA_F32 = 1
KDA_MXFP8 = 2
KDA_PREFIX_BLOCK = 512
KDA_PREFIX_NO_SLOT = -1     # kda_prefix_cache_insert: no slot could be given for that block end
KDA_PREFIX_STORED = -2      # kda_prefix_cache_insert: that block end already has a checkpoint slot
KDA_CHUNK = 64

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libkda.so")
_lib = None


class KDAError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {kda_status_string(status)} ({status})")
        self.status = status


def lib_path() -> str:
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"libkda.so is not built ({_LIB_PATH}); run "
                           "`python -m kda_linear_attention_02_b200.build` (needs nvcc)")
    L = ctypes.CDLL(_LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    L.kda_chunk_fwd_workspace_bytes.restype = sz
    L.kda_chunk_fwd_workspace_bytes.argtypes = [i64, i32, i32, i32, i32, i32]
    L.kda_chunk_fwd_min_workspace_bytes.restype = sz
    L.kda_chunk_fwd_min_workspace_bytes.argtypes = [i32, i32, i32, i32, i32]
    L.kda_chunk_fwd.restype = i32
    L.kda_chunk_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32, i32,
                                vp, vp, vp, vp, vp, vp, sz, vp]
    L.kda_chunk_fwd_mxfp8.restype = i32
    L.kda_chunk_fwd_mxfp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32,
                                      vp, vp, vp, vp, vp, vp, sz, vp]
    L.kda_chunk_fwd_noalloc.restype = i32
    L.kda_chunk_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32, i32,
                                        vp, vp, vp, vp, vp, vp]
    L.kda_recurrent_step.restype = i32
    L.kda_recurrent_step.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, vp]
    L.kda_recurrent_step_mxfp8.restype = i32
    L.kda_recurrent_step_mxfp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, vp, vp]
    L.kda_decode_verify.restype = i32
    L.kda_decode_verify.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, vp]
    L.kda_decode_commit.restype = i32
    L.kda_decode_commit.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp]
    u64, i64p = ctypes.c_uint64, ctypes.POINTER(ctypes.c_int64)
    L.kda_prefix_block_hashes.restype = i64
    L.kda_prefix_block_hashes.argtypes = [vp, i64, u64, vp]
    L.kda_prefix_cache_create.restype = i32
    L.kda_prefix_cache_create.argtypes = [i64, i32, i32, ctypes.POINTER(vp)]
    L.kda_prefix_cache_destroy.restype = None
    L.kda_prefix_cache_destroy.argtypes = [vp]
    L.kda_prefix_cache_lookup.restype = i32
    L.kda_prefix_cache_lookup.argtypes = [vp, vp, i64, i64p, i64p, ctypes.POINTER(i32)]
    L.kda_prefix_cache_plan.restype = i64
    L.kda_prefix_cache_plan.argtypes = [vp, i64, i64, vp, i64]
    L.kda_prefix_cache_insert.restype = i32
    L.kda_prefix_cache_insert.argtypes = [vp, vp, i64, vp, i64, vp]
    for name in ("kda_prefix_cache_commit", "kda_prefix_cache_abort"):
        getattr(L, name).restype = i32
        getattr(L, name).argtypes = [vp, vp, i64]
    L.kda_prefix_cache_release.restype = i32
    L.kda_prefix_cache_release.argtypes = [vp, i32]
    L.kda_prefix_cache_stats.restype = i32
    L.kda_prefix_cache_stats.argtypes = [vp, i64p, ctypes.POINTER(i32)]
    L.kda_segment_compose.restype = i32
    L.kda_segment_compose.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, vp, vp]
    L.kda_ckpt_offsets.restype = i32
    L.kda_ckpt_offsets.argtypes = [vp, i32, i32, vp]
    L.kda_get_device_status.restype = i32
    L.kda_get_device_status.argtypes = [vp]
    L.kda_status_string.restype = ctypes.c_char_p
    L.kda_status_string.argtypes = [i32]
    L.kda_version.restype = ctypes.c_char_p
    L.kda_version.argtypes = []
    L.kda_profile_begin.restype = i32
    L.kda_profile_begin.argtypes = [i32]
    L.kda_profile_end.restype = i32
    L.kda_profile_end.argtypes = [vp, vp, vp, vp]
    L.kda_selftest_wait_timeout.restype = i32
    L.kda_selftest_wait_timeout.argtypes = [i32, vp]
    L.kda_selftest_mma_rate.restype = i32
    L.kda_selftest_mma_rate.argtypes = [i32, i32, i32, i32, vp, i32, vp]
    L.kda_selftest_umma.restype = i32
    L.kda_selftest_umma.argtypes = [vp, vp, vp, i32, i32, vp]
    _lib = L
    return L


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    if t.dtype == torch.float32:
        return KDA_F32
    raise TypeError(f"q/k/v/o must be bfloat16 or float32, got {t.dtype}")


def _need(t, name, shape=None, dtype=None, device=None):
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name}: expected device {device}, got {t.device}")


def _opt(t, name, shape, dtype, device):
    if t is not None:
        _need(t, name, shape, dtype, device)


def _check(st: int, where: str):
    if st != 0:
        raise KDAError(st, where)


def kda_status_string(status: int) -> str:
    return _load().kda_status_string(int(status)).decode()


def kda_version() -> str:
    return _load().kda_version().decode()


def kda_chunk_fwd_workspace_bytes(total_tokens, n_seqs, H, dk, dv, dtype=KDA_BF16) -> int:
    return int(_load().kda_chunk_fwd_workspace_bytes(int(total_tokens), int(n_seqs), int(H), int(dk), int(dv),
                                                     int(dtype)))


def kda_chunk_fwd_min_workspace_bytes(n_seqs, H, dk, dv, dtype=KDA_BF16) -> int:
    return int(_load().kda_chunk_fwd_min_workspace_bytes(int(n_seqs), int(H), int(dk), int(dv), int(dtype)))


def kda_chunk_fwd(q, k, v, log_alpha, beta, initial_state, cu_seqlens, o, final_state=None, *,
                  ckpt_stride=0, checkpoints=None, ckpt_cu=None, final_transition=None, workspace=None,
                  stream=None):
    """Chunked KDA forward over a packed batch (C: kda_chunk_fwd).

    q, k, log_alpha [T,H,dk]; v, o [T,H,dv]; beta [T,H]; cu_seqlens int32 [N+1] (device);
    initial_state / final_state [N,H,dk,dv] fp32 or None; checkpoints [*,H,dk,dv] fp32 with
    ckpt_cu int32 [N+1] (device); final_transition [N,H,dk,dk] fp32 or None; workspace: uint8
    device tensor (allocated here from torch's allocator when None).  Outputs are written in place.
    """
    _need(q, "q")
    dev = q.device
    T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    n = cu_seqlens.numel() - 1
    _need(k, "k", (T, H, dk), q.dtype, dev)
    _need(v, "v", (T, H, dv), q.dtype, dev)
    _need(o, "o", (T, H, dv), q.dtype, dev)
    _need(log_alpha, "log_alpha", (T, H, dk), torch.float32, dev)
    _need(beta, "beta", (T, H), torch.float32, dev)
    _need(cu_seqlens, "cu_seqlens", (n + 1,), torch.int32, dev)
    _opt(initial_state, "initial_state", (n, H, dk, dv), torch.float32, dev)
    _opt(final_state, "final_state", (n, H, dk, dv), torch.float32, dev)
    _opt(final_transition, "final_transition", (n, H, dk, dk), torch.float32, dev)
    if ckpt_stride:
        _need(checkpoints, "checkpoints", None, torch.float32, dev)
        if checkpoints.dim() != 4 or tuple(checkpoints.shape[1:]) != (H, dk, dv):
            raise ValueError("checkpoints must be [n_ckpt, H, dk, dv]")
        _need(ckpt_cu, "ckpt_cu", (n + 1,), torch.int32, dev)
    if workspace is None:
        nbytes = kda_chunk_fwd_workspace_bytes(T, n, H, dk, dv, dt)
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
    _need(workspace, "workspace", None, torch.uint8, dev)
    st = _load().kda_chunk_fwd(_p(q), _p(k), _p(v), _p(log_alpha), _p(beta), _p(initial_state), _p(cu_seqlens),
                               n, T, H, dk, dv, dt, int(ckpt_stride), _p(o), _p(final_state),
                               _p(checkpoints if ckpt_stride else None), _p(ckpt_cu if ckpt_stride else None),
                               _p(final_transition), _p(workspace), workspace.numel(), _stream(stream))
    _check(st, "kda_chunk_fwd")
    return o


def _bytes_of(t, name, shape, dev, kinds):
    """A uint8 (or same-size float8) tensor of the given shape, as raw bytes."""
    if t is None:
        raise ValueError(f"{name} is required")
    if t.dtype not in kinds:
        raise TypeError(f"{name}: expected one of {kinds}, got {t.dtype}")
    _need(t, name, shape, None, dev)


def kda_chunk_fwd_mxfp8(q, q_scale, k, k_scale, v, v_scale, log_alpha, beta, initial_state, cu_seqlens, o,
                        final_state=None, *, ckpt_stride=0, checkpoints=None, ckpt_cu=None, final_transition=None,
                        workspace=None, stream=None):
    """Chunked KDA forward with MXFP8 q, k, v (C: kda_chunk_fwd_mxfp8).

    q, k [T,H,dk] and v [T,H,dv]: E4M3 codes (uint8 or torch.float8_e4m3fn); q_scale, k_scale [T,H,dk/32]
    and v_scale [T,H,dv/32]: E8M0 shared scales (uint8 or torch.float8_e8m0fnu), one per 32 channels.
    o [T,H,dv] bf16.  Everything else as kda_chunk_fwd.
    """
    codes = (torch.uint8, torch.float8_e4m3fn)
    scales = (torch.uint8, torch.float8_e8m0fnu)
    if q is None:
        raise ValueError("q is required")
    dev = q.device
    T, H, dk = q.shape
    dv = v.shape[-1]
    n = cu_seqlens.numel() - 1
    _bytes_of(q, "q", (T, H, dk), dev, codes)
    _bytes_of(k, "k", (T, H, dk), dev, codes)
    _bytes_of(v, "v", (T, H, dv), dev, codes)
    if dk % 32 or dv % 32:
        raise ValueError("dk and dv must be multiples of the 32-channel scale block")
    _bytes_of(q_scale, "q_scale", (T, H, dk // 32), dev, scales)
    _bytes_of(k_scale, "k_scale", (T, H, dk // 32), dev, scales)
    _bytes_of(v_scale, "v_scale", (T, H, dv // 32), dev, scales)
    _need(o, "o", (T, H, dv), torch.bfloat16, dev)
    _need(log_alpha, "log_alpha", (T, H, dk), torch.float32, dev)
    _need(beta, "beta", (T, H), torch.float32, dev)
    _need(cu_seqlens, "cu_seqlens", (n + 1,), torch.int32, dev)
    _opt(initial_state, "initial_state", (n, H, dk, dv), torch.float32, dev)
    _opt(final_state, "final_state", (n, H, dk, dv), torch.float32, dev)
    _opt(final_transition, "final_transition", (n, H, dk, dk), torch.float32, dev)
    if ckpt_stride:
        _need(checkpoints, "checkpoints", None, torch.float32, dev)
        if checkpoints.dim() != 4 or tuple(checkpoints.shape[1:]) != (H, dk, dv):
            raise ValueError("checkpoints must be [n_ckpt, H, dk, dv]")
        _need(ckpt_cu, "ckpt_cu", (n + 1,), torch.int32, dev)
    if workspace is None:
        nbytes = kda_chunk_fwd_workspace_bytes(T, n, H, dk, dv, KDA_MXFP8)
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
    _need(workspace, "workspace", None, torch.uint8, dev)
    st = _load().kda_chunk_fwd_mxfp8(_p(q), _p(q_scale), _p(k), _p(k_scale), _p(v), _p(v_scale), _p(log_alpha),
                                     _p(beta), _p(initial_state), _p(cu_seqlens), n, T, H, dk, dv, int(ckpt_stride),
                                     _p(o), _p(final_state), _p(checkpoints if ckpt_stride else None),
                                     _p(ckpt_cu if ckpt_stride else None), _p(final_transition), _p(workspace),
                                     workspace.numel(), _stream(stream))
    _check(st, "kda_chunk_fwd_mxfp8")
    return o


def kda_chunk_fwd_noalloc(q, k, v, log_alpha, beta, initial_state, cu_seqlens, o, final_state=None, *,
                          ckpt_stride=0, checkpoints=None, ckpt_cu=None, final_transition=None, stream=None):
    """kda_chunk_fwd for callers that may not allocate device memory (C: kda_chunk_fwd_noalloc).

    Same arguments and results as kda_chunk_fwd, without a workspace: the library uses its own
    fixed 64 MiB device array instead, so nothing is allocated here or in the library.  Calls that
    could overlap on the GPU share that array and must not be issued concurrently.
    """
    _need(q, "q")
    dev = q.device
    T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    n = cu_seqlens.numel() - 1
    _need(k, "k", (T, H, dk), q.dtype, dev)
    _need(v, "v", (T, H, dv), q.dtype, dev)
    _need(o, "o", (T, H, dv), q.dtype, dev)
    _need(log_alpha, "log_alpha", (T, H, dk), torch.float32, dev)
    _need(beta, "beta", (T, H), torch.float32, dev)
    _need(cu_seqlens, "cu_seqlens", (n + 1,), torch.int32, dev)
    _opt(initial_state, "initial_state", (n, H, dk, dv), torch.float32, dev)
    _opt(final_state, "final_state", (n, H, dk, dv), torch.float32, dev)
    _opt(final_transition, "final_transition", (n, H, dk, dk), torch.float32, dev)
    if ckpt_stride:
        _need(checkpoints, "checkpoints", None, torch.float32, dev)
        _need(ckpt_cu, "ckpt_cu", (n + 1,), torch.int32, dev)
    st = _load().kda_chunk_fwd_noalloc(_p(q), _p(k), _p(v), _p(log_alpha), _p(beta), _p(initial_state),
                                       _p(cu_seqlens), n, T, H, dk, dv, dt, int(ckpt_stride), _p(o),
                                       _p(final_state), _p(checkpoints if ckpt_stride else None),
                                       _p(ckpt_cu if ckpt_stride else None), _p(final_transition),
                                       _stream(stream))
    _check(st, "kda_chunk_fwd_noalloc")
    return o


def kda_recurrent_step(state, q, k, v, log_alpha, beta, o, *, stream=None):
    """One decode step, state [n,H,dk,dv] fp32 updated in place (C: kda_recurrent_step).

    q, k [n,H,dk]; v, o [n,H,dv] (bf16 or fp32); log_alpha [n,H,dk] fp32; beta [n,H] fp32.
    """
    _need(state, "state", None, torch.float32)
    dev = state.device
    n, H, dk, dv = state.shape
    dt = _dtype_code(q)
    _need(q, "q", (n, H, dk), q.dtype, dev)
    _need(k, "k", (n, H, dk), q.dtype, dev)
    _need(v, "v", (n, H, dv), q.dtype, dev)
    _need(o, "o", (n, H, dv), q.dtype, dev)
    _need(log_alpha, "log_alpha", (n, H, dk), torch.float32, dev)
    _need(beta, "beta", (n, H), torch.float32, dev)
    st = _load().kda_recurrent_step(_p(state), _p(q), _p(k), _p(v), _p(log_alpha), _p(beta), n, H, dk, dv, dt,
                                    _p(o), _stream(stream))
    _check(st, "kda_recurrent_step")
    return o


def kda_recurrent_step_mxfp8(state, q, q_scale, k, k_scale, v, v_scale, log_alpha, beta, o, *, stream=None):
    """One decode step with MXFP8 q, k, v (C: kda_recurrent_step_mxfp8).

    q, k [n,H,dk] and v [n,H,dv]: E4M3 codes (uint8 or torch.float8_e4m3fn); q_scale, k_scale [n,H,dk/32],
    v_scale [n,H,dv/32]: E8M0 scales (uint8 or torch.float8_e8m0fnu); o [n,H,dv] bf16; state as
    kda_recurrent_step.
    """
    _need(state, "state", None, torch.float32)
    dev = state.device
    n, H, dk, dv = state.shape
    codes = (torch.uint8, torch.float8_e4m3fn)
    scales = (torch.uint8, torch.float8_e8m0fnu)
    if dk % 32 or dv % 32:
        raise ValueError("dk and dv must be multiples of the 32-channel scale block")
    _bytes_of(q, "q", (n, H, dk), dev, codes)
    _bytes_of(k, "k", (n, H, dk), dev, codes)
    _bytes_of(v, "v", (n, H, dv), dev, codes)
    _bytes_of(q_scale, "q_scale", (n, H, dk // 32), dev, scales)
    _bytes_of(k_scale, "k_scale", (n, H, dk // 32), dev, scales)
    _bytes_of(v_scale, "v_scale", (n, H, dv // 32), dev, scales)
    _need(o, "o", (n, H, dv), torch.bfloat16, dev)
    _need(log_alpha, "log_alpha", (n, H, dk), torch.float32, dev)
    _need(beta, "beta", (n, H), torch.float32, dev)
    st = _load().kda_recurrent_step_mxfp8(_p(state), _p(q), _p(q_scale), _p(k), _p(k_scale), _p(v), _p(v_scale),
                                          _p(log_alpha), _p(beta), n, H, dk, dv, _p(o), _stream(stream))
    _check(st, "kda_recurrent_step_mxfp8")
    return o


def _draft_shapes(state, k, name="k"):
    _need(state, "state", None, torch.float32)
    n, H, dk, dv = state.shape
    if k.dim() != 3 or k.shape[1] != H or k.shape[2] != dk or (n > 0 and k.shape[0] % n):
        raise ValueError(f"{name}: expected [n*n_draft, {H}, {dk}] for n = {n}, got {tuple(k.shape)}")
    n_draft = k.shape[0] // n if n > 0 else 1
    return n, n_draft, H, dk, dv


def kda_decode_verify(state, q, k, v, log_alpha, beta, o, *, stream=None):
    """Outputs of n_draft draft tokens per sequence from the committed state (C: kda_decode_verify).

    state [n,H,dk,dv] fp32 (read only); drafts token-major, sequence i at rows i*n_draft ..:
    q, k [n*n_draft,H,dk]; v, o [n*n_draft,H,dv] (bf16 or fp32); log_alpha [n*n_draft,H,dk] fp32;
    beta [n*n_draft,H] fp32.
    """
    n, n_draft, H, dk, dv = _draft_shapes(state, k)
    dev = state.device
    dt = _dtype_code(q)
    T = n * n_draft
    _need(q, "q", (T, H, dk), q.dtype, dev)
    _need(k, "k", (T, H, dk), q.dtype, dev)
    _need(v, "v", (T, H, dv), q.dtype, dev)
    _need(o, "o", (T, H, dv), q.dtype, dev)
    _need(log_alpha, "log_alpha", (T, H, dk), torch.float32, dev)
    _need(beta, "beta", (T, H), torch.float32, dev)
    st = _load().kda_decode_verify(_p(state), _p(q), _p(k), _p(v), _p(log_alpha), _p(beta), n, n_draft, H, dk, dv,
                                   dt, _p(o), _stream(stream))
    _check(st, "kda_decode_verify")
    return o


def kda_decode_commit(state, k, v, log_alpha, beta, n_accept, *, stream=None):
    """State after the first n_accept[i] drafts of each sequence, in place (C: kda_decode_commit).

    Same draft layout as kda_decode_verify (q is not needed); n_accept int32 [n] on the device,
    each in 0..n_draft.
    """
    n, n_draft, H, dk, dv = _draft_shapes(state, k)
    dev = state.device
    dt = _dtype_code(k)
    T = n * n_draft
    _need(k, "k", (T, H, dk), k.dtype, dev)
    _need(v, "v", (T, H, dv), k.dtype, dev)
    _need(log_alpha, "log_alpha", (T, H, dk), torch.float32, dev)
    _need(beta, "beta", (T, H), torch.float32, dev)
    _need(n_accept, "n_accept", (n,), torch.int32, dev)
    st = _load().kda_decode_commit(_p(state), _p(k), _p(v), _p(log_alpha), _p(beta), _p(n_accept), n, n_draft, H,
                                   dk, dv, dt, _stream(stream))
    _check(st, "kda_decode_commit")
    return state


def kda_segment_compose(transitions, zero_states, seg_cu, init, start_states, end_states=None, *, stream=None):
    """Prefix scan X_{s+1} = M_s X_s + Z_s over each sequence's segments (C: kda_segment_compose).

    transitions [S,H,dk,dk]; zero_states, start_states [S,H,dk,dv]; seg_cu int32 [N+1] (device);
    init / end_states [N,H,dk,dv] or None.  All fp32.
    """
    _need(zero_states, "zero_states", None, torch.float32)
    dev = zero_states.device
    S, H, dk, dv = zero_states.shape
    n = seg_cu.numel() - 1
    _need(transitions, "transitions", (S, H, dk, dk), torch.float32, dev)
    _need(seg_cu, "seg_cu", (n + 1,), torch.int32, dev)
    _need(start_states, "start_states", (S, H, dk, dv), torch.float32, dev)
    _opt(init, "init", (n, H, dk, dv), torch.float32, dev)
    _opt(end_states, "end_states", (n, H, dk, dv), torch.float32, dev)
    st = _load().kda_segment_compose(_p(transitions), _p(zero_states), _p(seg_cu), _p(init), n, S, H, dk, dv,
                                     _p(start_states), _p(end_states), _stream(stream))
    _check(st, "kda_segment_compose")
    return start_states


def kda_ckpt_offsets(cu_seqlens_host, stride: int) -> torch.Tensor:
    """Host-only checkpoint offsets (C: kda_ckpt_offsets); returns an int32 CPU tensor [N+1]."""
    cu = torch.as_tensor(cu_seqlens_host, dtype=torch.int32).contiguous().cpu()
    n = cu.numel() - 1
    out = torch.empty(n + 1, dtype=torch.int32)
    _check(_load().kda_ckpt_offsets(_p(cu), n, int(stride), _p(out)), "kda_ckpt_offsets")
    return out


def kda_get_device_status(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device status word."""
    return int(_load().kda_get_device_status(_stream(stream)))


def kda_profile_begin(max_calls: int):
    """Record per-kernel CUDA events in the next max_calls kda_chunk_fwd calls (C: kda_profile_begin)."""
    _check(_load().kda_profile_begin(int(max_calls)), "kda_profile_begin")


def kda_profile_end():
    """Returns (ms_index, ms_prep, ms_state, n_calls) summed over the recorded calls (C: kda_profile_end)."""
    a, b, c, n = ctypes.c_float(), ctypes.c_float(), ctypes.c_float(), ctypes.c_int()
    _check(_load().kda_profile_end(ctypes.byref(a), ctypes.byref(b), ctypes.byref(c), ctypes.byref(n)),
           "kda_profile_end")
    return a.value, b.value, c.value, n.value


def kda_selftest_wait_timeout(limit_us: int = 2000, stream=None) -> int:
    return int(_load().kda_selftest_wait_timeout(int(limit_us), _stream(stream)))


def kda_selftest_mma_rate(n, k, *, b_mn_major=False, a_mn_major=False, m64=False, reps=256, grid=None, stream=None):
    """SM cycles per 128 x n x k bf16 tensor-core product, back to back and one at a time
    (C: kda_selftest_mma_rate): a float32 tensor [grid, 2] on the current device."""
    dev = torch.device("cuda", torch.cuda.current_device())
    if grid is None:
        grid = torch.cuda.get_device_properties(dev).multi_processor_count
    cyc = torch.empty(grid, 2, dtype=torch.float32, device=dev)
    majors = ((KDA_SELFTEST_B_MN_MAJOR if b_mn_major else 0) | (KDA_SELFTEST_A_MN_MAJOR if a_mn_major else 0) |
              (KDA_SELFTEST_M64 if m64 else 0))
    _check(_load().kda_selftest_mma_rate(int(n), int(k), majors, int(reps), _p(cyc), int(grid),
                                         _stream(stream)), "kda_selftest_mma_rate")
    return cyc


KDA_SELFTEST_B_MN_MAJOR = 1
KDA_SELFTEST_A_TMEM = 2
KDA_SELFTEST_A_MN_MAJOR = 4
KDA_SELFTEST_M64 = 8


def kda_selftest_umma(a, b, d, *, b_mn_major=False, a_tmem=False, a_mn_major=False, m64=False, stream=None):
    n = b.shape[0]
    _need(a, "a", (128, 64), torch.bfloat16)
    _need(b, "b", (n, 64), torch.bfloat16, a.device)
    _need(d, "d", (128, n), torch.float32, a.device)
    flags = ((KDA_SELFTEST_B_MN_MAJOR if b_mn_major else 0) | (KDA_SELFTEST_A_TMEM if a_tmem else 0) |
             (KDA_SELFTEST_A_MN_MAJOR if a_mn_major else 0) | (KDA_SELFTEST_M64 if m64 else 0))
    _check(_load().kda_selftest_umma(_p(a), _p(b), _p(d), n, flags, _stream(stream)), "kda_selftest_umma")
    return d


# ---------------------------------------------------------------------------------------------- prefix reuse
def _host_array(x, dtype):
    import numpy as np
    a = np.ascontiguousarray(x.cpu().numpy() if isinstance(x, torch.Tensor) else np.asarray(x), dtype=dtype)
    return a


def kda_prefix_block_hashes(tokens, seed=0):
    """Chained FNV-1a hashes of the full 512-token blocks of `tokens` (C: kda_prefix_block_hashes).
    Returns a numpy uint64 array of len(tokens) // 512 entries."""
    import numpy as np
    t = _host_array(tokens, np.int32)
    out = np.zeros(max(len(t) // KDA_PREFIX_BLOCK, 1), dtype=np.uint64)
    n = _load().kda_prefix_block_hashes(t.ctypes.data, len(t), int(seed) & (2 ** 64 - 1), out.ctypes.data)
    if n < 0:
        raise KDAError(-1, "kda_prefix_block_hashes")
    return out[:n]


def kda_prefix_cache_create(max_blocks, n_slots, unit_blocks):
    """Opaque prefix-reuse directory handle (C: kda_prefix_cache_create); free it with kda_prefix_cache_destroy."""
    h = ctypes.c_void_p()
    _check(_load().kda_prefix_cache_create(int(max_blocks), int(n_slots), int(unit_blocks), ctypes.byref(h)),
           "kda_prefix_cache_create")
    return h


def kda_prefix_cache_destroy(cache):
    _load().kda_prefix_cache_destroy(cache)


def kda_prefix_cache_lookup(cache, hashes):
    """(matched_blocks, resume_blocks, resume_slot) for a request's block hashes (C: kda_prefix_cache_lookup)."""
    import numpy as np
    h = _host_array(hashes, np.uint64)
    m, r, sl = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int32()
    _check(_load().kda_prefix_cache_lookup(cache, h.ctypes.data, len(h), ctypes.byref(m), ctypes.byref(r),
                                           ctypes.byref(sl)), "kda_prefix_cache_lookup")
    return m.value, r.value, sl.value


def kda_prefix_cache_plan(cache, n_blocks, resume_blocks):
    """Block ends after which a request stores its state (C: kda_prefix_cache_plan)."""
    import numpy as np
    n = _load().kda_prefix_cache_plan(cache, int(n_blocks), int(resume_blocks), None, 0)
    if n < 0:
        raise KDAError(-1, "kda_prefix_cache_plan")
    out = np.zeros(max(n, 1), dtype=np.int64)
    _load().kda_prefix_cache_plan(cache, int(n_blocks), int(resume_blocks), out.ctypes.data, n)
    return out[:n].tolist()


def kda_prefix_cache_insert(cache, hashes, ends):
    """Record a processed request; returns the slot of each planned end, -1 where none could be freed
    (C: kda_prefix_cache_insert)."""
    import numpy as np
    h = _host_array(hashes, np.uint64)
    e = _host_array(ends, np.int64)
    out = np.full(max(len(e), 1), -1, dtype=np.int32)
    _check(_load().kda_prefix_cache_insert(cache, h.ctypes.data, len(h), e.ctypes.data, len(e), out.ctypes.data),
           "kda_prefix_cache_insert")
    return out[:len(e)].tolist()


def _slot_array(slots):
    import numpy as np
    return np.ascontiguousarray(np.asarray(list(slots), dtype=np.int32))


def kda_prefix_cache_commit(cache, slots):
    """Mark the slots handed out by an insert as holding their copied states (C: kda_prefix_cache_commit)."""
    a = _slot_array(slots)
    _check(_load().kda_prefix_cache_commit(cache, a.ctypes.data if a.size else None, a.size),
           "kda_prefix_cache_commit")


def kda_prefix_cache_abort(cache, slots):
    """Give pending slots back when their copies will not happen (C: kda_prefix_cache_abort)."""
    a = _slot_array(slots)
    _check(_load().kda_prefix_cache_abort(cache, a.ctypes.data if a.size else None, a.size),
           "kda_prefix_cache_abort")


def kda_prefix_cache_release(cache, slot):
    """End the pin that a lookup put on its resume slot (C: kda_prefix_cache_release)."""
    _check(_load().kda_prefix_cache_release(cache, int(slot)), "kda_prefix_cache_release")


def kda_prefix_cache_stats(cache):
    """(cached block hashes, slots in use) (C: kda_prefix_cache_stats)."""
    nb, ns = ctypes.c_int64(), ctypes.c_int32()
    _check(_load().kda_prefix_cache_stats(cache, ctypes.byref(nb), ctypes.byref(ns)), "kda_prefix_cache_stats")
    return nb.value, ns.value
