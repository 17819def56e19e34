"""fp64 CPU oracle of the KDA operator -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import this
package.  It shares no code with the CUDA path and never imports the product package.

The arithmetic lives in ``kda_oracle.c`` (plain loops in double; see its header for the recurrence
and the passages it follows).  This module only compiles it with gcc, loads it with ctypes and
marshals numpy arrays.  ctypes releases the GIL during a foreign call, so ``run_slices`` spreads
independent (sequence, head) slices over host threads.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "libkda_oracle.so")
_lib = None

_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, IEEE semantics: no -ffast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        lib.oracle_decay_floor.restype = ctypes.c_double
        lib.oracle_kda_seq.restype = ctypes.c_int
        lib.oracle_kda_seq.argtypes = [
            ctypes.c_long, ctypes.c_int, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_long, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p]
        lib.oracle_segment_compose.restype = ctypes.c_int
        lib.oracle_segment_compose.argtypes = [
            ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        lib.oracle_e4m3_value.restype = ctypes.c_double
        lib.oracle_e4m3_value.argtypes = [ctypes.c_ubyte]
        lib.oracle_e8m0_value.restype = ctypes.c_double
        lib.oracle_e8m0_value.argtypes = [ctypes.c_ubyte]
        lib.oracle_mxfp8_decode.restype = ctypes.c_int
        lib.oracle_mxfp8_decode.argtypes = [ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        del dp
        _lib = lib
    return _lib


def decay_floor() -> float:
    """ln(0.0067): the per-step log-decay floor, as the oracle computes it."""
    return _load().oracle_decay_floor()


def _ptr(a):
    return None if a is None else a.ctypes.data


def _f32(a, shape):
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    if a.shape != shape:
        raise ValueError(f"expected shape {shape}, got {a.shape}")
    return a


def kda_seq(q, k, v, log_alpha, beta, s0=None, *, marks=None, want_o=True,
            want_transition=False):
    """Sequential fp64 recurrence over one (sequence, head) slice.

    q, k, log_alpha: [T, dk]; v: [T, dv]; beta: [T]; s0: [dk, dv] or None (zero).
    Returns a dict with 'o' [T, dv] (if want_o), 'state' [dk, dv], 'marks' [n, dk, dv] (states after
    marks[i] tokens) and 'transition' [dk, dk] (if asked).
    """
    q = np.asarray(q)
    T, dk = q.shape
    dv = np.asarray(v).shape[1]
    q = _f32(q, (T, dk)); k = _f32(k, (T, dk)); v = _f32(v, (T, dv))
    la = _f32(log_alpha, (T, dk)); b = _f32(beta, (T,))
    s0d = None if s0 is None else np.ascontiguousarray(np.asarray(s0, dtype=np.float64).reshape(dk, dv))
    o = np.empty((T, dv), np.float64) if want_o else None
    st = np.empty((dk, dv), np.float64)
    if marks is not None and len(marks):
        mk = np.ascontiguousarray(np.asarray(marks, dtype=np.int64))
        if np.any(np.diff(mk) <= 0) or mk[0] < 0 or mk[-1] > T:
            raise ValueError("marks must be strictly increasing in [0, T]")
        ms = np.empty((len(mk), dk, dv), np.float64)
    else:
        mk, ms = None, None
    tr = np.empty((dk, dk), np.float64) if want_transition else None
    rc = _load().oracle_kda_seq(T, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(s0d),
                                _ptr(o), _ptr(st), 0 if mk is None else len(mk), _ptr(mk), _ptr(ms),
                                _ptr(tr))
    if rc != 0:
        raise RuntimeError("oracle_kda_seq failed")
    out = {"state": st}
    if want_o:
        out["o"] = o
    if mk is not None:
        out["marks"] = ms
    if want_transition:
        out["transition"] = tr
    return out


def e4m3_value(code: int) -> float:
    """Value of one FP8 E4M3 code (OCP MX v1.0 element type)."""
    return _load().oracle_e4m3_value(int(code))


def e8m0_value(code: int) -> float:
    """Value of one E8M0 shared-scale code (OCP MX v1.0)."""
    return _load().oracle_e8m0_value(int(code))


def mxfp8_decode(codes, scales, block=32):
    """MXFP8 -> float64: codes uint8 [..., d], scales uint8 [..., d / block] (one scale per `block`
    consecutive elements of the last axis)."""
    codes = np.ascontiguousarray(np.asarray(codes, dtype=np.uint8))
    scales = np.ascontiguousarray(np.asarray(scales, dtype=np.uint8))
    d = codes.shape[-1]
    n = codes.size // d if d else 0
    if d % block or scales.shape[:-1] != codes.shape[:-1] or scales.shape[-1] != d // block:
        raise ValueError("scales must be [..., d / block]")
    out = np.empty(codes.shape, np.float64)
    if out.size and _load().oracle_mxfp8_decode(n, d, block, _ptr(codes), _ptr(scales), _ptr(out)) != 0:
        raise RuntimeError("oracle_mxfp8_decode failed")
    return out


def segment_compose(M, Z, x0=None):
    """X_0 = x0, X_{s+1} = M_s X_s + Z_s for one (sequence, head).  Returns (starts, end)."""
    M = np.ascontiguousarray(np.asarray(M, dtype=np.float64))
    Z = np.ascontiguousarray(np.asarray(Z, dtype=np.float64))
    nseg, dk, dv = Z.shape
    if M.shape != (nseg, dk, dk):
        raise ValueError("M must be [nseg, dk, dk]")
    x0d = None if x0 is None else np.ascontiguousarray(np.asarray(x0, dtype=np.float64).reshape(dk, dv))
    starts = np.empty((nseg, dk, dv), np.float64)
    end = np.empty((dk, dv), np.float64)
    rc = _load().oracle_segment_compose(nseg, dk, dv, _ptr(M), _ptr(Z), _ptr(x0d), _ptr(starts), _ptr(end))
    if rc != 0:
        raise RuntimeError("oracle_segment_compose failed")
    return starts, end


def run_slices(jobs, threads=None):
    """Run kda_seq over many independent slices on host threads.

    jobs: iterable of (key, kwargs-dict for kda_seq).  Returns {key: result}.
    """
    threads = threads or len(os.sched_getaffinity(0))
    jobs = list(jobs)
    with ThreadPoolExecutor(max_workers=threads) as ex:
        futs = {key: ex.submit(lambda kw: kda_seq(**kw), kw) for key, kw in jobs}
        return {key: f.result() for key, f in futs.items()}


def threads_used(threads=None) -> int:
    return threads or len(os.sched_getaffinity(0))
