"""fp64 CPU oracle for exact attention -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` use
this package.  It computes the plain three-step definition of attention (scores, softmax,
weighted sum of values; "FlashAttention 与高效注意力内核" tutorial, section 标准注意力三步)
and its analytic gradients in double precision, in C (``attn_oracle.c``), and shares no
code with the CUDA library.  Inputs are upcast to float64 exactly (bf16 and fp32 values
are representable in fp64).

Layouts follow the library's: q/o/do/dq ``[T, Hq, d]``, k/v/dk/dv ``[T, Hkv, d]``,
lse ``[Hq, T]``; ``cu_seqlens`` is an int32 prefix-sum array with a leading 0.
"""
import ctypes
import os

import numpy as np

from .build import build as _build

_lib = None


def _load():
    if _lib is None:
        _bind(ctypes.CDLL(_build()))
    return _lib


def _bind(lib):
    global _lib
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int32)
    up = ctypes.POINTER(ctypes.c_uint8)
    i32, f64 = ctypes.c_int32, ctypes.c_double
    lib.oracle_attn_fwd.argtypes = [dp, dp, dp, ip, i32, i32, i32, i32, f64, i32, up, dp, dp, i32]
    lib.oracle_attn_fwd.restype = ctypes.c_int
    lib.oracle_attn_bwd.argtypes = [dp, dp, dp, dp, ip, i32, i32, i32, i32, f64, i32,
                                    up, up, dp, dp, dp, dp, dp, i32]
    lib.oracle_attn_bwd.restype = ctypes.c_int
    lib.oracle_attn_bwd_ex.argtypes = [dp, dp, dp, dp, ip, i32, i32, i32, i32, f64, i32,
                                       up, up, dp, dp, dp, dp, dp, dp, dp, i32]
    lib.oracle_attn_bwd_ex.restype = ctypes.c_int
    lib.oracle_attn_probs.argtypes = [dp, dp, i32, i32, f64, i32, dp, dp]
    lib.oracle_attn_fwd_cross.argtypes = [dp, dp, dp, ip, ip, i32, i32, i32, i32, f64, i32, dp, dp, i32]
    lib.oracle_attn_fwd_fp8sim.argtypes = [dp, dp, dp, ip, i32, i32, i32, i32, f64, i32, i32, dp, dp, i32]
    lib.oracle_round_e4m3.argtypes = [f64]
    lib.oracle_round_e4m3.restype = f64
    lib.oracle_attn_probs.restype = ctypes.c_int
    _lib = lib


class using_library:
    """Temporarily route every oracle call through another build of ``attn_oracle.c``
    (the mutation tests load deliberately broken copies this way)."""

    def __init__(self, path):
        self.path = path

    def __enter__(self):
        global _lib
        self.saved = _load()
        _lib = None
        _bind(ctypes.CDLL(self.path))
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def _f64(x):
    """Any array-like (numpy, torch CPU tensor of any float dtype) -> contiguous float64."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().float().numpy() if str(x.dtype) == "torch.bfloat16" else x.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a, t=ctypes.c_double):
    return a.ctypes.data_as(ctypes.POINTER(t)) if a is not None else None


def _cu(cu_seqlens, total):
    if cu_seqlens is None:
        return np.array([0, total], dtype=np.int32)
    return np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))


def _sel(sel, total):
    if sel is None:
        return None
    s = np.zeros(total, dtype=np.uint8)
    s[np.asarray(sel, dtype=np.int64)] = 1
    return s


def attn_fwd(q, k, v, cu_seqlens=None, scale=None, causal=False, rows=None, threads=None):
    """O [T,Hq,d] and LSE [Hq,T] (float64).  ``cu_seqlens=None`` means one sequence.
    ``rows`` (optional token indices) limits which rows are computed; others are NaN."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, hq, d = q.shape
    hkv = k.shape[1]
    cu = _cu(cu_seqlens, T)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.full((T, hq, d), np.nan)
    lse = np.full((hq, T), np.nan)
    sel = _sel(rows, T)
    rc = _load().oracle_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(cu, ctypes.c_int32), len(cu) - 1,
                                 hq, hkv, d, float(scale), int(bool(causal)), _ptr(sel, ctypes.c_uint8),
                                 _ptr(o), _ptr(lse), threads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle_attn_fwd failed with code {rc}")
    return o, lse


def attn_fwd_cross(q, k, v, cu_q, cu_k, scale=None, causal=False, threads=None):
    """Decoding-shaped forward: sequence b has cu_q[b+1]-cu_q[b] query rows (the last
    positions of the sequence) and cu_k[b+1]-cu_k[b] keys.  O [Tq,Hq,d], LSE [Hq,Tq]
    (float64); under ``causal`` query row i sees keys j <= Lk - Lq + i."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    Tq, hq, d = q.shape
    hkv = k.shape[1]
    cq = np.ascontiguousarray(np.asarray(cu_q, dtype=np.int32))
    ck = np.ascontiguousarray(np.asarray(cu_k, dtype=np.int32))
    if len(cq) != len(ck) or cq[-1] != Tq or ck[-1] != k.shape[0]:
        raise ValueError("cu_q / cu_k do not match the tensors")
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.full((Tq, hq, d), np.nan)
    lse = np.full((hq, Tq), np.nan)
    rc = _load().oracle_attn_fwd_cross(_ptr(q), _ptr(k), _ptr(v), _ptr(cq, ctypes.c_int32), _ptr(ck, ctypes.c_int32),
                                       len(cq) - 1, hq, hkv, d, float(scale), int(bool(causal)), _ptr(o), _ptr(lse),
                                       threads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle_attn_fwd_cross failed with code {rc}")
    return o, lse


def round_e4m3(x: float) -> float:
    """x rounded to the nearest e4m3 value (ties to even), saturating at +-448."""
    return float(_load().oracle_round_e4m3(float(x)))


def attn_fwd_fp8sim(q, k, v, cu_seqlens=None, scale=None, causal=False, round_p=True, threads=None):
    """The FP8 forward's steps on dequantised Q, K, V: blockwise online softmax (128-key
    blocks, running max moved only past 8 log2 units) with the probabilities that
    multiply V rounded to e4m3.  round_p=False is the exact forward."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, hq, d = q.shape
    hkv = k.shape[1]
    cu = _cu(cu_seqlens, T)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.full((T, hq, d), np.nan)
    lse = np.full((hq, T), np.nan)
    rc = _load().oracle_attn_fwd_fp8sim(_ptr(q), _ptr(k), _ptr(v), _ptr(cu, ctypes.c_int32), len(cu) - 1, hq, hkv, d,
                                        float(scale), int(bool(causal)), int(bool(round_p)), _ptr(o), _ptr(lse),
                                        threads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle_attn_fwd_fp8sim failed with code {rc}")
    return o, lse


def attn_bwd(q, k, v, do, cu_seqlens=None, scale=None, causal=False, rows=None, keys=None,
             threads=None, o=None, lse=None):
    """dQ [T,Hq,d], dK, dV [T,Hkv,d], and the oracle's own O, LSE (float64).
    ``rows`` / ``keys`` (optional token indices) limit which dQ rows / dK,dV keys are
    produced; the others are NaN.  ``o`` [T,Hq,d] / ``lse`` [Hq,T] (optional) are the
    forward's saved outputs: D is then formed from ``o`` and P from ``lse`` (the backward
    as a function of its inputs); without them the result is the exact gradient."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    T, hq, d = q.shape
    hkv = k.shape[1]
    cu = _cu(cu_seqlens, T)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    dq = np.full((T, hq, d), np.nan)
    dk = np.full((T, hkv, d), np.nan)
    dv = np.full((T, hkv, d), np.nan)
    rsel, ksel = _sel(rows, T), _sel(keys, T)
    o_in = None if o is None else _f64(o)
    lse_in = None if lse is None else _f64(lse)
    o_out = np.empty((T, hq, d))
    lse_out = np.empty((hq, T))
    rc = _load().oracle_attn_bwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(cu, ctypes.c_int32),
                                    len(cu) - 1, hq, hkv, d, float(scale), int(bool(causal)),
                                    _ptr(rsel, ctypes.c_uint8), _ptr(ksel, ctypes.c_uint8),
                                    _ptr(o_in), _ptr(lse_in),
                                    _ptr(dq), _ptr(dk), _ptr(dv), _ptr(o_out), _ptr(lse_out),
                                    threads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle_attn_bwd failed with code {rc}")
    return dq, dk, dv, o_out, lse_out


def attn_probs(q, k, scale=None, causal=False):
    """The probability matrix P [n,n] and LSE [n] of one (sequence, head): q, k [n,d]."""
    q, k = _f64(q), _f64(k)
    n, d = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    p = np.empty((n, n))
    lse = np.empty(n)
    rc = _load().oracle_attn_probs(_ptr(q), _ptr(k), n, d, float(scale), int(bool(causal)),
                                   _ptr(p), _ptr(lse))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_probs failed with code {rc}")
    return p, lse
