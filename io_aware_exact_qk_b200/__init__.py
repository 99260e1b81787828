"""io_aware_exact_qk_b200 -- exact scaled-dot-product attention on one B200 (sm_100a).

A thin ctypes binding over ``libattn.so`` (declared in ``include/attn.h``).  The functions
carry the C ABI's names and only marshal arguments: tensors are PyTorch device tensors
(PyTorch is used for device memory and streams), every step of the computation runs in
the library's CUDA kernels, and there is no CPU or library fallback -- if the shared
library is missing or fails to load, every call raises.

    o, lse = attn_fwd(q, k, v, cu_seqlens=None, max_seqlen=None, scale=None, causal=False)
    dq, dk, dv = attn_bwd(q, k, v, o, do, lse, ...)

Layouts: q, o, do, dq ``[T, Hq, d]``; k, v, dk, dv ``[T, Hkv, d]``; lse ``[Hq, T]`` fp32;
cu_seqlens int32 ``[B+1]`` on the device (varlen), or ``None`` with ``batch`` equal-length
sequences of ``T // batch`` tokens.
"""
import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIBRARY_PATH = os.path.join(_HERE, "libattn.so")

ATTN_OK, ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED, ATTN_ERR_CUDA, ATTN_ERR_TIMEOUT = range(5)
ATTN_BF16, ATTN_FP32 = 0, 1

_lib = None


class AttnError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"{message} (status {status})")
        self.status = status


def load_library():
    """Load libattn.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIBRARY_PATH):
        raise RuntimeError(f"{LIBRARY_PATH} is missing; build it with `python -m io_aware_exact_qk_b200.build`")
    lib = ctypes.CDLL(LIBRARY_PATH)
    vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    lib.attn_fwd.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, f32, i32, i32, vp, vp, vp, sz, vp]
    lib.attn_fwd.restype = ctypes.c_int
    lib.attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, f32, i32, i32,
                             vp, vp, vp, vp, sz, vp]
    lib.attn_bwd.restype = ctypes.c_int
    for name in ("attn_fwd_workspace_size", "attn_bwd_workspace_size"):
        fn = getattr(lib, name)
        fn.argtypes = [i32] * 7
        fn.restype = sz
    lib.attn_get_device_error.argtypes = [vp]
    lib.attn_get_device_error.restype = ctypes.c_int
    lib.attn_status_string.argtypes = [ctypes.c_int]
    lib.attn_status_string.restype = ctypes.c_char_p
    lib.attn_last_error_message.argtypes = []
    lib.attn_last_error_message.restype = ctypes.c_char_p
    lib.attn_version.argtypes = []
    lib.attn_version.restype = i32
    lib.attn_profile_enable.argtypes = [i32]
    lib.attn_profile_enable.restype = ctypes.c_int
    lib.attn_profile_kernel_count.argtypes = []
    lib.attn_profile_kernel_count.restype = i32
    lib.attn_profile_kernel_name.argtypes = [i32]
    lib.attn_profile_kernel_name.restype = ctypes.c_char_p
    lib.attn_profile_collect.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64), i32]
    lib.attn_profile_collect.restype = ctypes.c_int
    lib.attn_bwd_accumulate.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, f32, i32,
                                        vp, vp, vp, vp, sz, vp]
    lib.attn_bwd_accumulate.restype = ctypes.c_int
    lib.attn_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, f32, i32, i32,
                                     vp, vp, vp, vp]
    lib.attn_bwd_noalloc.restype = ctypes.c_int
    lib.attn_fwd_decode.argtypes = [vp, vp, vp, vp, vp] + [i32] * 10 + [f32, i32, i32, vp, vp, vp, sz, vp]
    lib.attn_fwd_decode.restype = ctypes.c_int
    lib.attn_fwd_decode_workspace_size.argtypes = [i32] * 10
    lib.attn_fwd_decode_workspace_size.restype = sz
    lib.attn_merge_partial.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, vp]
    lib.attn_merge_partial.restype = ctypes.c_int
    lib.attn_merge_finish.argtypes = [vp, vp, i32, i32, i32, vp]
    lib.attn_merge_finish.restype = ctypes.c_int
    lib.attn_fp8_quantize.argtypes = [vp, vp, vp] + [i32] * 5 + [vp] * 6 + [vp]
    lib.attn_fp8_quantize.restype = ctypes.c_int
    lib.attn_fwd_fp8.argtypes = [vp] * 6 + [i32] * 5 + [f32, i32, vp, vp, vp, sz, vp]
    lib.attn_fwd_fp8.restype = ctypes.c_int
    lib.attn_fwd_bwd_host_scratch_size.argtypes = [i32] * 5
    lib.attn_fwd_bwd_host_scratch_size.restype = sz
    lib.attn_fwd_bwd_host.argtypes = [vp] * 5 + [i32] * 7 + [f32, i32] + [vp] * 6 + [sz, vp]
    lib.attn_fwd_bwd_host.restype = ctypes.c_int
    lib.attn_fp8_quantize_varlen.argtypes = [vp, vp, vp, vp] + [i32] * 6 + [vp] * 6 + [vp]
    lib.attn_fp8_quantize_varlen.restype = ctypes.c_int
    lib.attn_fwd_fp8_varlen.argtypes = [vp] * 7 + [i32] * 6 + [f32, i32, vp, vp, vp, sz, vp]
    lib.attn_fwd_fp8_varlen.restype = ctypes.c_int
    lib.attn_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.attn_set_wait_limit_ns.restype = ctypes.c_int
    lib.attn_get_wait_limit_ns.argtypes = []
    lib.attn_get_wait_limit_ns.restype = ctypes.c_uint64
    lib.attn_selftest_wait.argtypes = [i32, vp]
    lib.attn_selftest_wait.restype = ctypes.c_int
    lib.attn_selftest_exp2.argtypes = [vp, vp, vp, ctypes.c_int64, vp]
    lib.attn_selftest_exp2.restype = ctypes.c_int
    lib.attn_launch_count.argtypes = []
    lib.attn_launch_count.restype = ctypes.c_int64
    _lib = lib
    return lib


def _check(status):
    if status != ATTN_OK:
        lib = load_library()
        msg = lib.attn_last_error_message().decode() or lib.attn_status_string(status).decode()
        raise AttnError(status, msg)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return ATTN_BF16
    if t.dtype == torch.float32:
        return ATTN_FP32
    raise AttnError(ATTN_ERR_UNSUPPORTED, f"dtype {t.dtype} is not supported (bf16, or fp32 check mode)")


def _shape_args(q, k, cu_seqlens, max_seqlen, batch):
    T, hq, d = q.shape
    hkv = k.shape[1]
    if cu_seqlens is None:
        batch = 1 if batch is None else int(batch)
        seqlen = T // batch if batch > 0 else 0
        max_seqlen = seqlen
    else:
        batch = cu_seqlens.numel() - 1
        seqlen = 0
        if max_seqlen is None:
            raise AttnError(ATTN_ERR_INVALID_ARG, "varlen calls need max_seqlen")
    return batch, seqlen, int(max_seqlen), T, hq, hkv, d


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def workspace_size(kind, q, k, cu_seqlens=None, max_seqlen=None, batch=None):
    """Bytes of workspace attn_fwd ("fwd") or attn_bwd ("bwd") needs."""
    lib = load_library()
    b, _, ms, T, hq, hkv, d = _shape_args(q, k, cu_seqlens, max_seqlen, batch)
    fn = lib.attn_fwd_workspace_size if kind == "fwd" else lib.attn_bwd_workspace_size
    return int(fn(b, ms, T, hq, hkv, d, _dtype_code(q)))


def attn_fwd(q, k, v, cu_seqlens=None, max_seqlen=None, scale=None, causal=False, batch=None,
             o=None, lse=None, workspace=None, stream=None):
    """Forward.  Returns (o [T,Hq,d], lse [Hq,T] fp32)."""
    lib = load_library()
    b, seqlen, ms, T, hq, hkv, d = _shape_args(q, k, cu_seqlens, max_seqlen, batch)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(hq, T, dtype=torch.float32, device=q.device)
    ws = workspace_size("fwd", q, k, cu_seqlens, max_seqlen, batch)
    if ws and workspace is None:
        workspace = torch.empty(ws, dtype=torch.uint8, device=q.device)
    _check(lib.attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), b, seqlen, ms, T, hq, hkv, d,
                        float(scale), int(bool(causal)), _dtype_code(q), _ptr(o), _ptr(lse),
                        _ptr(workspace), ws if workspace is not None else 0, _stream(stream)))
    return o, lse


def attn_bwd(q, k, v, o, do, lse, cu_seqlens=None, max_seqlen=None, scale=None, causal=False, batch=None,
             dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Backward.  Returns (dq [T,Hq,d], dk [T,Hkv,d], dv [T,Hkv,d])."""
    lib = load_library()
    b, seqlen, ms, T, hq, hkv, d = _shape_args(q, k, cu_seqlens, max_seqlen, batch)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    ws = workspace_size("bwd", q, k, cu_seqlens, max_seqlen, batch)
    if ws and workspace is None:
        workspace = torch.empty(ws, dtype=torch.uint8, device=q.device)
    _check(lib.attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(cu_seqlens), b, seqlen,
                        ms, T, hq, hkv, d, float(scale), int(bool(causal)), _dtype_code(q), _ptr(dq), _ptr(dk),
                        _ptr(dv), _ptr(workspace), ws if workspace is not None else 0, _stream(stream)))
    return dq, dk, dv


def attn_bwd_accumulate(q, k, v, o, do, lse, dq_acc, dk_acc, dv_acc, cu_seqlens=None, max_seqlen=None, scale=None,
                        causal=False, batch=None, workspace=None, stream=None):
    """Backward that ADDS its gradients into the float32 tensors dq_acc [T,Hq,d], dk_acc,
    dv_acc [T,Hkv,d] (bf16 inputs); returns them."""
    lib = load_library()
    b, seqlen, ms, T, hq, hkv, d = _shape_args(q, k, cu_seqlens, max_seqlen, batch)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    for t in (dq_acc, dk_acc, dv_acc):
        if t.dtype != torch.float32:
            raise AttnError(ATTN_ERR_INVALID_ARG, "the accumulators must be float32")
    ws = workspace_size("bwd", q, k, cu_seqlens, max_seqlen, batch)
    if ws and workspace is None:
        workspace = torch.empty(ws, dtype=torch.uint8, device=q.device)
    _check(lib.attn_bwd_accumulate(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(cu_seqlens), b,
                                   seqlen, ms, T, hq, hkv, d, float(scale), int(bool(causal)), _ptr(dq_acc),
                                   _ptr(dk_acc), _ptr(dv_acc), _ptr(workspace), ws if workspace is not None else 0,
                                   _stream(stream)))
    return dq_acc, dk_acc, dv_acc


def attn_bwd_noalloc(q, k, v, o, do, lse, cu_seqlens=None, max_seqlen=None, scale=None, causal=False,
                     batch=None, dq=None, dk=None, dv=None, stream=None):
    """Backward for callers that cannot allocate device memory when they run it (engines
    that reserve all device memory up front, hosts with no allocator to give a
    workspace from).  Same results as attn_bwd; the scratch is the library's built-in
    64 MiB array, so larger problems are refused and concurrent calls on one device race.
    (dq/dk/dv are allocated here only when not passed in.)"""
    lib = load_library()
    b, seqlen, ms, T, hq, hkv, d = _shape_args(q, k, cu_seqlens, max_seqlen, batch)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check(lib.attn_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(cu_seqlens), b,
                                seqlen, ms, T, hq, hkv, d, float(scale), int(bool(causal)), _dtype_code(q),
                                _ptr(dq), _ptr(dk), _ptr(dv), _stream(stream)))
    return dq, dk, dv


def _decode_shape(q, k, cu_q, cu_k, max_seqlen_q, max_seqlen_k, batch):
    Tq, hq, d = q.shape
    Tk, hkv = k.shape[0], k.shape[1]
    if (cu_q is None) != (cu_k is None):
        raise ValueError("give both cu_seqlens_q and cu_seqlens_k, or neither")
    if cu_q is None:
        if batch is None:
            raise ValueError("batch mode needs batch=")
        sq, sk = Tq // batch if batch else 0, Tk // batch if batch else 0
        return batch, sq, sk, sq, sk, Tq, Tk, hq, hkv, d
    if max_seqlen_q is None or max_seqlen_k is None:
        raise ValueError("varlen mode needs max_seqlen_q= and max_seqlen_k=")
    return len(cu_q) - 1, 0, 0, int(max_seqlen_q), int(max_seqlen_k), Tq, Tk, hq, hkv, d


def decode_workspace_size(q, k, cu_seqlens_q=None, cu_seqlens_k=None, max_seqlen_q=None, max_seqlen_k=None,
                          batch=None, num_splits=0):
    b, _, _, mq, mk, Tq, Tk, hq, hkv, d = _decode_shape(q, k, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                                                        max_seqlen_k, batch)
    return int(load_library().attn_fwd_decode_workspace_size(b, mq, mk, Tq, Tk, hq, hkv, d,
                                                             int(cu_seqlens_q is not None), int(num_splits)))


def attn_fwd_decode(q, k, v, cu_seqlens_q=None, cu_seqlens_k=None, max_seqlen_q=None, max_seqlen_k=None,
                    scale=None, causal=False, batch=None, num_splits=0, o=None, lse=None, workspace=None,
                    stream=None):
    """Split-KV decoding forward: sequence b has Lq query rows (the newest positions) and Lk
    keys.  Returns (o [Tq,Hq,d] bf16, lse [Hq,Tq] fp32)."""
    lib = load_library()
    b, sq, sk, mq, mk, Tq, Tk, hq, hkv, d = _decode_shape(q, k, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                                                          max_seqlen_k, batch)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(hq, Tq, dtype=torch.float32, device=q.device)
    ws = int(lib.attn_fwd_decode_workspace_size(b, mq, mk, Tq, Tk, hq, hkv, d, int(cu_seqlens_q is not None),
                                                int(num_splits)))
    if ws and workspace is None:
        workspace = torch.empty(ws, dtype=torch.uint8, device=q.device)
    _check(lib.attn_fwd_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), b, sq, sk, mq, mk,
                               Tq, Tk, hq, hkv, d, float(scale), int(bool(causal)), int(num_splits), _ptr(o),
                               _ptr(lse), _ptr(workspace), workspace.numel() if workspace is not None else 0,
                               _stream(stream)))
    return o, lse


def attn_merge_partial(o_acc, lse_acc, o_part, lse_part, first=False, stream=None):
    """Folds a bf16 partial (o_part [T,Hq,d], lse_part [Hq,T]) over a disjoint key set into
    the float32 accumulators o_acc [T,Hq,d], lse_acc [Hq,T] (first=True: start from it)."""
    T, hq, d = o_part.shape
    _check(load_library().attn_merge_partial(_ptr(o_acc), _ptr(lse_acc), _ptr(o_part), _ptr(lse_part), T, hq, d,
                                             int(bool(first)), _stream(stream)))


def attn_merge_finish(o_acc, o=None, stream=None):
    """bf16 copy of the accumulated O."""
    T, hq, d = o_acc.shape
    if o is None:
        o = torch.empty(o_acc.shape, dtype=torch.bfloat16, device=o_acc.device)
    _check(load_library().attn_merge_finish(_ptr(o_acc), _ptr(o), T, hq, d, _stream(stream)))
    return o


def fp8_vt_pitch(seqlen):
    """Token pitch of the transposed e4m3 V: the longest sequence rounded up to a multiple
    of 16."""
    return (int(seqlen) + 15) // 16 * 16


def attn_fp8_quantize(q, k, v, batch=None, cu_seqlens=None, max_seqlen=None, stream=None):
    """Per-head e4m3 operands of the FP8 forward from bf16 q [T, Hq, d], k, v [T, Hkv, d]
    (d = 64 or 128; `batch` sequences of T / batch tokens, or the packed sequences of
    cu_seqlens with max_seqlen): returns (q8, k8 as uint8 [T, H, d], vt8 uint8
    [batch Hkv, d, fp8_vt_pitch(max_seqlen)], descale_q [Hq], descale_k [Hkv],
    descale_v [Hkv] float32)."""
    lib = load_library()
    b, seqlen, ms, T, hq, hkv, d = _shape_args(q, k, cu_seqlens, max_seqlen, batch)
    dev = q.device
    q8 = torch.empty(q.shape, dtype=torch.uint8, device=dev)
    k8 = torch.empty(k.shape, dtype=torch.uint8, device=dev)
    vt8 = torch.empty(b * hkv, d, fp8_vt_pitch(ms), dtype=torch.uint8, device=dev)
    ds = [torch.empty(n, dtype=torch.float32, device=dev) for n in (hq, hkv, hkv)]
    outs = (_ptr(q8), _ptr(k8), _ptr(vt8), _ptr(ds[0]), _ptr(ds[1]), _ptr(ds[2]), _stream(stream))
    if cu_seqlens is None:
        _check(lib.attn_fp8_quantize(_ptr(q), _ptr(k), _ptr(v), b, seqlen, hq, hkv, d, *outs))
    else:
        _check(lib.attn_fp8_quantize_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), b, ms, T, hq, hkv, d, *outs))
    return q8, k8, vt8, ds[0], ds[1], ds[2]


def attn_fwd_fp8(q8, k8, vt8, descale_q, descale_k, descale_v, batch=None, scale=None, causal=False, o=None, lse=None,
                 workspace=None, stream=None, cu_seqlens=None, max_seqlen=None):
    """FP8 forward on attn_fp8_quantize's operands (the same batch, or the same cu_seqlens
    and max_seqlen).  Returns (o [T, Hq, d] bf16, lse [Hq, T] fp32)."""
    lib = load_library()
    b, seqlen, ms, T, hq, hkv, d = _shape_args(q8, k8, cu_seqlens, max_seqlen, batch)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if o is None:
        o = torch.empty(T, hq, d, dtype=torch.bfloat16, device=q8.device)
    if lse is None:
        lse = torch.empty(hq, T, dtype=torch.float32, device=q8.device)
    ws = int(lib.attn_fwd_workspace_size(b, ms, T, hq, hkv, d, 0))
    if ws and workspace is None:
        workspace = torch.empty(ws, dtype=torch.uint8, device=q8.device)
    operands = (_ptr(q8), _ptr(k8), _ptr(vt8), _ptr(descale_q), _ptr(descale_k), _ptr(descale_v))
    tail = (float(scale), int(bool(causal)), _ptr(o), _ptr(lse), _ptr(workspace),
            ws if workspace is not None else 0, _stream(stream))
    if cu_seqlens is None:
        _check(lib.attn_fwd_fp8(*operands, b, seqlen, hq, hkv, d, *tail))
    else:
        _check(lib.attn_fwd_fp8_varlen(*operands, _ptr(cu_seqlens), b, ms, T, hq, hkv, d, *tail))
    return o, lse


def attn_get_device_error(stream=None):
    """Synchronise the stream and raise if a kernel reported a device-side error."""
    _check(load_library().attn_get_device_error(_stream(stream)))


def attn_set_wait_limit_ns(ns):
    """Bound (ns of wall time) on every pipeline wait of the library's kernels, current device."""
    _check(load_library().attn_set_wait_limit_ns(int(ns)))


def attn_get_wait_limit_ns():
    return int(load_library().attn_get_wait_limit_ns())


def attn_selftest_wait(arrive, stream=None):
    """One CTA waits on a barrier with the library's bounded wait; without `arrive` the wait
    runs out and attn_get_device_error() raises with ATTN_ERR_TIMEOUT."""
    _check(load_library().attn_selftest_wait(int(bool(arrive)), _stream(stream)))


def attn_selftest_exp2(x, stream=None):
    """(y_fma, y_sfu): the forward's FMA-pipe 2^x and the special-function unit's 2^x of the
    float32 device tensor x."""
    x = x.contiguous()
    y_fma, y_sfu = torch.empty_like(x), torch.empty_like(x)
    _check(load_library().attn_selftest_exp2(_ptr(x), _ptr(y_fma), _ptr(y_sfu), x.numel(), _stream(stream)))
    return y_fma, y_sfu


def attn_version():
    return int(load_library().attn_version())


def attn_profile_enable(on=True):
    """Turn per-launch CUDA-event timing of the library's kernels on or off."""
    _check(load_library().attn_profile_enable(int(bool(on))))


def attn_profile_collect():
    """{kernel name: (total ms, launches)} for the launches timed since the last collect."""
    lib = load_library()
    n = lib.attn_profile_kernel_count()
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int64 * n)()
    _check(lib.attn_profile_collect(ms, cnt, n))
    return {lib.attn_profile_kernel_name(i).decode(): (ms[i], cnt[i]) for i in range(n) if cnt[i]}


def attn_launch_count():
    """Kernel launches made by the library since it was loaded."""
    return int(load_library().attn_launch_count())


def attn_fwd_bwd_host(q, k, v, do, cu_seqlens=None, max_seqlen=None, scale=None, causal=False, batch=None,
                      out=None, scratch=None, stream=None):
    """Forward and backward on HOST tensors (bf16 q [T,Hq,d], k, v [T,Hkv,d], do [T,Hq,d],
    ideally pinned; cu_seqlens a host int32 tensor or None) through the library's own
    copy/compute pipeline.  Returns ((o, lse, dq, dk, dv) host tensors, scratch); ``out``
    may hold those five host tensors (pinned) and ``scratch`` the device scratch from a
    previous call."""
    lib = load_library()
    b, seqlen, ms, T, hq, hkv, d = _shape_args(q, k, cu_seqlens, max_seqlen, batch)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = (torch.empty(q.shape, dtype=q.dtype, pin_memory=True),
               torch.empty(hq, T, dtype=torch.float32, pin_memory=True),
               torch.empty(q.shape, dtype=q.dtype, pin_memory=True),
               torch.empty(k.shape, dtype=k.dtype, pin_memory=True),
               torch.empty(v.shape, dtype=v.dtype, pin_memory=True))
    need = int(lib.attn_fwd_bwd_host_scratch_size(b, T, hq, hkv, d))
    if scratch is None:
        scratch = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
    cu = None if cu_seqlens is None else cu_seqlens.to(torch.int32).contiguous()
    o, lse, dq, dk, dv = out
    _check(lib.attn_fwd_bwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(cu), b, seqlen, ms, T, hq, hkv, d,
                                 float(scale), int(bool(causal)), _ptr(o), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
                                 _ptr(scratch), scratch.numel(), _stream(stream)))
    return out, scratch


def attention_host(q, k, v, do, cu_seqlens=None, max_seqlen=None, scale=None, causal=False, batch=None,
                   stream=None, out=None):
    """attn_fwd_bwd_host with its buffers kept in a dict: returns ((o, lse, dq, dk, dv) on
    the host, bufs); passing ``out=bufs`` from a previous call reuses the pinned outputs and
    the device scratch."""
    bufs = out if out is not None else {}
    res, bufs["scratch"] = attn_fwd_bwd_host(q, k, v, do, cu_seqlens, max_seqlen, scale, causal, batch,
                                             out=bufs.get("host"), scratch=bufs.get("scratch"), stream=stream)
    bufs["host"] = res
    return res, bufs
