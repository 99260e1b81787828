"""attn_bwd_noalloc: the backward for callers that cannot allocate device memory.

Some callers cannot give the library a workspace where they run the backward: engines
that reserve all of their device memory at start-up and may not allocate afterwards
(cudaMalloc can synchronise the device, stall, or fail once a caching allocator holds the
free memory), and plain C hosts with no allocator of their own.  attn_bwd_noalloc serves
them from a fixed 64 MiB scratch array inside the library.

The GPU test runs it twice in a row (every call reuses the same scratch, so the second
call must not see the first one's leftovers) and holds each call to the fp64 oracle's
gradients at the backward's tolerance, and to attn_bwd (which takes a workspace): dK and
dV bit for bit (one CTA owns each key tile and sums in a fixed order), dQ to within one
bf16 rounding per element (its fp32 partial sums arrive from several CTAs in an order
that varies from run to run).  It also checks that no device memory is taken: neither
torch's allocator nor cudaMemGetInfo sees a change across the second call.  The CPU
tests check that a problem too large for the scratch, and malformed calls, are refused
on the host before anything touches the GPU.

This file sorts last so that, in a run that stops at the first failure, every other test
has already run."""
import ctypes

import numpy as np
import pytest
import torch

import attn_workloads as W
import io_aware_exact_qk_b200 as attn
from tests import parity as P


def _call(lib, **kw):
    a = dict(q=16, k=16, v=16, o=16, do=16, lse=16, cu=None, batch=1, seqlen=8, max_seqlen=8, total=8, hq=2, hkv=2,
             d=128, scale=0.088, causal=0, dtype=attn.ATTN_BF16, dq=16, dk=16, dv=16)
    a.update(kw)
    vp = ctypes.c_void_p
    return lib.attn_bwd_noalloc(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["o"]), vp(a["do"]), vp(a["lse"]),
                                vp(a["cu"]), a["batch"], a["seqlen"], a["max_seqlen"], a["total"], a["hq"], a["hkv"],
                                a["d"], a["scale"], a["causal"], a["dtype"], vp(a["dq"]), vp(a["dk"]), vp(a["dv"]),
                                None)


def test_too_large_problem_is_refused_on_the_host():
    lib = attn.load_library()
    T = 1 << 20                            # needs about 8.6 GB of scratch
    st = _call(lib, batch=1, seqlen=T, max_seqlen=T, total=T, hq=16, hkv=16)
    assert st == attn.ATTN_ERR_INVALID_ARG
    assert b"64 MiB" in lib.attn_last_error_message()


@pytest.mark.parametrize("kw,status", [
    (dict(hq=3, hkv=2), attn.ATTN_ERR_UNSUPPORTED),
    (dict(q=None), attn.ATTN_ERR_INVALID_ARG),
    (dict(dv=0x1008), attn.ATTN_ERR_INVALID_ARG),
    (dict(batch=-1, total=-8), attn.ATTN_ERR_INVALID_ARG),
    (dict(total=9), attn.ATTN_ERR_INVALID_ARG),
    (dict(d=96), attn.ATTN_ERR_UNSUPPORTED),
])
def test_malformed_calls_are_refused_before_the_gpu(kw, status):
    """Validation runs before the scratch address is looked up: on a machine without a GPU
    a well-sized but malformed call still gets its argument error, not a CUDA error."""
    lib = attn.load_library()
    assert _call(lib, **kw) == status
    assert lib.attn_last_error_message() != b""


@pytest.mark.gpu
def test_no_alloc_backward_matches_oracle_and_workspace_backward_twice():
    w = W.custom("noalloc", [300, 77, 513], 8, 2, 128, True, seed=91)
    q, k, v, do, cu = W.make_inputs(w)
    qd, kd, vd, dod, cud = (t.cuda() for t in (q, k, v, do, cu))
    kw = dict(cu_seqlens=cud, max_seqlen=w.max_seqlen, scale=w.scale, causal=True)
    o, lse = attn.attn_fwd(qd, kd, vd, **kw)
    ref_ws = [P.to_np(t) for t in attn.attn_bwd(qd, kd, vd, o, dod, lse, **kw)]
    ref_or = P.oracle_bwd(w, q, k, v, do, cu)[:3]
    torch.cuda.synchronize()
    for call in range(2):
        dq, dk, dv = (torch.full_like(t, float("nan")) for t in (qd, kd, vd))
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        before_torch = torch.cuda.memory_allocated()
        before_free = torch.cuda.mem_get_info()[0]
        attn.attn_bwd_noalloc(qd, kd, vd, o, dod, lse, dq=dq, dk=dk, dv=dv, **kw)
        attn.attn_get_device_error()
        if call == 1:   # the first call may load the module; the second must take nothing
            assert torch.cuda.memory_allocated() == before_torch
            assert torch.cuda.mem_get_info()[0] == before_free
        got = [P.to_np(t) for t in (dq, dk, dv)]
        P.check_grads_bf16(got, ref_or, tag=f"call {call}")
        assert np.array_equal(got[1], ref_ws[1]) and np.array_equal(got[2], ref_ws[2]), f"call {call}: dK/dV"
        # dQ: at most one bf16 rounding step apart element by element (bf16 spacing = fp32
        # spacing * 2^16), with a floor of a few fp32 roundings of the largest partial sum
        # for elements that cancel to nearly zero
        ulp = np.spacing(np.abs(ref_ws[0]).astype(np.float32)).astype(np.float64) * 2 ** 16
        floor = 1e-5 * np.abs(ref_ws[0]).max()
        assert (np.abs(got[0] - ref_ws[0]) <= np.maximum(ulp, floor)).all(), f"call {call}: dQ"
        assert P.rel_l2(got[0], ref_ws[0]) <= 1e-3, f"call {call}: dQ"
