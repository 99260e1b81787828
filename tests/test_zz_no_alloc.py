"""attn_bwd_noalloc: the backward for callers that cannot allocate device memory.

Some callers cannot give the library a workspace where they run the backward: engines
that reserve all of their device memory at start-up and may not allocate afterwards
(cudaMalloc can synchronise the device, stall, or fail once a caching allocator holds the
free memory), and plain C hosts with no allocator of their own.  attn_bwd_noalloc serves
them from a fixed 64 MiB scratch array inside the library.  The GPU test compares it with
attn_bwd (which takes a workspace) on the same inputs, on two calls in a row, since every
call reuses the same scratch; the CPU test checks that a problem too large for the
scratch is refused before anything touches the GPU.

This file sorts last so that, in a run that stops at the first failure, every other test
has already run."""
import ctypes

import pytest
import torch

import attn_workloads as W
import io_aware_exact_qk_b200 as attn
from tests import parity as P


def test_too_large_problem_is_refused_on_the_host():
    lib = attn.load_library()
    vp = ctypes.c_void_p
    T, hq, d = 1 << 20, 16, 128            # needs about 8.6 GB of scratch
    st = lib.attn_bwd_noalloc(vp(16), vp(16), vp(16), vp(16), vp(16), vp(16), None, 1, T, T, T, hq, hq, d,
                              0.088, 0, attn.ATTN_BF16, vp(16), vp(16), vp(16), None)
    assert st == attn.ATTN_ERR_INVALID_ARG
    assert b"64 MiB" in lib.attn_last_error_message()


@pytest.mark.gpu
def test_no_alloc_backward_matches_workspace_backward_twice():
    w = W.custom("noalloc", [300, 77, 513], 8, 2, 128, True, seed=91)
    q, k, v, do, cu = (t.cuda() for t in W.make_inputs(w))
    kw = dict(cu_seqlens=cu, max_seqlen=w.max_seqlen, scale=w.scale, causal=True)
    o, lse = attn.attn_fwd(q, k, v, **kw)
    ref = attn.attn_bwd(q, k, v, o, do, lse, **kw)
    torch.cuda.synchronize()
    ref = [P.to_np(t) for t in ref]
    for call in range(2):
        dq, dk, dv = (torch.full_like(t, float("nan")) for t in (q, k, v))
        before = torch.cuda.memory_allocated()
        attn.attn_bwd_noalloc(q, k, v, o, do, lse, dq=dq, dk=dk, dv=dv, **kw)
        attn.attn_get_device_error()
        assert torch.cuda.memory_allocated() == before
        for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
            err = P.rel_l2(P.to_np(got), want)
            assert err <= P.BF16_GRAD_REL_L2, f"call {call}: {name} rel-L2 {err}"
