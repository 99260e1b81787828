"""attn_fwd_bwd_host on the GPU: the forward and backward from host buffers through the
library's copy/compute pipeline (sequences in up to four groups, three streams).

Each case compares the pipelined call with attn_fwd + attn_bwd on the same tensors in
device memory -- O, LSE, dK and dV bit for bit (every group is computed by the same
kernels, and each (tile, head) result does not depend on the schedule), dQ to within one
bf16 rounding of its fp32 sums -- and with the fp64 oracle at the usual tolerances.
"""
import numpy as np
import pytest
import torch

import attn_workloads as W
import io_aware_exact_qk_b200 as attn
from tests import parity as P

pytestmark = pytest.mark.gpu


def _pinned(t):
    return t.contiguous().pin_memory()


def _device_path(w, q, k, v, do, cu):
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    if w.varlen:
        kw = dict(cu_seqlens=cu.cuda(), max_seqlen=w.max_seqlen)
    else:
        kw = dict(batch=w.batch)
    o, lse = attn.attn_fwd(qd, kd, vd, scale=w.scale, causal=w.causal, **kw)
    dq, dk, dv = attn.attn_bwd(qd, kd, vd, o, dod, lse, scale=w.scale, causal=w.causal, **kw)
    attn.attn_get_device_error()
    return [t.cpu() for t in (o, lse, dq, dk, dv)]


def _check(w, got, q, k, v, do, cu):
    o, lse, dq, dk, dv = got
    ref = _device_path(w, q, k, v, do, cu)
    assert torch.equal(o, ref[0]) and torch.equal(lse, ref[1]), w.name
    assert torch.equal(dk, ref[3]) and torch.equal(dv, ref[4]), w.name
    dq32, rq32 = dq.float(), ref[2].float()
    assert float((dq32 - rq32).abs().max()) <= float(rq32.abs().max()) * 2.0 ** -7, w.name
    o_ref, lse_ref = P.oracle_fwd(w, q, k, v, cu)
    P.check_fwd_bf16(P.to_np(o), P.to_np(lse), o_ref, lse_ref, tag=w.name)
    g_ref = P.oracle_bwd(w, q, k, v, do, cu)
    P.check_grads_bf16((dq, dk, dv), g_ref[:3], tag=w.name)


@pytest.mark.parametrize("causal", [False, True])
def test_batch_mode_four_groups(causal):
    w = W.Workload("host_b5", 5, 700, 8, 2, 128, causal, seed=130)     # five sequences in four groups
    q, k, v, do, cu = W.make_inputs(w)
    got, _ = attn.attn_fwd_bwd_host(_pinned(q), _pinned(k), _pinned(v), _pinned(do), batch=w.batch,
                                    scale=w.scale, causal=causal)
    attn.attn_get_device_error()
    _check(w, got, q, k, v, do, cu)


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_uneven_groups(causal):
    w = W.custom("host_var", [1, 300, 0, 129, 777, 64, 2000, 5], 6, 2, 64, causal, seed=131)
    q, k, v, do, cu = W.make_inputs(w)
    got, _ = attn.attn_fwd_bwd_host(_pinned(q), _pinned(k), _pinned(v), _pinned(do), cu_seqlens=cu,
                                    max_seqlen=w.max_seqlen, scale=w.scale, causal=causal)
    attn.attn_get_device_error()
    _check(w, got, q, k, v, do, cu)


def test_single_sequence_and_reuse_on_a_side_stream():
    """One sequence (one group); the second call reuses the outputs and the scratch and is
    queued on a stream of the caller's that is not the current one."""
    w = W.Workload("host_b1", 1, 1500, 4, 4, 128, True, seed=132)
    q, k, v, do, cu = W.make_inputs(w)
    args = [_pinned(t) for t in (q, k, v, do)]
    out, scratch = attn.attn_fwd_bwd_host(*args, batch=1, scale=w.scale, causal=True)
    torch.cuda.current_stream().synchronize()     # calls that share a scratch must be ordered
    side = torch.cuda.Stream()
    out2, _ = attn.attn_fwd_bwd_host(*args, batch=1, scale=w.scale, causal=True, out=out, scratch=scratch,
                                     stream=side)
    side.synchronize()
    attn.attn_get_device_error()
    _check(w, out2, q, k, v, do, cu)


def test_attention_host_wrapper_matches():
    w = W.Workload("host_wrap", 2, 513, 4, 2, 64, False, seed=133)
    q, k, v, do, cu = W.make_inputs(w)
    res, bufs = attn.attention_host(_pinned(q), _pinned(k), _pinned(v), _pinned(do), batch=2, scale=w.scale)
    res2, _ = attn.attention_host(_pinned(q), _pinned(k), _pinned(v), _pinned(do), batch=2, scale=w.scale, out=bufs)
    torch.cuda.synchronize()
    attn.attn_get_device_error()
    _check(w, res2, q, k, v, do, cu)
