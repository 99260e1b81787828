"""Device-side failure reporting and the forward's FMA-pipe exponential, on the GPU.

- A sequence longer than max_seqlen is not covered by the kernels' work lists; the forward
  and the backward both report it through attn_get_device_error (ATTN_ERR_INVALID_ARG)
  instead of silently dropping its tail.  (The kernels then only skip tiles, so nothing
  reads or writes out of bounds.)
- Every pipeline wait is bounded.  A self-test kernel waits on a barrier that nothing
  arrives on; with a short limit the wait runs out, attn_get_device_error reports
  ATTN_ERR_TIMEOUT, the GPU still answers, and the next normal call is correct.
- ex2_fma_pair, the 2^x the forward computes on the FMA pipe for a quarter of its
  exponentials, is held to its stated bound (relative error < 7.6e-5 on [-125, 8])
  against float64 2^x, and compared with the special-function unit's 2^x.
"""
import numpy as np
import pytest
import torch

import attn_workloads as W
import io_aware_exact_qk_b200 as attn
from tests import parity as P

pytestmark = pytest.mark.gpu


def _expect_status(status):
    with pytest.raises(attn.AttnError) as e:
        attn.attn_get_device_error()
    assert e.value.status == status


@pytest.mark.parametrize("d", [64, 128])
def test_sequence_longer_than_max_seqlen_is_reported(d):
    w = W.custom(f"maxlen_d{d}", [100, 700, 300], 4, 2, d, True, seed=70 + d)
    q, k, v, do, cu = (t.cuda() for t in W.make_inputs(w))
    short = 512                                   # below the longest sequence (700)
    o, lse = attn.attn_fwd(q, k, v, cu_seqlens=cu, max_seqlen=short, scale=w.scale, causal=True)
    _expect_status(attn.ATTN_ERR_INVALID_ARG)
    # the backward on a correct forward, called with the same too-small bound
    o, lse = attn.attn_fwd(q, k, v, cu_seqlens=cu, max_seqlen=w.max_seqlen, scale=w.scale, causal=True)
    attn.attn_get_device_error()
    attn.attn_bwd(q, k, v, o, do, lse, cu_seqlens=cu, max_seqlen=short, scale=w.scale, causal=True)
    _expect_status(attn.ATTN_ERR_INVALID_ARG)
    # the word is cleared by the read: a correct call afterwards reports nothing
    attn.attn_bwd(q, k, v, o, do, lse, cu_seqlens=cu, max_seqlen=w.max_seqlen, scale=w.scale, causal=True)
    attn.attn_get_device_error()


def test_wait_timeout_is_reported_and_the_gpu_recovers():
    default = attn.attn_get_wait_limit_ns()
    assert default == 2_000_000_000
    try:
        attn.attn_set_wait_limit_ns(50_000_000)   # 50 ms
        assert attn.attn_get_wait_limit_ns() == 50_000_000
        attn.attn_selftest_wait(arrive=True)     # completes: nothing to report
        attn.attn_get_device_error()
        attn.attn_selftest_wait(arrive=False)    # nothing arrives: the wait runs out
        _expect_status(attn.ATTN_ERR_TIMEOUT)
        attn.attn_get_device_error()             # read once, then cleared
    finally:
        attn.attn_set_wait_limit_ns(default)
    # the context is still usable and the next real call is right
    w = W.custom("after_timeout", [257, 130], 4, 2, 128, True, seed=72)
    q, k, v, _, cu = W.make_inputs(w)
    o, lse = P.gpu_fwd(w, q, k, v, cu)
    o_ref, lse_ref = P.oracle_fwd(w, q, k, v, cu)
    P.check_fwd_bf16(o, lse, o_ref, lse_ref, tag=w.name)


def test_fma_pipe_exp2_error_bound():
    rng = np.random.default_rng(5)
    xs = np.concatenate([
        np.linspace(-125.0, 8.0, 1 << 21),                         # dense grid over the softmax range
        rng.uniform(-125.0, 8.0, 1 << 20),
        np.linspace(-0.5, 0.5, 1 << 16),                           # the reduced argument's own range
        np.arange(-125, 8) + 0.5, np.arange(-124, 9) - 0.5,        # rounding ties of n = round(x)
    ]).astype(np.float32)
    x = torch.from_numpy(xs).cuda()
    y_fma, y_sfu = attn.attn_selftest_exp2(x)
    torch.cuda.synchronize()
    y_fma, y_sfu = y_fma.cpu().double().numpy(), y_sfu.cpu().double().numpy()
    exact = np.exp2(xs.astype(np.float64))
    rel = np.abs(y_fma - exact) / exact
    assert rel.max() <= 7.6e-5, f"max relative error {rel.max():.3e}"
    # the special-function unit's value agrees to within both errors
    assert (np.abs(y_fma - y_sfu) / exact).max() <= 7.6e-5 + 2.0 ** -21
    # 2^n is applied exactly: at integer x the result is 2^x times the cubic's value at 0,
    # the same float for every n (the fit trades exactness at 0 for a smaller max error)
    ints = np.arange(-125, 9, dtype=np.float32)
    y_int, _ = attn.attn_selftest_exp2(torch.from_numpy(ints).cuda())
    torch.cuda.synchronize()
    mant = y_int.cpu().double().numpy() / np.exp2(ints.astype(np.float64))
    assert np.all(mant == mant[0]) and abs(mant[0] - 1.0) <= 7.6e-5
