"""Edge cases of the variable-length path on the GPU, forward and backward against the oracle.

- max_seqlen is an upper bound, not the exact longest length: work lists sized by a bound
  twice the longest sequence must skip the tiles past every sequence and give the same
  result as the exact bound.
- Many short sequences (2000 of 0..20 tokens, a quarter of them empty): one work item per
  tiny sequence and head, most query and key tiles ragged.
"""
import numpy as np
import pytest
import torch

import attn_workloads as W
import io_aware_exact_qk_b200 as attn
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_max_seqlen_above_the_longest_sequence(d, causal):
    w = W.custom(f"bound_d{d}", [1, 200, 0, 333, 129, 300, 310], 8, 2, d, causal, seed=110 + d)
    q, k, v, do, cu = W.make_inputs(w)
    qd, kd, vd, dod, cud = (t.cuda() for t in (q, k, v, do, cu))
    bound = 2 * w.max_seqlen          # (a bound may not exceed the total token count)
    assert bound <= w.total_tokens
    o, lse = attn.attn_fwd(qd, kd, vd, cu_seqlens=cud, max_seqlen=bound, scale=w.scale, causal=causal)
    dq, dk, dv = attn.attn_bwd(qd, kd, vd, o, dod, lse, cu_seqlens=cud, max_seqlen=bound, scale=w.scale,
                               causal=causal)
    attn.attn_get_device_error()
    o_ref, lse_ref = P.oracle_fwd(w, q, k, v, cu)
    P.check_fwd_bf16(P.to_np(o), P.to_np(lse), o_ref, lse_ref, tag=w.name)
    ref = P.oracle_bwd(w, q, k, v, do, cu)
    P.check_grads_bf16((dq, dk, dv), ref[:3], tag=w.name)
    # the exact bound gives bit-identical O, LSE, dK and dV (dQ sums its partials in a
    # run-dependent order)
    o2, lse2 = attn.attn_fwd(qd, kd, vd, cu_seqlens=cud, max_seqlen=w.max_seqlen, scale=w.scale, causal=causal)
    dq2, dk2, dv2 = attn.attn_bwd(qd, kd, vd, o2, dod, lse2, cu_seqlens=cud, max_seqlen=w.max_seqlen,
                                  scale=w.scale, causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    assert torch.equal(dk, dk2) and torch.equal(dv, dv2)


@pytest.mark.parametrize("causal", [False, True])
def test_many_short_sequences(causal):
    rng = np.random.default_rng(7)
    lens = rng.integers(0, 21, 2000)
    lens[rng.random(2000) < 0.25] = 0
    w = W.custom("many_short", lens.tolist(), 8, 2, 128, causal, seed=120)
    q, k, v, do, cu = W.make_inputs(w)
    o, lse = P.gpu_fwd(w, q, k, v, cu)
    o_ref, lse_ref = P.oracle_fwd(w, q, k, v, cu)
    P.check_fwd_bf16(P.to_np(o), P.to_np(lse), o_ref, lse_ref, tag=w.name)
    grads = P.gpu_bwd(w, q, k, v, o.cpu(), do, lse.cpu(), cu)
    ref = P.oracle_bwd(w, q, k, v, do, cu)
    P.check_grads_bf16(grads, ref[:3], tag=w.name)
