"""GPU parity of the forward (tcgen05 bf16 path and fp32 check mode) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import attn_workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("causal", [False, True])
def test_small_config(causal):
    w = W.small(causal)
    q, k, v, _, cu = W.make_inputs(w)
    o, lse = P.gpu_fwd(w, q, k, v, cu)
    o_ref, lse_ref = P.oracle_fwd(w, q, k, v, cu)
    P.check_fwd_bf16(o, lse, o_ref, lse_ref, tag=w.name)


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_ragged_varlen_gqa(d, causal):
    """Lengths around the 128-row tile and the 256-row CTA edges, one empty sequence, GQA 8:2."""
    w = W.custom(f"ragged_d{d}", [1, 127, 128, 129, 0, 255, 256, 257, 300, 513], 8, 2, d, causal, seed=7 + d)
    q, k, v, _, cu = W.make_inputs(w)
    o, lse = P.gpu_fwd(w, q, k, v, cu)
    o_ref, lse_ref = P.oracle_fwd(w, q, k, v, cu)
    P.check_fwd_bf16(o, lse, o_ref, lse_ref, tag=w.name)


@pytest.mark.parametrize("causal", [False, True])
def test_mha2k_config(causal):
    w = W.mha2k(causal)
    q, k, v, _, cu = W.make_inputs(w)
    o, lse = P.gpu_fwd(w, q, k, v, cu)
    o_ref, lse_ref = P.oracle_fwd(w, q, k, v, cu)
    P.check_fwd_bf16(o, lse, o_ref, lse_ref, tag=w.name)


def test_mqa_and_batch_mode_multi_tile():
    w = W.Workload("mqa", 3, 640, 6, 1, 64, True, seed=77)
    q, k, v, _, cu = W.make_inputs(w)
    o, lse = P.gpu_fwd(w, q, k, v, cu)
    o_ref, lse_ref = P.oracle_fwd(w, q, k, v, cu)
    P.check_fwd_bf16(o, lse, o_ref, lse_ref, tag=w.name)


def test_forward_is_deterministic():
    w = W.custom("det", [700, 333], 4, 4, 128, True, seed=11)
    q, k, v, _, cu = W.make_inputs(w)
    o1, l1 = P.gpu_fwd(w, q, k, v, cu)
    o2, l2 = P.gpu_fwd(w, q, k, v, cu)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_key_shift_invariance_and_constant_v():
    """Properties that hold at any size: K -> K + 1 u^T leaves O unchanged; constant V gives it back."""
    w = W.custom("inv", [1024], 4, 4, 128, False, seed=12)
    q, k, v, _, cu = W.make_inputs(w)
    u = torch.randn(1, 4, 128, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    o1, _ = P.gpu_fwd(w, q, k, v, cu)
    o2, _ = P.gpu_fwd(w, q, (k.float() + u.float()).to(torch.bfloat16), v, cu)
    assert P.rel_l2(P.to_np(o2), P.to_np(o1)) < 1e-2
    c = torch.randn(1, 4, 128).to(torch.bfloat16).expand_as(v).contiguous()
    o3, _ = P.gpu_fwd(w, q, k, c, cu)
    assert np.abs(P.to_np(o3) - P.to_np(c)).max() < 2e-2


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_fp32_check_mode(d, causal):
    w = W.custom(f"fp32_d{d}", [1, 77, 200], 4, 2, d, causal, seed=20 + d)
    q, k, v, _, cu = W.make_inputs(w, dtype=torch.float32)
    o, lse = P.gpu_fwd(w, q, k, v, cu)
    o_ref, lse_ref = P.oracle_fwd(w, q, k, v, cu)
    assert P.rel_l2(P.to_np(o), o_ref) <= P.FP32_REL
    assert P.max_rel(P.to_np(o), o_ref) <= P.FP32_REL
    assert P.max_rel(P.to_np(lse), lse_ref) <= P.FP32_REL
