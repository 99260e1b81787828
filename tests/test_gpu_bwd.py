"""GPU parity of the backward (tcgen05 bf16 path and fp32 check mode) against the fp64 oracle.

The GPU backward consumes the GPU forward's O and LSE, as a caller would; the oracle
forms its own from the definition."""
import numpy as np
import pytest
import torch

import attn_workloads as W
import io_aware_exact_qk_b200 as attn
from tests import parity as P

pytestmark = pytest.mark.gpu


def _run(w, dtype=torch.bfloat16):
    q, k, v, do, cu = W.make_inputs(w, dtype=dtype)
    o, lse = P.gpu_fwd(w, q, k, v, cu)
    grads = P.gpu_bwd(w, q, k, v, o.cpu(), do, lse.cpu(), cu)
    ref = P.oracle_bwd(w, q, k, v, do, cu)
    return grads, ref


@pytest.mark.parametrize("causal", [False, True])
def test_small_config(causal):
    w = W.small(causal)
    grads, ref = _run(w)
    P.check_grads_bf16(grads, ref[:3], tag=w.name)


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_ragged_varlen_gqa(d, causal):
    """Lengths around the 64/128-row tile edges, one empty sequence, GQA 8:2."""
    w = W.custom(f"ragged_d{d}", [1, 63, 64, 65, 127, 128, 129, 0, 200, 383], 8, 2, d, causal, seed=40 + d)
    grads, ref = _run(w)
    P.check_grads_bf16(grads, ref[:3], tag=w.name)


@pytest.mark.parametrize("causal", [False, True])
def test_mha2k_config(causal):
    w = W.mha2k(causal)
    grads, ref = _run(w)
    P.check_grads_bf16(grads, ref[:3], tag=w.name)


def test_mqa_batch_mode():
    w = W.Workload("mqa", 2, 520, 4, 1, 128, True, seed=78)
    grads, ref = _run(w)
    P.check_grads_bf16(grads, ref[:3], tag=w.name)


def test_gradient_sums_at_size():
    """Properties that hold at any size: per (sequence, kv head) sum_j dK_j = 0 and
    sum_j dV_j = sum over the group's query heads and rows of dO."""
    w = W.custom("sums", [3000, 1100], 8, 2, 128, True, seed=79)
    q, k, v, do, cu = W.make_inputs(w)
    o, lse = P.gpu_fwd(w, q, k, v, cu)
    dq, dk, dv = P.gpu_bwd(w, q, k, v, o.cpu(), do, lse.cpu(), cu)
    dk, dv, dof = P.to_np(dk), P.to_np(dv), do.double().numpy()
    G = w.hq // w.hkv
    for bi in range(2):
        sl = slice(int(cu[bi]), int(cu[bi + 1]))
        sk = dk[sl].sum(axis=0)
        assert np.abs(sk).max() <= 2e-2 * np.abs(dk[sl]).sum(axis=0).max()
        want = dof[sl].reshape(-1, w.hkv, G, w.d).sum(axis=(0, 2))
        assert P.rel_l2(dv[sl].sum(axis=0), want) < 1e-2


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_fp32_check_mode(d, causal):
    w = W.custom(f"fp32b_d{d}", [1, 77, 150], 4, 2, d, causal, seed=60 + d)
    grads, ref = _run(w, dtype=torch.float32)
    for name, g, r in zip(("dq", "dk", "dv"), grads, ref[:3]):
        g = P.to_np(g)
        assert P.rel_l2(g, r) <= P.FP32_REL, name
        assert P.max_rel(g, r) <= P.FP32_REL, name


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_accumulate_mode_adds_float32_gradients(d, causal):
    """attn_bwd_accumulate adds the gradients into float32 tensors: two calls on the same
    inputs give twice the gradient (each call within the backward's tolerance of the
    oracle), and one call agrees with attn_bwd up to attn_bwd's own bf16 rounding."""
    w = W.custom(f"acc_d{d}", [1, 130, 0, 257], 8, 2, d, causal, seed=90 + d)
    q, k, v, do, cu = W.make_inputs(w)
    qd, kd, vd, dod, cud = (t.cuda() for t in (q, k, v, do, cu))
    kw = dict(cu_seqlens=cud, max_seqlen=w.max_seqlen, scale=w.scale, causal=causal)
    o, lse = attn.attn_fwd(qd, kd, vd, **kw)
    accs = [torch.zeros(t.shape, dtype=torch.float32, device="cuda") for t in (qd, kd, vd)]
    attn.attn_bwd_accumulate(qd, kd, vd, o, dod, lse, *accs, **kw)
    once = [P.to_np(a) for a in accs]
    attn.attn_bwd_accumulate(qd, kd, vd, o, dod, lse, *accs, **kw)
    attn.attn_get_device_error()
    twice = [P.to_np(a) for a in accs]
    ref = P.oracle_bwd(w, q, k, v, do, cu)[:3]
    P.check_grads_bf16(once, ref, tag=w.name)
    for a, b in zip(once, twice):
        assert P.rel_l2(b, 2 * a) <= 1e-6
    bf = [P.to_np(t) for t in attn.attn_bwd(qd, kd, vd, o, dod, lse, **kw)]
    for name, a, b in zip(("dq", "dk", "dv"), once, bf):
        assert np.abs(a - b).max() <= 2 ** -8 * np.abs(a).max() + 1e-6, name


@pytest.mark.parametrize("scale", [0.05, 0.25])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_explicit_scale_and_three_heads_per_group(scale, d, causal):
    """The score scale is a free argument (here 0.05 and 0.25 instead of 1/sqrt(d)), with
    three query heads per K/V head and ragged sequences: forward and backward against the
    oracle at the same scale."""
    w = W.custom(f"scale{scale}_d{d}", [1, 129, 300, 64], 6, 2, d, causal, seed=95 + d, scale=scale)
    q, k, v, do, cu = W.make_inputs(w)
    o, lse = P.gpu_fwd(w, q, k, v, cu)
    o_ref, lse_ref = P.oracle_fwd(w, q, k, v, cu)
    P.check_fwd_bf16(P.to_np(o), P.to_np(lse), o_ref, lse_ref, tag=w.name)
    grads = P.gpu_bwd(w, q, k, v, o.cpu(), do, lse.cpu(), cu)
    ref = P.oracle_bwd(w, q, k, v, do, cu)
    P.check_grads_bf16(grads, ref[:3], tag=w.name)


@pytest.mark.parametrize("causal", [False, True])
def test_fp32_check_mode_explicit_scale(causal):
    """The fp32 check mode at a scale other than 1/sqrt(d), three heads per group."""
    w = W.custom("fp32_scale", [1, 77, 150], 6, 2, 64, causal, seed=99, scale=0.3)
    grads, ref = _run(w, dtype=torch.float32)
    for name, g, r in zip(("dq", "dk", "dv"), grads, ref[:3]):
        g = P.to_np(g)
        assert P.rel_l2(g, r) <= P.FP32_REL, name
        assert P.max_rel(g, r) <= P.FP32_REL, name
