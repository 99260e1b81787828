"""Helpers shared by the GPU parity tests: run the CUDA library and the fp64 oracle on the
same seeded inputs and compare them with the stated tolerances.

Tolerances (bf16 tensors, fp32 accumulation and statistics):
    forward    max |O - O_ref| <= 2e-2,  ||O - O_ref||_2 / ||O_ref||_2 <= 5e-3,
               max |LSE - LSE_ref| <= 1e-3
    backward   ||dX - dX_ref||_2 / ||dX_ref||_2 <= 1e-2 for dX in dQ, dK, dV
fp32 check mode (fp32 tensors and arithmetic): every output within a relative error of
1e-5 (both the relative L2 error and max |x - ref| / max |ref|), the order the
"FlashAttention 与高效注意力内核" tutorial asks of the forward in section 数值验证.
"""
import numpy as np
import torch

import io_aware_exact_qk_b200 as attn
import oracle

BF16_O_MAX_ABS = 2e-2
BF16_O_REL_L2 = 5e-3
BF16_LSE_MAX_ABS = 1e-3
BF16_GRAD_REL_L2 = 1e-2
FP32_REL = 1e-5


def rel_l2(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm((x - ref).ravel()) / max(np.linalg.norm(ref.ravel()), 1e-300))


def max_rel(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(x - ref).max() / max(np.abs(ref).max(), 1e-300))


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def device_inputs(q, k, v, do, cu):
    dev = torch.device("cuda")
    return (q.to(dev), k.to(dev), v.to(dev), None if do is None else do.to(dev), cu.to(dev))


def gpu_fwd(w, q, k, v, cu):
    """Runs attn_fwd on the device copies of the inputs (varlen calls pass cu_seqlens)."""
    qd, kd, vd, _, cud = device_inputs(q, k, v, None, cu)
    if w.varlen:
        o, lse = attn.attn_fwd(qd, kd, vd, cu_seqlens=cud, max_seqlen=w.max_seqlen, scale=w.scale, causal=w.causal)
    else:
        o, lse = attn.attn_fwd(qd, kd, vd, scale=w.scale, causal=w.causal, batch=w.batch)
    attn.attn_get_device_error()
    return o, lse


def gpu_bwd(w, q, k, v, o, do, lse, cu):
    qd, kd, vd, dod, cud = device_inputs(q, k, v, do, cu)
    od, lsed = o.cuda(), lse.cuda()
    if w.varlen:
        dq, dk, dv = attn.attn_bwd(qd, kd, vd, od, dod, lsed, cu_seqlens=cud, max_seqlen=w.max_seqlen,
                                   scale=w.scale, causal=w.causal)
    else:
        dq, dk, dv = attn.attn_bwd(qd, kd, vd, od, dod, lsed, scale=w.scale, causal=w.causal, batch=w.batch)
    attn.attn_get_device_error()
    return dq, dk, dv


def check_fwd_bf16(o, lse, o_ref, lse_ref, rows=None, tag=""):
    o, lse = to_np(o), to_np(lse)
    if rows is not None:
        o, o_ref = o[rows], o_ref[rows]
        lse, lse_ref = lse[:, rows], lse_ref[:, rows]
    assert np.isfinite(o).all() and np.isfinite(lse).all(), tag
    e_max = float(np.abs(o - o_ref).max())
    e_rel = rel_l2(o, o_ref)
    e_lse = float(np.abs(lse - lse_ref).max())
    assert e_max <= BF16_O_MAX_ABS, f"{tag} max|dO| {e_max}"
    assert e_rel <= BF16_O_REL_L2, f"{tag} relL2(O) {e_rel}"
    assert e_lse <= BF16_LSE_MAX_ABS, f"{tag} max|dLSE| {e_lse}"
    return e_max, e_rel, e_lse


def check_grads_bf16(got, ref, rows=None, keys=None, tag=""):
    errs = {}
    for name, g, r, sel in zip(("dq", "dk", "dv"), got, ref, (rows, keys, keys)):
        g = to_np(g)
        if sel is not None:
            g, r = g[sel], r[sel]
        assert np.isfinite(g).all(), f"{tag} {name} not finite"
        errs[name] = rel_l2(g, r)
        assert errs[name] <= BF16_GRAD_REL_L2, f"{tag} relL2({name}) {errs[name]}"
    return errs


def oracle_fwd(w, q, k, v, cu, rows=None):
    return oracle.attn_fwd(q, k, v, cu.numpy(), scale=w.scale, causal=w.causal, rows=rows)


def oracle_bwd(w, q, k, v, do, cu, rows=None, keys=None):
    return oracle.attn_bwd(q, k, v, do, cu.numpy(), scale=w.scale, causal=w.causal, rows=rows, keys=keys)
