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
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
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
    od, lsed = o.to("cuda"), lse.to("cuda")
    if w.varlen:
        dq, dk, dv = attn.attn_bwd(qd, kd, vd, od, dod, lsed, cu_seqlens=cud, max_seqlen=w.max_seqlen,
                                   scale=w.scale, causal=w.causal)
    else:
        dq, dk, dv = attn.attn_bwd(qd, kd, vd, od, dod, lsed, scale=w.scale, causal=w.causal, batch=w.batch)
    attn.attn_get_device_error()
    return dq, dk, dv


def fp32_lse_bound(q_rows, k_all, scale, causal, row_ids):
    """Per-row bound on |LSE - LSE_ref| for fp32 accumulation of the scores: the row's
    largest score S_ij* is a 128-term dot product accumulated in fp32 (at most 8 rounded
    partial sums of 16 exact products each, every rounding <= half an ulp of
    sum_c |q_ic k_j*c|), and the LSE itself is stored in fp32 (half an ulp of |LSE|,
    plus one ulp for forming m + ln l).  With one score dominating, LSE ~ S_ij*, so
        bound_i = 4 * scale * ulp32(sum_c |q_ic k_j*c|) + 1.5 * ulp32(|LSE_i|).
    q_rows [r, d], k_all [n, d] for one (sequence, head); row_ids the rows' positions."""
    s = scale * (q_rows @ k_all.T)
    if causal:
        s = np.where(np.arange(k_all.shape[0])[None, :] > np.asarray(row_ids)[:, None], -np.inf, s)
    jstar = s.argmax(axis=1)
    mag = np.abs(q_rows * k_all[jstar]).sum(axis=1)
    lse_mag = np.abs(s.max(axis=1))
    ulp = lambda x: np.spacing(np.asarray(x, dtype=np.float32)).astype(np.float64)
    return 4.0 * scale * ulp(mag) + 1.5 * ulp(lse_mag)


def check_fwd_bf16(o, lse, o_ref, lse_ref, rows=None, tag="", lse_tol=None):
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
    if lse_tol is None:
        assert e_lse <= BF16_LSE_MAX_ABS, f"{tag} max|dLSE| {e_lse}"
    else:
        tol = np.maximum(BF16_LSE_MAX_ABS, lse_tol)   # per row, broadcast over heads
        worst = float((np.abs(lse - lse_ref) / tol).max())
        assert worst <= 1.0, f"{tag} |dLSE| exceeds the fp32 bound: max error/bound {worst:.3f}"
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


def sample_indices(n, rng, k=16):
    """First k, last k and k random indices in between (all of them when n is small)."""
    if n <= 3 * k:
        return np.arange(n)
    mid = rng.choice(np.arange(k, n - k), size=k, replace=False)
    return np.sort(np.concatenate([np.arange(k), mid, np.arange(n - k, n)]))


def check_sampled(w, inputs, outputs, picks, seed=0, tag="", given=False, fp32_lse_bound_rows=False, strict=False):
    """Parity on sampled outputs of a full-size run.

    inputs  = (q, k, v, do, cu) CPU tensors; outputs = (o, lse, dq, dk, dv) device tensors.
    picks   = [(sequence b, kv head g), ...].  For each pick the oracle runs the whole
    (sequence, GQA group) slice -- every row enters the statistics -- and the comparison
    covers O/LSE and dQ on sampled query rows and dK/dV on sampled keys.

    given=True compares the backward as a function of its inputs: the oracle's own forward
    of the slice, stored as attn_fwd stores it (O rounded to bf16, LSE to fp32), is
    written over the slice of the device O / LSE, the GPU backward runs again on them,
    and the oracle's backward takes the same stored O (for D) and LSE (for P); no value
    the GPU computed enters the oracle.  Otherwise the reference is the exact gradient.  fp32_lse_bound_rows=True checks LSE against
    max(1e-3, fp32_lse_bound) per row instead of 1e-3 (for scores far above fp32's
    exact-integer range, where 1e-3 is below a few ulps of the LSE itself).

    strict=True also measures, without asserting, the errors against the plain definition
    on the same samples -- the device's own forward and backward against the exact
    gradients and the raw max |LSE - LSE_ref| -- and returns them as each report entry's
    fourth element ({"dq", "dk", "dv", "lse"}), so a test can hold them to recorded
    ceilings."""
    q, k, v, do, cu = inputs
    o, lse, dq, dk, dv = outputs
    G = w.hq // w.hkv
    rng = np.random.default_rng(seed)
    report = []
    for b, g in picks:
        t0, t1 = int(cu[b]), int(cu[b + 1])
        n = t1 - t0
        if n == 0:
            continue
        hs = slice(g * G, (g + 1) * G)
        sl = (slice(t0, t1), hs)
        ks = (slice(t0, t1), slice(g, g + 1))
        rows = sample_indices(n, rng)
        keys = sample_indices(n, rng)
        o_full = to_np(o[t0:t1, hs])
        lse_full = to_np(lse[hs, t0:t1])
        grads = (dq, dk, dv)
        extra = {}
        if given:
            o_or, lse_or = oracle.attn_fwd(q[sl], k[ks], v[ks], scale=w.scale, causal=w.causal)
            o_st = torch.from_numpy(o_or).to(torch.bfloat16)
            lse_st = torch.from_numpy(lse_or).to(torch.float32)
            o_dev, lse_dev = o.clone(), lse.clone()
            o_dev[t0:t1, hs] = o_st.to(o_dev.device)
            lse_dev[hs, t0:t1] = lse_st.to(lse_dev.device)
            grads = gpu_bwd(w, q, k, v, o_dev, do, lse_dev, cu)
            del o_dev, lse_dev
            extra = dict(o=o_st.double().numpy(), lse=lse_st.double().numpy())
        dq_r, dk_r, dv_r, o_r, lse_r = oracle.attn_bwd(q[sl], k[ks], v[ks], do[sl], scale=w.scale, causal=w.causal,
                                                       rows=rows, keys=keys, **extra)
        if given:   # the forward reference is the oracle's own forward either way
            o_r, lse_r = o_or, lse_or
        tg = f"{tag} seq{b} g{g}"
        lse_tol = None
        if fp32_lse_bound_rows:
            k_np = to_np(k[t0:t1, g])
            lse_tol = np.stack([fp32_lse_bound(to_np(q[t0:t1, h])[rows], k_np, w.scale, w.causal, rows)
                                for h in range(g * G, (g + 1) * G)])
        check_fwd_bf16(o_full[rows], lse_full[:, rows], o_r[rows], lse_r[:, rows], tag=tg, lse_tol=lse_tol)
        gq, gk, gv = grads
        errs = check_grads_bf16((gq[t0:t1, hs], gk[t0:t1, g:g + 1], gv[t0:t1, g:g + 1]),
                                (dq_r, dk_r, dv_r), rows=rows, keys=keys, tag=tg)
        if not strict:
            report.append((b, g, errs))
            continue
        if given:
            dq_e, dk_e, dv_e, _, lse_e = oracle.attn_bwd(q[sl], k[ks], v[ks], do[sl], scale=w.scale,
                                                         causal=w.causal, rows=rows, keys=keys)
        else:
            dq_e, dk_e, dv_e, lse_e = dq_r, dk_r, dv_r, lse_r
        exact = {"lse": float(np.abs(lse_full[:, rows] - lse_e[:, rows]).max())}
        for name, g_, r_, sel in (("dq", dq[t0:t1, hs], dq_e, rows), ("dk", dk[t0:t1, g:g + 1], dk_e, keys),
                                  ("dv", dv[t0:t1, g:g + 1], dv_e, keys)):
            exact[name] = rel_l2(to_np(g_)[sel], r_[sel])
        report.append((b, g, errs, exact))
    return report


def check_sum_properties(w, cu, do, dk, dv, tag=""):
    """Any-size invariants of the backward: per (sequence, kv head), sum_j dK_j = 0 and
    sum_j dV_j = sum over the group's query heads and rows of dO."""
    G = w.hq // w.hkv
    for b in range(len(cu) - 1):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        if t1 == t0:
            continue
        dk_s = dk[t0:t1].double().sum(dim=0).cpu().numpy()
        dk_abs = dk[t0:t1].double().abs().sum(dim=0).cpu().numpy()
        assert np.abs(dk_s).max() <= 2e-2 * dk_abs.max(), f"{tag} seq{b}: sum of dK not ~0"
        dv_s = dv[t0:t1].double().sum(dim=0).cpu().numpy()
        want = do[t0:t1].double().reshape(t1 - t0, w.hkv, G, w.d).sum(dim=(0, 2)).numpy()
        assert rel_l2(dv_s, want) <= 1e-2, f"{tag} seq{b}: sum of dV != sum of dO"


def run_full(w, inputs):
    """fwd + bwd of the whole workload on the device; returns (o, lse, dq, dk, dv)."""
    q, k, v, do, cu = inputs
    o, lse = gpu_fwd(w, q, k, v, cu)
    dq, dk, dv = gpu_bwd(w, q, k, v, o, do, lse, cu)
    return o, lse, dq, dk, dv
