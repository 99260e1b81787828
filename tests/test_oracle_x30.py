"""What the bf16 storage of O costs config 4b (Q and K x30, the tutorial's 验证清单 max-value
stability case) before any kernel is involved.

attn_bwd takes the O the forward stored (bf16) and forms D = rowsum(dO o O) from it.  With
scores in the thousands, P is nearly one-hot and dS = P (dP - D) is a cancellation, so the
rounding of O reaches the gradients amplified.  The oracle alone shows it: its backward
given its own forward, rounded exactly as attn_fwd stores it (O to bf16, LSE to fp32),
moves dQ and dK by more than the stated 1e-2 (rel-L2) from the exact gradient on the
sampled slice below, while dV (which does not go through D) stays near fp32's LSE
rounding.  So the 1e-2 tolerance on dQ / dK is out of reach for this configuration under
an ABI that passes a bf16 O; the GPU test holds the device to recorded ceilings instead."""
import numpy as np
import torch

import attn_workloads as W
import oracle
from tests import parity as P


def test_bf16_stored_o_alone_moves_x30_gradients_past_1e2():
    w = W.gqa8k(stability=True)
    q, k, v, do, cu = W.make_inputs(w)
    G = w.hq // w.hkv
    b, g = 1, 7                                  # the second sampled slice of the GPU test
    t0, t1 = int(cu[b]), int(cu[b + 1])
    hs = slice(g * G, (g + 1) * G)
    sl, ks = (slice(t0, t1), hs), (slice(t0, t1), slice(g, g + 1))
    rng = np.random.default_rng(0)
    rows = P.sample_indices(t1 - t0, rng)
    keys = P.sample_indices(t1 - t0, rng)
    o, lse = oracle.attn_fwd(q[sl], k[ks], v[ks], scale=w.scale, causal=True)
    o_st = torch.from_numpy(o).to(torch.bfloat16).double().numpy()
    lse_st = torch.from_numpy(lse).to(torch.float32).double().numpy()
    given = oracle.attn_bwd(q[sl], k[ks], v[ks], do[sl], scale=w.scale, causal=True, rows=rows, keys=keys,
                            o=o_st, lse=lse_st)
    exact = oracle.attn_bwd(q[sl], k[ks], v[ks], do[sl], scale=w.scale, causal=True, rows=rows, keys=keys)
    err = {n: P.rel_l2(given[i][sel], exact[i][sel]) for n, i, sel in (("dq", 0, rows), ("dk", 1, keys),
                                                                      ("dv", 2, keys))}
    assert err["dq"] > 1e-2 and err["dk"] > 1e-2, err
    assert err["dv"] < 1e-3, err
