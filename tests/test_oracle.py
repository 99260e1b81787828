"""Pins for the fp64 CPU oracle (no GPU).

Each test ties the oracle to something other than itself: a deliberately naive
brute-force evaluation, an independent library routine (torch's fp64 CPU
scaled_dot_product_attention and autograd), central finite differences, the online-softmax
worked example printed in the "FlashAttention 与高效注意力内核" tutorial (section 流式过程),
closed forms and invariants of the definition.  Together they are chosen so that a dropped
term, a wrong sign, a wrong index or a transposed operand anywhere in the oracle fails
at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _cu(lengths):
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)


# ---------------------------------------------------------------------------------------
# brute force: a second, deliberately naive evaluation (explicit softmax, no max shift)
# ---------------------------------------------------------------------------------------
def naive_fwd(q, k, v, lengths, scale, causal):
    T, hq, d = q.shape
    hkv = k.shape[1]
    o = np.zeros_like(q)
    lse = np.zeros((hq, T))
    start = 0
    for n in lengths:
        for h in range(hq):
            g = h // (hq // hkv)
            for i in range(n):
                num = [0.0] * d
                den = 0.0
                for j in range(n):
                    if causal and j > i:
                        continue
                    s = scale * sum(q[start + i, h, c] * k[start + j, g, c] for c in range(d))
                    e = math.exp(s)
                    den += e
                    for c in range(d):
                        num[c] += e * v[start + j, g, c]
                for c in range(d):
                    o[start + i, h, c] = num[c] / den
                lse[h, start + i] = math.log(den)
        start += n
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("lengths,hq,hkv,d", [([5], 1, 1, 3), ([8], 2, 2, 4), ([3, 7, 1], 4, 2, 2),
                                             ([6, 2], 3, 1, 4)])
def test_forward_matches_brute_force(lengths, hq, hkv, d, causal):
    T = sum(lengths)
    q, k, v = _rand((T, hq, d), 1), _rand((T, hkv, d), 2), _rand((T, hkv, d), 3)
    scale = 0.7
    o, lse = oracle.attn_fwd(q, k, v, _cu(lengths), scale=scale, causal=causal)
    o_ref, lse_ref = naive_fwd(q, k, v, lengths, scale, causal)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------------------
# independent library cross-check: torch fp64 CPU SDPA + autograd (test dependency only)
# ---------------------------------------------------------------------------------------
def torch_ref(q, k, v, do, scale, causal):
    """q [n,hq,d] etc. for one sequence -> O, dQ, dK, dV via torch's SDPA and autograd."""
    hq, hkv = q.shape[1], k.shape[1]
    qt = torch.tensor(q, requires_grad=True)
    kt = torch.tensor(k, requires_grad=True)
    vt = torch.tensor(v, requires_grad=True)
    kr = kt.repeat_interleave(hq // hkv, dim=1)
    vr = vt.repeat_interleave(hq // hkv, dim=1)
    out = torch.nn.functional.scaled_dot_product_attention(
        qt.transpose(0, 1), kr.transpose(0, 1), vr.transpose(0, 1), is_causal=causal, scale=scale)
    out = out.transpose(0, 1)
    out.backward(torch.tensor(do))
    return out.detach().numpy(), qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n,hq,hkv,d", [(9, 2, 2, 8), (33, 4, 1, 16), (20, 6, 3, 5)])
def test_matches_torch_sdpa_and_autograd(n, hq, hkv, d, causal):
    q, k, v, do = _rand((n, hq, d), 4), _rand((n, hkv, d), 5), _rand((n, hkv, d), 6), _rand((n, hq, d), 7)
    scale = 1.0 / math.sqrt(d)
    o_t, dq_t, dk_t, dv_t = torch_ref(q, k, v, do, scale, causal)
    o, _ = oracle.attn_fwd(q, k, v, scale=scale, causal=causal)
    dq, dk, dv, o2, _ = oracle.attn_bwd(q, k, v, do, scale=scale, causal=causal)
    for a, b in [(o, o_t), (o2, o_t), (dq, dq_t), (dk, dk_t), (dv, dv_t)]:
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-11)


# ---------------------------------------------------------------------------------------
# gradients: central finite differences of L = sum(dO * O)  (the tutorial's "gradcheck")
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_gradients_match_finite_differences(causal):
    lengths, hq, hkv, d = [5, 4], 4, 2, 3
    T = sum(lengths)
    cu = _cu(lengths)
    q, k, v, do = _rand((T, hq, d), 8), _rand((T, hkv, d), 9), _rand((T, hkv, d), 10), _rand((T, hq, d), 11)
    scale = 0.9
    dq, dk, dv, _, _ = oracle.attn_bwd(q, k, v, do, cu, scale=scale, causal=causal)

    def loss(qq, kk, vv):
        o, _ = oracle.attn_fwd(qq, kk, vv, cu, scale=scale, causal=causal)
        return float(np.sum(o * do))

    h = 1e-6
    rng = np.random.default_rng(12)
    for name, x, g in [("q", q, dq), ("k", k, dk), ("v", v, dv)]:
        for _ in range(12):
            idx = tuple(int(rng.integers(0, s)) for s in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - g[idx]) <= 1e-6 * max(1.0, abs(g[idx])), (name, idx, fd, g[idx])


# ---------------------------------------------------------------------------------------
# the tutorial's online-softmax worked example (section 流式过程)
# ---------------------------------------------------------------------------------------
def test_worked_example_online_merge():
    ex = json.load(open(os.path.join(HERE, "golden", "online_softmax_worked_example.json")))["printed_on_page"]
    m1, l1, m2 = ex["block1_max"], ex["block1_sum"], ex["block2_max"]
    assert (m1, l1, m2) == (2.0, 3.1, 3.5)
    # block 1 scores: max 2.0 and sum_j exp(s_j - 2.0) = 1 + 1 + 1 + 0.1 = 3.1
    b1 = [2.0, 2.0, 2.0, 2.0 + math.log(0.1)]
    # block 2 scores: max 3.5, own sum 1 + 0.7 = 1.7 (not printed on the page)
    b2 = [3.5, 3.5 + math.log(0.7)]
    l2 = 1.7
    scores = b1 + b2
    # one query row with d=1, q=1, k_j=s_j, scale=1 gives S_0j = s_j exactly
    n = len(scores)
    q = np.zeros((n, 1, 1)); q[:, 0, 0] = 1.0
    k = np.array(scores, dtype=np.float64).reshape(n, 1, 1)
    v = np.arange(n, dtype=np.float64).reshape(n, 1, 1)
    _, lse = oracle.attn_fwd(q, k, v, scale=1.0, causal=False)
    # the page's update rule: m_new = max(m_old, m_block), l_new = l_old*exp(m_old-m_new) + l_block
    m_new = max(m1, m2)
    rescaled = l1 * math.exp(m1 - m_new)
    assert abs(math.exp(m1 - m2) - 0.2231302) < 1e-7     # exp(2.0 - 3.5)
    assert abs(rescaled - 0.6917035) < 1e-7              # 3.1 * exp(-1.5)
    l_new = rescaled + l2
    assert abs(lse[0, 0] - (m_new + math.log(l_new))) < 1e-14
    # the block-1 share of the final softmax is the rescaled block-1 sum over the total
    p, _ = oracle.attn_probs(q[:, 0, :], k[:, 0, :], scale=1.0)
    assert abs(p[0, :4].sum() - rescaled / l_new) < 1e-14
    assert abs(p[0, 4:].sum() - l2 / l_new) < 1e-14


# ---------------------------------------------------------------------------------------
# closed forms and invariants
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_probability_rows(causal):
    n, d = 37, 8
    q, k = _rand((n, d), 13, 3.0), _rand((n, d), 14, 3.0)
    p, lse = oracle.attn_probs(q, k, scale=0.5, causal=causal)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    assert (p >= 0).all()
    if causal:
        assert (p[np.triu_indices(n, 1)] == 0.0).all()
    s = 0.5 * q @ k.T
    if causal:
        s[np.triu_indices(n, 1)] = -np.inf
    m = s.max(axis=1)
    assert (lse >= m - 1e-12).all() and (lse <= m + np.log(n) + 1e-12).all()


@pytest.mark.parametrize("causal", [False, True])
def test_constant_v_gives_constant(causal):
    T, hq, d = 21, 2, 6
    q, k = _rand((T, hq, d), 15), _rand((T, hq, d), 16)
    c = _rand((d,), 17)
    v = np.broadcast_to(c, (T, hq, d)).copy()
    o, _ = oracle.attn_fwd(q, k, v, causal=causal)
    np.testing.assert_allclose(o, np.broadcast_to(c, o.shape), rtol=1e-14, atol=1e-14)


def test_causal_row0_and_single_token():
    T, hq, d = 17, 3, 5
    q, k, v = _rand((T, hq, d), 18), _rand((T, hq, d), 19), _rand((T, hq, d), 20)
    o, lse = oracle.attn_fwd(q, k, v, causal=True)
    assert np.array_equal(o[0], v[0])
    np.testing.assert_allclose(lse[:, 0], np.einsum("hc,hc->h", q[0], k[0]) / math.sqrt(d), atol=1e-14)
    o1, _ = oracle.attn_fwd(q[:1], k[:1], v[:1], causal=False)
    assert np.array_equal(o1, v[:1])


@pytest.mark.parametrize("causal", [False, True])
def test_zero_queries_give_uniform_average(causal):
    lengths, hq, hkv, d = [7, 12], 4, 2, 3
    T = sum(lengths)
    q = np.zeros((T, hq, d))
    k, v = _rand((T, hkv, d), 21), _rand((T, hkv, d), 22)
    o, lse = oracle.attn_fwd(q, k, v, _cu(lengths), causal=causal)
    start = 0
    for n in lengths:
        for i in range(n):
            cnt = i + 1 if causal else n
            for h in range(hq):
                g = h // (hq // hkv)
                np.testing.assert_allclose(o[start + i, h], v[start:start + cnt, g].mean(axis=0), atol=1e-14)
                assert abs(lse[h, start + i] - math.log(cnt)) < 1e-14
        start += n


@pytest.mark.parametrize("causal", [False, True])
def test_key_shift_invariance(causal):
    T, hq, d = 19, 2, 4
    q, k, v = _rand((T, hq, d), 23), _rand((T, hq, d), 24), _rand((T, hq, d), 25)
    u = _rand((hq, d), 26)
    scale = 0.6
    o, lse = oracle.attn_fwd(q, k, v, scale=scale, causal=causal)
    o2, lse2 = oracle.attn_fwd(q, k + u[None], v, scale=scale, causal=causal)
    np.testing.assert_allclose(o2, o, atol=1e-12)
    shift = scale * np.einsum("thc,hc->ht", q, u)
    np.testing.assert_allclose(lse2, lse + shift, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_gradient_invariants(causal):
    lengths, hq, hkv, d = [9, 14], 6, 2, 5
    T = sum(lengths)
    cu = _cu(lengths)
    q, k, v, do = _rand((T, hq, d), 27), _rand((T, hkv, d), 28), _rand((T, hkv, d), 29), _rand((T, hq, d), 30)
    dq, dk, dv, o, lse = oracle.attn_bwd(q, k, v, do, cu, causal=causal)
    G = hq // hkv
    for b in range(len(lengths)):
        sl = slice(cu[b], cu[b + 1])
        # rows of dS sum to zero  =>  sum over keys of dK is zero per kv head
        np.testing.assert_allclose(dk[sl].sum(axis=0), 0.0, atol=1e-12)
        # rows of P sum to one  =>  sum over keys of dV = sum over rows of dO (group-summed)
        do_grp = do[sl].reshape(-1, hkv, G, d).sum(axis=2)
        np.testing.assert_allclose(dv[sl].sum(axis=0), do_grp.sum(axis=0), atol=1e-12)
    # D_i = sum_c dO_ic O_ic = sum_j P_ij dP_ij  (one head, first sequence)
    n = lengths[0]
    p, _ = oracle.attn_probs(q[:n, 0], k[:n, 0], scale=1 / math.sqrt(d), causal=causal)
    dp = do[:n, 0] @ v[:n, 0].T
    np.testing.assert_allclose((p * dp).sum(axis=1), np.einsum("ic,ic->i", do[:n, 0], o[:n, 0]), atol=1e-12)


def test_gqa_equals_repeated_mha():
    T, hq, hkv, d = 23, 6, 2, 4
    G = hq // hkv
    q, k, v, do = _rand((T, hq, d), 31), _rand((T, hkv, d), 32), _rand((T, hkv, d), 33), _rand((T, hq, d), 34)
    kr, vr = np.repeat(k, G, axis=1), np.repeat(v, G, axis=1)
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, v, causal=causal)
        o_r, lse_r = oracle.attn_fwd(q, kr, vr, causal=causal)
        np.testing.assert_allclose(o, o_r, atol=1e-14)
        np.testing.assert_allclose(lse, lse_r, atol=1e-14)
        dq, dk, dv, _, _ = oracle.attn_bwd(q, k, v, do, causal=causal)
        dq_r, dk_r, dv_r, _, _ = oracle.attn_bwd(q, kr, vr, do, causal=causal)
        np.testing.assert_allclose(dq, dq_r, atol=1e-13)
        np.testing.assert_allclose(dk, dk_r.reshape(T, hkv, G, d).sum(axis=2), atol=1e-13)
        np.testing.assert_allclose(dv, dv_r.reshape(T, hkv, G, d).sum(axis=2), atol=1e-13)


def test_varlen_equals_separate_calls():
    lengths, hq, hkv, d = [4, 1, 9, 6], 2, 1, 3
    T = sum(lengths)
    cu = _cu(lengths)
    q, k, v, do = _rand((T, hq, d), 35), _rand((T, hkv, d), 36), _rand((T, hkv, d), 37), _rand((T, hq, d), 38)
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, v, cu, causal=causal)
        dq, dk, dv, _, _ = oracle.attn_bwd(q, k, v, do, cu, causal=causal)
        for b in range(len(lengths)):
            sl = slice(cu[b], cu[b + 1])
            o_b, lse_b = oracle.attn_fwd(q[sl], k[sl], v[sl], causal=causal)
            dq_b, dk_b, dv_b, _, _ = oracle.attn_bwd(q[sl], k[sl], v[sl], do[sl], causal=causal)
            assert np.array_equal(o[sl], o_b) and np.array_equal(lse[:, sl], lse_b)
            assert np.array_equal(dq[sl], dq_b) and np.array_equal(dk[sl], dk_b) and np.array_equal(dv[sl], dv_b)


def test_empty_sequence_is_legal():
    lengths = [3, 0, 2]
    T = sum(lengths)
    q, k, v, do = _rand((T, 1, 2), 39), _rand((T, 1, 2), 40), _rand((T, 1, 2), 41), _rand((T, 1, 2), 42)
    o, lse = oracle.attn_fwd(q, k, v, _cu(lengths), causal=True)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    dq, dk, dv, _, _ = oracle.attn_bwd(q, k, v, do, _cu(lengths), causal=True)
    assert np.isfinite(dq).all() and np.isfinite(dk).all() and np.isfinite(dv).all()


def test_stability_large_scores():
    """x30 scores (row maxima far above 88, where a plain exp would overflow)."""
    T, hq, d = 40, 2, 16
    q, k, v = _rand((T, hq, d), 43, 30.0), _rand((T, hq, d), 44, 30.0), _rand((T, hq, d), 45)
    scale = 1 / math.sqrt(d)
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, v, scale=scale, causal=causal)
        assert np.isfinite(o).all() and np.isfinite(lse).all()
        for h in range(hq):
            s = scale * q[:, h] @ k[:, h].T
            if causal:
                s[np.triu_indices(T, 1)] = -np.inf
            m = s.max(axis=1)
            assert m.max() > 88
            cnt = np.arange(1, T + 1) if causal else np.full(T, T)
            assert (lse[h] >= m - 1e-9).all() and (lse[h] <= m + np.log(cnt) + 1e-9).all()


def test_row_and_key_selection_match_full():
    lengths, hq, hkv, d = [30, 11], 4, 2, 4
    T = sum(lengths)
    cu = _cu(lengths)
    q, k, v, do = _rand((T, hq, d), 46), _rand((T, hkv, d), 47), _rand((T, hkv, d), 48), _rand((T, hq, d), 49)
    rows = [0, 5, 29, 30, 40]
    keys = [1, 17, 31, 39]
    o, lse = oracle.attn_fwd(q, k, v, cu, causal=True)
    o_s, lse_s = oracle.attn_fwd(q, k, v, cu, causal=True, rows=rows)
    assert np.array_equal(o_s[rows], o[rows]) and np.array_equal(lse_s[:, rows], lse[:, rows])
    dq, dk, dv, _, _ = oracle.attn_bwd(q, k, v, do, cu, causal=True)
    dq_s, dk_s, dv_s, _, _ = oracle.attn_bwd(q, k, v, do, cu, causal=True, rows=rows, keys=keys)
    assert np.array_equal(dq_s[rows], dq[rows])
    assert np.array_equal(dk_s[keys], dk[keys]) and np.array_equal(dv_s[keys], dv[keys])


def test_thread_count_does_not_change_results():
    lengths, hq, hkv, d = [70, 33], 4, 2, 8
    T = sum(lengths)
    cu = _cu(lengths)
    q, k, v, do = _rand((T, hq, d), 50), _rand((T, hkv, d), 51), _rand((T, hkv, d), 52), _rand((T, hq, d), 53)
    a = oracle.attn_bwd(q, k, v, do, cu, causal=True, threads=1)
    b = oracle.attn_bwd(q, k, v, do, cu, causal=True, threads=7)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


# ---------------------------------------------------------------------------------------
# the backward as a function of its inputs (given O and LSE)
# ---------------------------------------------------------------------------------------
def test_backward_with_its_own_saved_outputs_is_unchanged():
    lengths, hq, hkv, d = [13, 6], 4, 2, 5
    T = sum(lengths)
    cu = _cu(lengths)
    q, k, v, do = _rand((T, hq, d), 60), _rand((T, hkv, d), 61), _rand((T, hkv, d), 62), _rand((T, hq, d), 63)
    a = oracle.attn_bwd(q, k, v, do, cu, causal=True)
    b = oracle.attn_bwd(q, k, v, do, cu, causal=True, o=a[3], lse=a[4])
    for x, y in zip(a[:3], b[:3]):
        np.testing.assert_allclose(x, y, rtol=0, atol=1e-13)


def test_given_lse_shift_scales_gradients_exactly():
    """LSE + c gives P e^-c, so dV, dS and with them dQ, dK scale by e^-c (D comes from O)."""
    T, hq, d = 17, 2, 4
    q, k, v, do = _rand((T, hq, d), 64), _rand((T, hq, d), 65), _rand((T, hq, d), 66), _rand((T, hq, d), 67)
    a = oracle.attn_bwd(q, k, v, do, causal=False)
    c = 0.37
    b = oracle.attn_bwd(q, k, v, do, causal=False, o=a[3], lse=a[4] + c)
    for x, y in zip(a[:3], b[:3]):
        np.testing.assert_allclose(y, x * math.exp(-c), rtol=1e-12, atol=1e-14)


def test_given_o_changes_dq_by_closed_form():
    """O + delta changes D_i by dO_i . delta_i; then dQ_i changes by
    -scale * (dO_i . delta_i) * sum_j P_ij K_j, and sum_j P_ij K_j is the forward with V = K."""
    T, hq, d = 15, 2, 3
    scale = 0.8
    q, k, v, do = _rand((T, hq, d), 68), _rand((T, hq, d), 69), _rand((T, hq, d), 70), _rand((T, hq, d), 71)
    a = oracle.attn_bwd(q, k, v, do, scale=scale, causal=True)
    delta = _rand((T, hq, d), 72, 1e-2)
    b = oracle.attn_bwd(q, k, v, do, scale=scale, causal=True, o=a[3] + delta, lse=a[4])
    pk, _ = oracle.attn_fwd(q, k, k, scale=scale, causal=True)
    want = a[0] - scale * np.einsum("thc,thc->th", do, delta)[:, :, None] * pk
    np.testing.assert_allclose(b[0], want, rtol=0, atol=1e-12)
