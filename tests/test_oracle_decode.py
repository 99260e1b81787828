"""Pins of the oracle's decoding-shaped forward (``oracle.attn_fwd_cross``).

The decode variant of the "FlashAttention 与高效注意力内核" tutorial (section
"FlashAttention 变体族谱", FlashDecoding: one query against a long KV) computes the same
three steps as the forward; only the shapes differ: sequence b has Lq query rows, the last
Lq positions of a sequence of Lk keys.  Each pin below comes from somewhere other than the
oracle's own code: a naive loop over explicit positions, torch's SDPA with an explicit
mask, the self-attention oracle (pinned in ``test_oracle``) when Lq = Lk, closed forms.
"""
import numpy as np
import pytest
import torch

import oracle


def _rand(rng, *shape, scale=1.0):
    return rng.standard_normal(shape) * scale


def _brute(q, k, v, cu_q, cu_k, scale, causal):
    """Naive: explicit query/key positions, exp without max subtraction (small inputs)."""
    Tq, hq, d = q.shape
    hkv = k.shape[1]
    o = np.zeros_like(q)
    lse = np.zeros((hq, Tq))
    for b in range(len(cu_q) - 1):
        lq, lk = cu_q[b + 1] - cu_q[b], cu_k[b + 1] - cu_k[b]
        for i in range(lq):
            pos = lk - lq + i                      # absolute position of query row i
            for h in range(hq):
                g = h // (hq // hkv)
                w, acc = 0.0, np.zeros(d)
                for j in range(lk):
                    if causal and j > pos:
                        continue
                    e = np.exp(scale * float(q[cu_q[b] + i, h] @ k[cu_k[b] + j, g]))
                    w += e
                    acc += e * v[cu_k[b] + j, g]
                o[cu_q[b] + i, h] = acc / w if w > 0 else 0.0
                lse[h, cu_q[b] + i] = np.log(w) if w > 0 else -np.inf
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("lens", [([1, 1, 1], [5, 1, 9]), ([2, 3], [7, 3]), ([4], [4]), ([1, 3], [2, 6])])
def test_cross_matches_brute_force(lens, causal):
    rng = np.random.default_rng(11)
    lq, lk = lens
    cu_q, cu_k = np.concatenate([[0], np.cumsum(lq)]), np.concatenate([[0], np.cumsum(lk)])
    hq, hkv, d = 4, 2, 3
    q, k, v = _rand(rng, cu_q[-1], hq, d, scale=0.7), _rand(rng, cu_k[-1], hkv, d, scale=0.7), _rand(rng, cu_k[-1], hkv, d)
    o, lse = oracle.attn_fwd_cross(q, k, v, cu_q, cu_k, scale=0.9, causal=causal)
    ob, lb = _brute(q, k, v, cu_q, cu_k, 0.9, causal)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lb, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_cross_matches_torch_sdpa_with_explicit_mask(causal):
    rng = np.random.default_rng(5)
    lq, lk, hq, hkv, d = 3, 17, 6, 3, 8
    q, k, v = _rand(rng, lq, hq, d), _rand(rng, lk, hkv, d), _rand(rng, lk, hkv, d)
    o, lse = oracle.attn_fwd_cross(q, k, v, [0, lq], [0, lk], causal=causal)
    G = hq // hkv
    qt = torch.tensor(q).permute(1, 0, 2)                              # [hq, lq, d]
    kt = torch.tensor(k).permute(1, 0, 2).repeat_interleave(G, 0)     # [hq, lk, d]
    vt = torch.tensor(v).permute(1, 0, 2).repeat_interleave(G, 0)
    pos_q = torch.arange(lq)[:, None] + (lk - lq)
    mask = (torch.arange(lk)[None, :] <= pos_q) if causal else torch.ones(lq, lk, dtype=torch.bool)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask)
    np.testing.assert_allclose(o, ref.permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)
    s = (qt @ kt.transpose(1, 2)) / np.sqrt(d)
    s = s.masked_fill(~mask, float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_cross_with_equal_lengths_is_self_attention(causal):
    rng = np.random.default_rng(3)
    cu = np.array([0, 5, 12, 13])
    q, k, v = _rand(rng, 13, 4, 8), _rand(rng, 13, 1, 8), _rand(rng, 13, 1, 8)
    o, lse = oracle.attn_fwd_cross(q, k, v, cu, cu, causal=causal)
    o2, lse2 = oracle.attn_fwd(q, k, v, cu_seqlens=cu, causal=causal)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)


def test_cross_zero_queries_average_the_visible_values():
    """Q = 0: every visible key has the same score, so O is the mean of the visible V
    rows and LSE = ln(number visible)."""
    rng = np.random.default_rng(8)
    lq, lk, d = 3, 10, 4
    q, k, v = np.zeros((lq, 2, d)), _rand(rng, lk, 1, d), _rand(rng, lk, 1, d)
    o, lse = oracle.attn_fwd_cross(q, k, v, [0, lq], [0, lk], causal=True)
    for i in range(lq):
        vis = lk - lq + i + 1
        np.testing.assert_allclose(o[i, :, :], np.broadcast_to(v[:vis, 0].mean(0), (2, d)), rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[:, i], np.log(vis), rtol=0, atol=1e-14)


def test_cross_single_query_sees_every_key():
    rng = np.random.default_rng(9)
    q, k, v = _rand(rng, 2, 2, 4), _rand(rng, 11, 2, 4), _rand(rng, 11, 2, 4)
    a = oracle.attn_fwd_cross(q, k, v, [0, 1, 2], [0, 6, 11], causal=True)
    b = oracle.attn_fwd_cross(q, k, v, [0, 1, 2], [0, 6, 11], causal=False)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_cross_empty_kv_gives_zero_output_and_minus_inf():
    rng = np.random.default_rng(2)
    q, k, v = _rand(rng, 2, 2, 4), _rand(rng, 3, 2, 4), _rand(rng, 3, 2, 4)
    o, lse = oracle.attn_fwd_cross(q, k, v, [0, 1, 2], [0, 0, 3])
    assert np.all(o[0] == 0.0) and np.all(lse[:, 0] == -np.inf)
    assert np.all(np.isfinite(o[1])) and np.all(np.isfinite(lse[:, 1]))


def test_cross_gqa_equals_repeated_heads():
    rng = np.random.default_rng(4)
    q, k, v = _rand(rng, 2, 8, 4), _rand(rng, 9, 2, 4), _rand(rng, 9, 2, 4)
    a = oracle.attn_fwd_cross(q, k, v, [0, 2], [0, 9], causal=True)
    b = oracle.attn_fwd_cross(q, np.repeat(k, 4, axis=1), np.repeat(v, 4, axis=1), [0, 2], [0, 9], causal=True)
    np.testing.assert_allclose(a[0], b[0], rtol=0, atol=1e-14)
    np.testing.assert_allclose(a[1], b[1], rtol=0, atol=1e-14)
