"""Pins of the oracle's FP8 forward (``oracle.attn_fwd_fp8sim``, ``oracle.round_e4m3``).

The FP8 forward is an approximation, so the oracle takes its steps (blockwise online
softmax with conditional rescaling, probabilities rounded to e4m3 before they multiply
V).  Each pin comes from outside that code: torch's float8_e4m3fn conversion for the
rounding, the exact forward (pinned in ``test_oracle``) for the blockwise softmax with the
rounding switched off, closed forms, and a two-key example whose rounding is stated by
hand.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def test_e4m3_rounding_matches_torch():
    grid = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).float()   # every finite value >= 0
    grid = grid[torch.isfinite(grid)]
    mids = (grid[1:] + grid[:-1]) / 2                                                    # ties: to even
    rng = np.random.default_rng(0)
    rand = torch.tensor(rng.uniform(-448, 448, 4000), dtype=torch.float32)
    small = torch.tensor(rng.uniform(-0.05, 0.05, 4000), dtype=torch.float32)
    for x in (grid, -grid, mids, -mids, rand, small):
        want = x.to(torch.float8_e4m3fn).float().numpy()
        got = np.array([oracle.round_e4m3(float(v)) for v in x.numpy()])
        np.testing.assert_array_equal(got, want)
    assert oracle.round_e4m3(500.0) == 448.0 and oracle.round_e4m3(-1e6) == -448.0   # saturating


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("mult", [1.0, 30.0])
def test_unrounded_steps_equal_the_exact_forward(causal, mult):
    """round_p = False: the blockwise online softmax (several 128-key blocks, rescales
    skipped below 8 log2 units and taken above) reaches the plain definition."""
    rng = np.random.default_rng(3)
    cu = np.array([0, 300, 301, 700])
    hq, hkv, d = 4, 2, 16
    q = rng.standard_normal((700, hq, d)) * mult
    k = rng.standard_normal((700, hkv, d)) * mult
    v = rng.standard_normal((700, hkv, d))
    o, lse = oracle.attn_fwd_fp8sim(q, k, v, cu, causal=causal, round_p=False)
    o2, lse2 = oracle.attn_fwd(q, k, v, cu, causal=causal)
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse2, rtol=1e-14, atol=1e-11)


def test_zero_queries_give_the_exact_average_even_rounded():
    """Q = 0: every visible probability is exactly 1 = e4m3(1), so O is the mean of the
    visible V rows and LSE = ln(count), rounding or not."""
    rng = np.random.default_rng(4)
    n, d = 260, 8
    q = np.zeros((n, 2, d))
    k, v = rng.standard_normal((n, 1, d)), rng.standard_normal((n, 1, d))
    o, lse = oracle.attn_fwd_fp8sim(q, k, v, causal=True)
    for i in (0, 127, 128, 259):
        np.testing.assert_allclose(o[i, 0], v[:i + 1, 0].mean(0), rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[0, i], math.log(i + 1), rtol=0, atol=1e-14)


def test_two_key_example_rounds_the_weights_but_not_the_sum():
    """One query, keys with scores 0 and ln(1.0625) (scale 1): the block max makes the
    probabilities 1/1.0625 = 0.94117... and 1.  On the e4m3 grid (spacing 2^-4 in
    [0.5, 1)) 0.94117 rounds to 0.9375 and 1 stays 1; the row sum is not rounded.  With
    v = (1, 0): O = 0.9375 / (1/1.0625 + 1), LSE = ln(1 + 1.0625)."""
    q = np.array([[[1.0]]])
    k = np.array([[[0.0]], [[math.log(1.0625)]]])
    v = np.array([[[1.0]], [[0.0]]])
    o, lse = oracle.attn_fwd_fp8sim(np.repeat(q, 2, axis=0), k, v, [0, 2], scale=1.0)
    assert oracle.round_e4m3(1 / 1.0625) == 0.9375
    np.testing.assert_allclose(o[0, 0, 0], 0.9375 / (1 / 1.0625 + 1), rtol=1e-15)
    np.testing.assert_allclose(lse[0, 0], math.log(1 + 1.0625), rtol=1e-15)


def test_rounding_changes_the_output_by_a_bounded_amount():
    """Rounded vs exact on random data: each weight moves by at most 2^-4 relative, so O
    moves by at most 2^-4 max|V| and typically far less."""
    rng = np.random.default_rng(5)
    q, k, v = rng.standard_normal((400, 2, 32)), rng.standard_normal((400, 2, 32)), rng.standard_normal((400, 2, 32))
    o, _ = oracle.attn_fwd_fp8sim(q, k, v, causal=True)
    o2, _ = oracle.attn_fwd_fp8sim(q, k, v, causal=True, round_p=False)
    err = np.abs(o - o2).max()
    assert 0 < err <= 2 ** -4 * np.abs(v).max()


@pytest.mark.parametrize("causal", [False, True])
def test_rounded_weights_leave_the_lse_exact(causal):
    """The row sum is formed from the unrounded weights, so with the rounding on the LSE
    is still the exact one (the rounding only touches the weighted sum of V)."""
    rng = np.random.default_rng(7)
    cu = np.array([0, 260, 700])
    hq, hkv, d = 2, 1, 32
    q = rng.standard_normal((700, hq, d)) * 2.0
    k = rng.standard_normal((700, hkv, d)) * 2.0
    v = rng.standard_normal((700, hkv, d))
    o, lse = oracle.attn_fwd_fp8sim(q, k, v, cu, causal=causal, round_p=True)
    o2, lse2 = oracle.attn_fwd(q, k, v, cu, causal=causal)
    np.testing.assert_allclose(lse, lse2, rtol=1e-14, atol=1e-11)
    assert np.abs(o - o2).max() > 1e-6          # while O does move with the rounding
