"""Parity at the full sizes of the five benchmark configurations.

The GPU runs every configuration whole, in the launch configuration bench.py uses.  The
fp64 oracle then recomputes sampled (sequence, GQA group) slices -- each slice whole, so
every row enters the statistics -- and the outputs are compared on sampled query rows
(O, LSE, dQ) and sampled keys (dK, dV).  Sum invariants of the backward are checked over
everything."""
import functools

import pytest
import torch

import attn_workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu


@functools.lru_cache(maxsize=2)
def _inputs(name, d=None, n=None):
    if name == "sweep":
        return W.make_inputs(W.sweep(d, n))
    if name == "gqa8k":
        return W.make_inputs(W.gqa8k())
    if name == "gqa8k_x30":
        return W.make_inputs(W.gqa8k(stability=True))
    if name == "varlen16":
        return W.make_inputs(W.varlen16())
    if name == "long32k":
        return W.make_inputs(W.long32k())
    raise KeyError(name)


def _run_and_check(w, inputs, picks, seed, **kw):
    out = P.run_full(w, inputs)
    report = P.check_sampled(w, inputs, out, picks, seed=seed, tag=w.name, **kw)
    P.check_sum_properties(w, inputs[4], inputs[3], out[3], out[4], tag=w.name)
    del out
    torch.cuda.empty_cache()
    return report


# Config 4b against the plain definition (the device's forward and backward against the
# exact fp64 gradients and LSE), measured on B200 over the sampled slices below: max over
# slices of rel-L2 dQ 2.76e-2, dK 1.08e-2, dV 1.7e-3 and max |LSE - LSE_ref| 1.09e-3, against
# stated tolerances of 1e-2 and 1e-3.  dQ and dK miss them, and no backward that takes a
# bf16 O can meet them here: the oracle's own backward, given its own forward rounded as
# attn_fwd stores it (bf16 O, fp32 LSE), is already 1.31e-2 (dQ) and 1.12e-2 (dK) away
# from the exact gradient on slice (1, 7) (tests/test_oracle_x30.py pins this).  With P
# nearly one-hot, dS = P (dP - D) cancels, and D = rowsum(dO o O) carries the rounding of
# the stored O.  The LSE misses 1e-3 by 9%: 1e-3 is below two fp32 ulps at |LSE| ~ 5000.
# These ceilings catch a regression; they do not claim the tolerance is met.
X30_STRICT_CEILING = {"dq": 3.0e-2, "dk": 1.2e-2, "dv": 2.5e-3, "lse": 1.2e-3}


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n", W.SWEEP_N)
@pytest.mark.parametrize("d", W.SWEEP_D)
def test_sweep(d, n, causal):
    w = W.sweep(d, n, causal)
    picks = [(0, 0), (w.batch - 1, w.hkv - 1)] if n <= 4096 else [(w.batch - 1, w.hkv - 1)]
    _run_and_check(w, _inputs("sweep", d, n), picks, seed=d + n)


def test_gqa8k():
    w = W.gqa8k()
    _run_and_check(w, _inputs("gqa8k"), [(0, 0), (1, 7)], seed=8)


def test_gqa8k_stability_x30():
    """Q and K x30: row maxima of the scores in the thousands.  The online max / rescale
    must stay finite and exact.  Two checks differ from the other configurations, both
    derived from the arithmetic rather than loosened:
      - LSE: 1e-3 is below two fp32 ulps at |LSE| ~ 5000, so each row is held to
        max(1e-3, fp32_lse_bound) (fp32 accumulation of the row's largest score, fp32
        storage of the LSE);
      - gradients: with P nearly one-hot, dS = P (dP - D) is a cancellation that
        amplifies the rounding of the saved bf16 O (through D) about a hundredfold
        relative to dS, so the backward is compared as a function of its inputs -- the
        oracle's forward of each sampled slice, stored as bf16 O and fp32 LSE, is given
        to both the GPU backward (rerun on it) and the oracle's backward -- at the usual
        1e-2."""
    w = W.gqa8k(stability=True)
    report = _run_and_check(w, _inputs("gqa8k_x30"), [(0, 0), (1, 7)], seed=8, given=True,
                            fp32_lse_bound_rows=True, strict=True)
    worst = {k: max(r[3][k] for r in report) for k in X30_STRICT_CEILING}
    print(f"gqa8k_x30 against the exact definition: {worst}")
    for k, ceiling in X30_STRICT_CEILING.items():
        assert worst[k] <= ceiling, f"x30 strict {k}: {worst[k]:.3e} above the recorded ceiling {ceiling:.1e}"


def test_varlen16():
    w = W.varlen16()
    lens = list(w.lengths)
    shortest, longest = lens.index(min(lens)), lens.index(max(lens))
    _run_and_check(w, _inputs("varlen16"), [(shortest, 3), (longest, 11), (7, 0)], seed=16)


def test_long32k():
    w = W.long32k()
    _run_and_check(w, _inputs("long32k"), [(0, 0), (0, 15)], seed=32)
