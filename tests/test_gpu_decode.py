"""Parity of the split-KV decoding forward (attn_fwd_decode) with the fp64 oracle.

Every case runs the CUDA library through the C ABI and ``oracle.attn_fwd_cross`` on the
same seeded bf16 inputs, element by element, with the forward's tolerances
(max |O - O_ref| <= 2e-2, rel-L2(O) <= 5e-3, max |LSE - LSE_ref| <= 1e-3).  Rows with
no visible key must come out exactly as the definition says: O = 0, LSE = -inf.
"""
import numpy as np
import pytest
import torch

import attn_workloads as W
import io_aware_exact_qk_b200 as attn
import oracle
from tests import parity

pytestmark = pytest.mark.gpu


def run_gpu(w, q, k, v, cu_q, cu_k, num_splits=0, varlen=True):
    dev = torch.device("cuda")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    if varlen:
        o, lse = attn.attn_fwd_decode(qd, kd, vd, cu_seqlens_q=cu_q.to(dev), cu_seqlens_k=cu_k.to(dev),
                                      max_seqlen_q=max(w.q_lens), max_seqlen_k=w.max_k, scale=w.scale,
                                      causal=w.causal, num_splits=num_splits)
    else:
        o, lse = attn.attn_fwd_decode(qd, kd, vd, batch=w.batch, scale=w.scale, causal=w.causal,
                                      num_splits=num_splits)
    attn.attn_get_device_error()
    return o, lse


def check(w, o, lse, o_ref, lse_ref, tag):
    o, lse = parity.to_np(o), parity.to_np(lse)
    empty = ~np.isfinite(lse_ref)                      # [hq, Tq]: rows with no visible key
    assert np.array_equal(~np.isfinite(lse), empty), f"{tag}: rows without keys differ"
    assert np.all(lse[empty] == -np.inf), tag
    assert np.all(o.transpose(1, 0, 2)[empty] == 0.0), f"{tag}: O of a row without keys is not 0"
    full = ~empty.T                                    # [Tq, hq]
    if full.any():
        oo, orf = o[full], o_ref[full]
        e_max = float(np.abs(oo - orf).max())
        e_rel = parity.rel_l2(oo, orf)
        e_lse = float(np.abs(lse[~empty] - lse_ref[~empty]).max())
        assert np.isfinite(oo).all(), tag
        assert e_max <= parity.BF16_O_MAX_ABS, f"{tag} max|dO| {e_max}"
        assert e_rel <= parity.BF16_O_REL_L2, f"{tag} relL2(O) {e_rel}"
        assert e_lse <= parity.BF16_LSE_MAX_ABS, f"{tag} max|dLSE| {e_lse}"


def case(name, q_lens, k_lens, hq, hkv, d, causal, seed, splits=(0,), varlen=True, scale=None):
    w = W.decode_custom(name, q_lens, k_lens, hq, hkv, d, causal, seed, scale=scale)
    q, k, v, cu_q, cu_k = W.make_decode_inputs(w)
    o_ref, lse_ref = oracle.attn_fwd_cross(q, k, v, cu_q.numpy(), cu_k.numpy(), scale=w.scale, causal=causal)
    for s in splits:
        o, lse = run_gpu(w, q, k, v, cu_q, cu_k, num_splits=s, varlen=varlen)
        check(w, o, lse, o_ref, lse_ref, f"{name} splits={s}")


@pytest.mark.parametrize("d", [128, 64, 32])
def test_batch_mode_single_query_gqa(d):
    # 3 sequences of 1000 keys (a ragged last tile), one query each, 4 query heads per KV head
    case(f"b3_d{d}", [1] * 3, [1000] * 3, 8, 2, d, False, 2001, splits=(0, 1, 3, 8), varlen=False)


def test_varlen_lengths_around_tile_edges():
    case("edges", [1] * 6, [1, 127, 128, 129, 700, 2049], 16, 4, 128, False, 2002, splits=(0, 1, 2, 5))


def test_empty_kv_sequence():
    case("empty_kv", [1, 1, 1], [300, 0, 5], 8, 8, 128, False, 2003, splits=(0, 1, 3))


@pytest.mark.parametrize("d", [128, 64])
def test_speculative_rows_causal(d):
    # 4 newest tokens per sequence, bottom-right causal; 8 query heads per KV head = 32 rows
    case(f"spec_d{d}", [4, 4, 4], [4, 130, 515], 16, 2, d, True, 2004, splits=(0, 1, 2))


def test_more_query_rows_than_keys_leaves_early_rows_empty():
    # Lq = 4 > Lk = 2: causal rows 0 and 1 see no key (O = 0, LSE = -inf)
    case("lq_gt_lk", [4, 4], [2, 9], 4, 1, 128, True, 2005, splits=(0, 1, 2))


def test_full_tile_of_rows_and_mha():
    case("rows128", [4, 4], [600, 333], 32, 1, 128, True, 2006, splits=(0, 3))      # 32 heads x 4 rows = 128
    case("mha_one_row", [1, 1], [777, 1500], 4, 4, 64, False, 2007, splits=(0, 4))  # one row per tile


@pytest.mark.parametrize("scale", [0.04, 0.3])
def test_explicit_scale_three_heads_per_group(scale):
    # a score scale other than 1/sqrt(d), 3 query heads per KV head, causal speculative rows
    case(f"scale{scale}", [2, 3, 1], [700, 65, 2000], 6, 2, 128, True, 2010, splits=(0, 1, 3), scale=scale)


def test_varlen_query_lengths_differ():
    case("mixed_q", [1, 3, 2], [50, 400, 129], 8, 2, 128, True, 2008, splits=(0, 2))


@pytest.mark.parametrize("make", [W.decode8k, W.decode_var, W.decode_spec4])
def test_full_size_decode_workloads(make):
    """The full decode workloads, every row against the oracle (fp64, all host threads)."""
    w = make()
    q, k, v, cu_q, cu_k = W.make_decode_inputs(w)
    o_ref, lse_ref = oracle.attn_fwd_cross(q, k, v, cu_q.numpy(), cu_k.numpy(), scale=w.scale, causal=w.causal)
    o, lse = run_gpu(w, q, k, v, cu_q, cu_k)
    check(w, o, lse, o_ref, lse_ref, w.name)


def test_split_count_does_not_change_the_result_beyond_rounding():
    """Splitting is exact up to rounding: 1, 2 and 7 splits agree to fp32-combine accuracy
    (the partial O_s are fp32; the combine adds at most a few ulps)."""
    w = W.decode_custom("split_inv", [1] * 4, [3000] * 4, 8, 2, 128, False, 2009)
    q, k, v, cu_q, cu_k = W.make_decode_inputs(w)
    outs = [run_gpu(w, q, k, v, cu_q, cu_k, num_splits=s) for s in (1, 2, 7)]
    base_o, base_l = parity.to_np(outs[0][0]), parity.to_np(outs[0][1])
    for o, lse in outs[1:]:
        assert float(np.abs(parity.to_np(o) - base_o).max()) <= 2 ** -7   # within bf16 output rounding
        assert float(np.abs(parity.to_np(lse) - base_l).max()) <= 1e-5
