"""Parity of the FP8 (e4m3) forward with the fp64 oracle.

Two calls are under test, both through the C ABI:

* ``attn_fp8_quantize`` must reproduce, byte for byte, the per-head quantisation that this
  file states on the CPU: descale = amax / 448 in fp32, x8 = e4m3(x / descale) with an
  fp32 division and round-to-nearest-even (torch's float8_e4m3fn conversion, which
  ``test_oracle_fp8`` pins to the oracle's rounding).  V goes out transposed per
  (sequence, kv head) with a zero-padded token pitch.
* ``attn_fwd_fp8`` runs on operands quantised here on the CPU (never on the GPU's own
  quantisation), and ``oracle.attn_fwd_fp8sim`` runs on the same operands dequantised to
  fp64.  The oracle takes the kernel's steps (128-key blocks, running max moved only past
  8 log2 units, probabilities rounded to e4m3 before they multiply V), so the two agree
  to the forward's bf16 tolerances (max |O - O_ref| <= 2e-2, rel-L2(O) <= 5e-3,
  max |LSE - LSE_ref| <= 1e-3).  Against the exact forward of the dequantised operands
  the probability rounding alone leaves a few 1e-2 of relative error, bounded below.
"""
import numpy as np
import pytest
import torch

import attn_workloads as W
import io_aware_exact_qk_b200 as attn
import oracle
from tests import parity

pytestmark = pytest.mark.gpu

E4M3_MAX = 448.0
# rel-L2 of O against the exact forward of the dequantised operands: P rounded to e4m3
# has a relative error of at most 2^-4 per entry, about 2^-6 in root-mean-square.
FP8_EXACT_REL_L2 = 3e-2


def pitch_of(seqlen):
    return (seqlen + 15) // 16 * 16


def quantize_cpu(x, heads):
    """x [T, heads, d] bf16 -> (e4m3 bytes [T, heads, d] uint8, descale [heads] float32)."""
    xf = x.float()
    amax = xf.abs().amax(dim=(0, 2))                                    # exact: bf16 values
    ds = torch.where(amax > 0, amax / torch.tensor(E4M3_MAX, dtype=torch.float32), torch.ones_like(amax))
    y = (xf / ds[None, :, None]).clamp(-E4M3_MAX, E4M3_MAX)            # fp32 division
    x8 = y.to(torch.float8_e4m3fn).view(torch.uint8)
    return x8, ds


def transpose_v_cpu(v8, batch, seqlen):
    """v8 [B S, hkv, d] -> [B hkv, d, pitch] with zero padding."""
    T, hkv, d = v8.shape
    out = torch.zeros(batch * hkv, d, pitch_of(seqlen), dtype=torch.uint8)
    out[:, :, :seqlen] = v8.view(batch, seqlen, hkv, d).permute(0, 2, 3, 1).reshape(batch * hkv, d, seqlen)
    return out


def transpose_v_cpu_varlen(v8, cu, max_seqlen):
    """v8 [T, hkv, d] packed by cu_seqlens -> [batch hkv, d, pitch(max_seqlen)]: sequence b's
    tokens at columns 0 .. len_b - 1, zeros after them."""
    T, hkv, d = v8.shape
    batch = len(cu) - 1
    out = torch.zeros(batch, hkv, d, pitch_of(max_seqlen), dtype=torch.uint8)
    for b in range(batch):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        out[b, :, :, :s1 - s0] = v8[s0:s1].permute(1, 2, 0)
    return out.reshape(batch * hkv, d, pitch_of(max_seqlen))


def dequant(x8, ds):
    return x8.view(torch.float8_e4m3fn).double() * ds.double()[None, :, None]


def fp8_case(name, batch, seqlen, hq, hkv, causal, seed, qk_mult=1.0, d=128):
    w = W.custom(name, [seqlen] * batch, hq, hkv, d, causal, seed, qk_mult=qk_mult)
    q, k, v, _, _ = W.make_inputs(w, with_grad=False)
    return w, q, k, v


CASES = [
    # name, batch, seqlen, hq, hkv, causal, seed, d
    ("fp8-1000-gqa", 2, 1000, 4, 2, False, 11, 128),
    ("fp8-1000-gqa-causal", 2, 1000, 4, 2, True, 12, 128),
    ("fp8-257", 1, 257, 2, 2, False, 13, 128),
    ("fp8-257-causal", 1, 257, 2, 1, True, 14, 128),
    ("fp8-2048-causal", 1, 2048, 2, 2, True, 15, 128),
    ("fp8-77", 3, 77, 2, 1, False, 16, 128),
    ("fp8-1", 2, 1, 2, 2, True, 20, 128),
    ("fp8-d64-1000-gqa", 2, 1000, 4, 2, False, 17, 64),
    ("fp8-d64-300-causal", 1, 300, 8, 2, True, 18, 64),
    ("fp8-d64-2048-causal", 1, 2048, 2, 2, True, 19, 64),
    ("fp8-d64-33", 3, 33, 2, 1, False, 21, 64),
]


def run_fwd(w, q8, k8, vt8, dq, dk, dv):
    dev = torch.device("cuda")
    o, lse = attn.attn_fwd_fp8(q8.to(dev), k8.to(dev), vt8.to(dev), dq.to(dev), dk.to(dev), dv.to(dev),
                               batch=w.batch, scale=w.scale, causal=w.causal)
    attn.attn_get_device_error()
    return parity.to_np(o), parity.to_np(lse)


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_fp8_quantize_bit_exact(case):
    name, batch, seqlen, hq, hkv, causal, seed, d = case
    w, q, k, v = fp8_case(name, batch, seqlen, hq, hkv, causal, seed, d=d)
    dev = torch.device("cuda")
    q8, k8, vt8, dq, dk, dv = attn.attn_fp8_quantize(q.to(dev), k.to(dev), v.to(dev), batch)
    attn.attn_get_device_error()
    q8_ref, dq_ref = quantize_cpu(q, hq)
    k8_ref, dk_ref = quantize_cpu(k, hkv)
    v8_ref, dv_ref = quantize_cpu(v, hkv)
    assert torch.equal(dq.cpu(), dq_ref) and torch.equal(dk.cpu(), dk_ref) and torch.equal(dv.cpu(), dv_ref)
    assert torch.equal(q8.cpu(), q8_ref)
    assert torch.equal(k8.cpu(), k8_ref)
    assert tuple(vt8.shape) == (batch * hkv, d, pitch_of(seqlen))
    assert torch.equal(vt8.cpu(), transpose_v_cpu(v8_ref, batch, seqlen))


def test_fp8_quantize_zero_head_and_outlier_head():
    """An all-zero head gets descale 1 and zero bytes; a head 300x larger gets its own scale."""
    batch, seqlen, hq, hkv = 1, 200, 3, 3
    w, q, k, v = fp8_case("fp8-heads", batch, seqlen, hq, hkv, False, 21)
    q[:, 0] = 0
    k[:, 2] *= 300
    dev = torch.device("cuda")
    q8, k8, vt8, dq, dk, dv = attn.attn_fp8_quantize(q.to(dev), k.to(dev), v.to(dev), batch)
    attn.attn_get_device_error()
    assert float(dq[0]) == 1.0 and int(q8[:, 0].abs().sum()) == 0
    k8_ref, dk_ref = quantize_cpu(k, hkv)
    assert torch.equal(dk.cpu(), dk_ref) and torch.equal(k8.cpu(), k8_ref)


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_fp8_forward_matches_oracle(case):
    name, batch, seqlen, hq, hkv, causal, seed, d = case
    w, q, k, v = fp8_case(name, batch, seqlen, hq, hkv, causal, seed, d=d)
    q8, dq = quantize_cpu(q, hq)
    k8, dk = quantize_cpu(k, hkv)
    v8, dv = quantize_cpu(v, hkv)
    vt8 = transpose_v_cpu(v8, batch, seqlen)
    o, lse = run_fwd(w, q8, k8, vt8, dq, dk, dv)
    qd, kd, vd = dequant(q8, dq).numpy(), dequant(k8, dk).numpy(), dequant(v8, dv).numpy()
    cu = w.cu_seqlens().numpy()
    o_ref, lse_ref = oracle.attn_fwd_fp8sim(qd, kd, vd, cu, scale=w.scale, causal=causal)
    parity.check_fwd_bf16(o, lse, o_ref, lse_ref, tag=name)
    # the approximation itself: against the exact forward of the same operands
    o_ex, lse_ex = oracle.attn_fwd(qd, kd, vd, cu, scale=w.scale, causal=causal)
    assert parity.rel_l2(o, o_ex) <= FP8_EXACT_REL_L2, name
    assert np.abs(lse - lse_ex).max() <= parity.BF16_LSE_MAX_ABS, name


@pytest.mark.parametrize("scale", [0.03, 0.3])
def test_fp8_forward_explicit_scale(scale):
    """A score scale other than 1/sqrt(d) (it multiplies the two descales in the kernel),
    three query heads per K/V head, packed sequences."""
    w = W.custom(f"fp8-scale{scale}", [300, 129, 513], 6, 2, 128, True, 58, scale=scale)
    q, k, v, _, cu = W.make_inputs(w, with_grad=False)
    q8, dq = quantize_cpu(q, w.hq)
    k8, dk = quantize_cpu(k, w.hkv)
    v8, dv = quantize_cpu(v, w.hkv)
    vt8 = transpose_v_cpu_varlen(v8, cu.tolist(), w.max_seqlen)
    dev = torch.device("cuda")
    o, lse = attn.attn_fwd_fp8(q8.to(dev), k8.to(dev), vt8.to(dev), dq.to(dev), dk.to(dev), dv.to(dev),
                               cu_seqlens=cu.to(dev), max_seqlen=w.max_seqlen, scale=scale, causal=True)
    attn.attn_get_device_error()
    qd, kd, vd = dequant(q8, dq).numpy(), dequant(k8, dk).numpy(), dequant(v8, dv).numpy()
    o_ref, lse_ref = oracle.attn_fwd_fp8sim(qd, kd, vd, cu.numpy(), scale=scale, causal=True)
    parity.check_fwd_bf16(parity.to_np(o), parity.to_np(lse), o_ref, lse_ref, tag=w.name)


def test_fp8_forward_large_scores_and_uneven_scales():
    """Q and K four times larger (scores of ~±20 in log2 units: the running max moves in
    large jumps and stays stale by up to 8) and per-head scales that differ by orders of
    magnitude."""
    batch, seqlen, hq, hkv = 1, 640, 4, 2
    w, q, k, v = fp8_case("fp8-large", batch, seqlen, hq, hkv, True, 31, qk_mult=4.0)
    q[:, 1] *= 0.01
    k[:, 1] *= 40.0
    q8, dq = quantize_cpu(q, hq)
    k8, dk = quantize_cpu(k, hkv)
    v8, dv = quantize_cpu(v, hkv)
    o, lse = run_fwd(w, q8, k8, transpose_v_cpu(v8, batch, seqlen), dq, dk, dv)
    qd, kd, vd = dequant(q8, dq).numpy(), dequant(k8, dk).numpy(), dequant(v8, dv).numpy()
    o_ref, lse_ref = oracle.attn_fwd_fp8sim(qd, kd, vd, w.cu_seqlens().numpy(), scale=w.scale, causal=True)
    parity.check_fwd_bf16(o, lse, o_ref, lse_ref, tag="fp8-large")


def test_fp8_end_to_end_through_quantize():
    """attn_fp8_quantize then attn_fwd_fp8 on the device, compared with the oracle on the
    CPU-quantised operands (equal bytes, checked above)."""
    batch, seqlen, hq, hkv = 2, 384, 4, 4
    w, q, k, v = fp8_case("fp8-e2e", batch, seqlen, hq, hkv, False, 41)
    dev = torch.device("cuda")
    ops = attn.attn_fp8_quantize(q.to(dev), k.to(dev), v.to(dev), batch)
    o, lse = attn.attn_fwd_fp8(*ops, batch=batch, scale=w.scale, causal=False)
    attn.attn_get_device_error()
    q8, dq = quantize_cpu(q, hq)
    k8, dk = quantize_cpu(k, hkv)
    v8, dv = quantize_cpu(v, hkv)
    o_ref, lse_ref = oracle.attn_fwd_fp8sim(dequant(q8, dq).numpy(), dequant(k8, dk).numpy(),
                                            dequant(v8, dv).numpy(), w.cu_seqlens().numpy(), scale=w.scale)
    parity.check_fwd_bf16(parity.to_np(o), parity.to_np(lse), o_ref, lse_ref, tag="fp8-e2e")


def test_fp8_empty_batch_is_a_no_op():
    dev = torch.device("cuda")
    z8 = torch.empty(0, 2, 128, dtype=torch.uint8, device=dev)
    vt = torch.empty(0, 128, 0, dtype=torch.uint8, device=dev)
    ds = torch.ones(2, dtype=torch.float32, device=dev)
    o, lse = attn.attn_fwd_fp8(z8, z8, vt, ds, ds, ds, batch=0)
    attn.attn_get_device_error()
    assert o.numel() == 0 and lse.numel() == 0


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_forward_bench_size_sampled_heads(causal):
    """The bench's FP8 configuration (B=4, H=16, N=2048, d=128) in one launch, as the bench
    runs it; the oracle checks two whole heads of two sequences (its cost grows with N^2
    per head, so not all 64 (sequence, head) pairs)."""
    w = W.mha2k(causal)
    q, k, v, _, _ = W.make_inputs(w, with_grad=False)
    q8, dq = quantize_cpu(q, w.hq)
    k8, dk = quantize_cpu(k, w.hkv)
    v8, dv = quantize_cpu(v, w.hkv)
    o, lse = run_fwd(w, q8, k8, transpose_v_cpu(v8, w.batch, w.seqlen), dq, dk, dv)
    qd, kd, vd = dequant(q8, dq).numpy(), dequant(k8, dk).numpy(), dequant(v8, dv).numpy()
    n = w.seqlen
    for b, h in ((0, 3), (3, 14)):
        rows = slice(b * n, (b + 1) * n)
        o_ref, lse_ref = oracle.attn_fwd_fp8sim(qd[rows, h:h + 1], kd[rows, h:h + 1], vd[rows, h:h + 1],
                                                scale=w.scale, causal=causal)
        parity.check_fwd_bf16(o[rows, h:h + 1], lse[h:h + 1, rows], o_ref, lse_ref, tag=f"fp8 b{b} h{h}")


VARLEN_CASES = [
    # name, sequence lengths, hq, hkv, causal, seed, d
    ("fp8-varlen-gqa", [100, 700, 300, 1, 129], 4, 2, False, 51, 128),
    ("fp8-varlen-gqa-causal", [100, 700, 300, 1, 129], 4, 2, True, 52, 128),
    ("fp8-varlen-d64-causal", [513, 64, 1000, 17], 8, 2, True, 53, 64),
    ("fp8-varlen-d64", [256, 255, 2], 2, 1, False, 54, 64),
    ("fp8-varlen-empty-seq", [300, 0, 130], 2, 2, True, 55, 128),
]


def fp8_varlen_case(case):
    name, lens, hq, hkv, causal, seed, d = case
    w = W.custom(name, lens, hq, hkv, d, causal, seed)
    q, k, v, _, cu = W.make_inputs(w, with_grad=False)
    return w, q, k, v, cu


@pytest.mark.parametrize("case", VARLEN_CASES, ids=[c[0] for c in VARLEN_CASES])
def test_fp8_quantize_varlen_bit_exact(case):
    """Packed sequences: Q8 / K8 / descales as for a fixed-length batch; V^T per (sequence,
    kv head) with the longest sequence's pitch and each shorter sequence zero-padded."""
    w, q, k, v, cu = fp8_varlen_case(case)
    dev = torch.device("cuda")
    q8, k8, vt8, dq, dk, dv = attn.attn_fp8_quantize(q.to(dev), k.to(dev), v.to(dev), cu_seqlens=cu.to(dev),
                                                     max_seqlen=w.max_seqlen)
    attn.attn_get_device_error()
    q8_ref, dq_ref = quantize_cpu(q, w.hq)
    k8_ref, dk_ref = quantize_cpu(k, w.hkv)
    v8_ref, dv_ref = quantize_cpu(v, w.hkv)
    assert torch.equal(dq.cpu(), dq_ref) and torch.equal(dk.cpu(), dk_ref) and torch.equal(dv.cpu(), dv_ref)
    assert torch.equal(q8.cpu(), q8_ref) and torch.equal(k8.cpu(), k8_ref)
    assert tuple(vt8.shape) == (w.batch * w.hkv, w.d, pitch_of(w.max_seqlen))
    assert torch.equal(vt8.cpu(), transpose_v_cpu_varlen(v8_ref, cu.tolist(), w.max_seqlen))


@pytest.mark.parametrize("case", VARLEN_CASES, ids=[c[0] for c in VARLEN_CASES])
def test_fp8_forward_varlen_matches_oracle(case):
    """The FP8 forward over packed sequences, on operands quantised here on the CPU."""
    w, q, k, v, cu = fp8_varlen_case(case)
    q8, dq = quantize_cpu(q, w.hq)
    k8, dk = quantize_cpu(k, w.hkv)
    v8, dv = quantize_cpu(v, w.hkv)
    vt8 = transpose_v_cpu_varlen(v8, cu.tolist(), w.max_seqlen)
    dev = torch.device("cuda")
    o, lse = attn.attn_fwd_fp8(q8.to(dev), k8.to(dev), vt8.to(dev), dq.to(dev), dk.to(dev), dv.to(dev),
                               cu_seqlens=cu.to(dev), max_seqlen=w.max_seqlen, scale=w.scale, causal=w.causal)
    attn.attn_get_device_error()
    o, lse = parity.to_np(o), parity.to_np(lse)
    qd, kd, vd = dequant(q8, dq).numpy(), dequant(k8, dk).numpy(), dequant(v8, dv).numpy()
    o_ref, lse_ref = oracle.attn_fwd_fp8sim(qd, kd, vd, cu.numpy(), scale=w.scale, causal=w.causal)
    parity.check_fwd_bf16(o, lse, o_ref, lse_ref, tag=w.name)
    o_ex, _ = oracle.attn_fwd(qd, kd, vd, cu.numpy(), scale=w.scale, causal=w.causal)
    assert parity.rel_l2(o, o_ex) <= FP8_EXACT_REL_L2, w.name


def test_fp8_varlen_end_to_end_through_quantize():
    """attn_fp8_quantize then attn_fwd_fp8 on packed sequences, both on the device."""
    w, q, k, v, cu = fp8_varlen_case(("fp8-varlen-e2e", [384, 1000, 5, 640], 4, 2, True, 56, 128))
    dev = torch.device("cuda")
    cu_d = cu.to(dev)
    ops = attn.attn_fp8_quantize(q.to(dev), k.to(dev), v.to(dev), cu_seqlens=cu_d, max_seqlen=w.max_seqlen)
    o, lse = attn.attn_fwd_fp8(*ops, cu_seqlens=cu_d, max_seqlen=w.max_seqlen, scale=w.scale, causal=True)
    attn.attn_get_device_error()
    q8, dq = quantize_cpu(q, w.hq)
    k8, dk = quantize_cpu(k, w.hkv)
    v8, dv = quantize_cpu(v, w.hkv)
    o_ref, lse_ref = oracle.attn_fwd_fp8sim(dequant(q8, dq).numpy(), dequant(k8, dk).numpy(),
                                            dequant(v8, dv).numpy(), cu.numpy(), scale=w.scale, causal=True)
    parity.check_fwd_bf16(parity.to_np(o), parity.to_np(lse), o_ref, lse_ref, tag=w.name)


def test_fp8_varlen_sequence_longer_than_max_seqlen_is_reported():
    """As for the bf16 forward: a max_seqlen below the longest sequence is reported through
    attn_get_device_error, not silently truncated."""
    w, q, k, v, cu = fp8_varlen_case(("fp8-varlen-short", [100, 700, 300], 4, 2, True, 57, 128))
    dev = torch.device("cuda")
    cu_d = cu.to(dev)
    ops = attn.attn_fp8_quantize(q.to(dev), k.to(dev), v.to(dev), cu_seqlens=cu_d, max_seqlen=512)
    attn.attn_fwd_fp8(*ops, cu_seqlens=cu_d, max_seqlen=512, scale=w.scale, causal=True)
    with pytest.raises(attn.AttnError) as e:
        attn.attn_get_device_error()
    assert e.value.status == attn.ATTN_ERR_INVALID_ARG
