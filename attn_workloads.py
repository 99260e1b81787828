"""Seeded synthetic workloads for exact attention.

This module only draws inputs and describes shapes; it holds none of the attention
arithmetic.  Both the fp64 CPU oracle and the CUDA library are fed from it, so the two
sides always see the same bf16 (or fp32) tensors.

Recipe: every tensor (Q, K, V and the upstream gradient dO) is i.i.d. N(0, 1), drawn in
fp32 on the CPU from ``torch.Generator().manual_seed(seed)`` in the order
(lengths, Q, K, V, dO), then rounded to bf16 (round-to-nearest-even) unless fp32 is
asked for.  The stability variant multiplies Q and K by 30 before the rounding.  Variable
lengths are ``torch.randint(64, 4097, (16,))`` from the same generator.

Workloads (the validation checklist of the "FlashAttention 与高效注意力内核" tutorial asks
for causal masks, max-value stability and packed variable-length sequences; the
"相关工作" page asks for head dims 32/64/128 and grouped K/V heads):

  small     B=1,  H=2,  N=256,   d=64,  scale 1/8
  mha2k     B=4,  H=16, N=2048,  d=128
  sweep     d in {32,64,128}, H=2048/d, N in {512..16384}, B=16384/N  (16k tokens)
  gqa8k     B=2,  Hq=32, Hkv=8, N=8192, d=128, causal   (+ x30 stability variant)
  varlen16  16 sequences, lengths U{64..4096}, H=16, d=128, causal
  long32k   B=1,  H=16, N=32768, d=128, causal

Decoding-shaped workloads (the tutorial's FlashDecoding case, "one query against a long
KV"): sequence b has Lq_b query rows (the newest tokens) and Lk_b cached keys; Q is
[sum Lq, Hq, d], K and V are [sum Lk, Hkv, d], drawn in the order (lengths, Q, K, V):

  decode8k      16 sequences, Lq=1, Lk=8192,          Hq=32, Hkv=8, d=128
  decode_var    16 sequences, Lq=1, Lk ~ U{64..32768}, Hq=32, Hkv=8, d=128
  decode_spec4  16 sequences, Lq=4 (causal), Lk=4096,  Hq=32, Hkv=8, d=128
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int              # number of sequences
    seqlen: int             # per-sequence length in batch mode (0 for varlen)
    hq: int
    hkv: int
    d: int
    causal: bool
    seed: int
    lengths: Optional[tuple] = None   # varlen: per-sequence lengths
    qk_mult: float = 1.0              # stability variant: Q and K multiplied before rounding
    scale_arg: Optional[float] = None   # the score scale if not 1/sqrt(d)

    @property
    def scale(self) -> float:
        return self.scale_arg if self.scale_arg is not None else 1.0 / math.sqrt(self.d)

    @property
    def seqlens(self) -> List[int]:
        return list(self.lengths) if self.lengths is not None else [self.seqlen] * self.batch

    @property
    def total_tokens(self) -> int:
        return sum(self.seqlens)

    @property
    def max_seqlen(self) -> int:
        return max(self.seqlens) if self.seqlens else 0

    @property
    def varlen(self) -> bool:
        return self.lengths is not None

    def cu_seqlens(self) -> torch.Tensor:
        cu = [0]
        for n in self.seqlens:
            cu.append(cu[-1] + n)
        return torch.tensor(cu, dtype=torch.int32)

    def fwd_flops(self) -> float:
        """4 * H * N^2 * d per sequence, halved for causal."""
        f = sum(4.0 * self.hq * n * n * self.d for n in self.seqlens)
        return f / 2 if self.causal else f

    def bwd_flops(self) -> float:
        return 2.5 * self.fwd_flops()

    def with_causal(self, causal: bool) -> "Workload":
        return dataclasses.replace(self, causal=causal, name=self.name.split("+")[0] + ("+causal" if causal else ""))


def _varlen_lengths(seed: int, count: int = 16, lo: int = 64, hi: int = 4096) -> tuple:
    g = torch.Generator().manual_seed(seed)
    return tuple(int(x) for x in torch.randint(lo, hi + 1, (count,), generator=g))


def small(causal=False) -> Workload:
    return Workload("small", 1, 256, 2, 2, 64, causal, seed=1001)


def mha2k(causal=False) -> Workload:
    return Workload("mha2k" + ("+causal" if causal else ""), 4, 2048, 16, 16, 128, causal, seed=1002)


def sweep(d: int, n: int, causal=False) -> Workload:
    h = 2048 // d
    return Workload(f"sweep_d{d}_n{n}" + ("+causal" if causal else ""), 16384 // n, n, h, h, d,
                    causal, seed=1003)


SWEEP_D = (32, 64, 128)
SWEEP_N = (512, 1024, 2048, 4096, 8192, 16384)


def gqa8k(stability=False) -> Workload:
    return Workload("gqa8k_x30" if stability else "gqa8k", 2, 8192, 32, 8, 128, True, seed=1004,
                    qk_mult=30.0 if stability else 1.0)


def varlen16() -> Workload:
    return Workload("varlen16", 16, 0, 16, 16, 128, True, seed=1005, lengths=_varlen_lengths(1005))


def long32k() -> Workload:
    return Workload("long32k", 1, 32768, 16, 16, 128, True, seed=1006)


def custom(name, seqlens, hq, hkv, d, causal, seed, qk_mult=1.0, scale=None) -> Workload:
    """Any other shape (tests use this for ragged and edge cases, and for a score scale
    other than 1/sqrt(d))."""
    seqlens = tuple(int(n) for n in seqlens)
    return Workload(name, len(seqlens), 0, hq, hkv, d, causal, seed, lengths=seqlens, qk_mult=qk_mult,
                    scale_arg=scale)


def make_inputs(w: Workload, dtype: torch.dtype = torch.bfloat16, with_grad: bool = True):
    """Seeded CPU tensors q [T,Hq,d], k, v [T,Hkv,d], do [T,Hq,d] and cu_seqlens int32."""
    g = torch.Generator().manual_seed(w.seed)
    if w.varlen:
        _ = _varlen_lengths(w.seed)  # the lengths come first from the same stream
        g = torch.Generator().manual_seed(w.seed)
        torch.randint(64, 4097, (len(w.lengths),), generator=g)
    T = w.total_tokens
    q = torch.randn(T, w.hq, w.d, generator=g, dtype=torch.float32)
    k = torch.randn(T, w.hkv, w.d, generator=g, dtype=torch.float32)
    v = torch.randn(T, w.hkv, w.d, generator=g, dtype=torch.float32)
    do = torch.randn(T, w.hq, w.d, generator=g, dtype=torch.float32) if with_grad else None
    if w.qk_mult != 1.0:
        q = q * w.qk_mult
        k = k * w.qk_mult
    if dtype != torch.float32:
        q, k, v = q.to(dtype), k.to(dtype), v.to(dtype)
        do = do.to(dtype) if do is not None else None
    return q, k, v, do, w.cu_seqlens()


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    name: str
    q_lens: tuple           # query rows per sequence (the newest positions)
    k_lens: tuple           # keys per sequence
    hq: int
    hkv: int
    d: int
    causal: bool
    seed: int
    random_k: Optional[tuple] = None   # (lo, hi): k_lens drawn from the seed stream first
    scale_arg: Optional[float] = None   # the score scale if not 1/sqrt(d)

    @property
    def scale(self) -> float:
        return self.scale_arg if self.scale_arg is not None else 1.0 / math.sqrt(self.d)

    @property
    def batch(self) -> int:
        return len(self.k_lens)

    @property
    def total_q(self) -> int:
        return sum(self.q_lens)

    @property
    def total_k(self) -> int:
        return sum(self.k_lens)

    @property
    def max_k(self) -> int:
        return max(self.k_lens) if self.k_lens else 0

    def cu_q(self) -> torch.Tensor:
        return torch.tensor([0] + [sum(self.q_lens[:i + 1]) for i in range(len(self.q_lens))], dtype=torch.int32)

    def cu_k(self) -> torch.Tensor:
        return torch.tensor([0] + [sum(self.k_lens[:i + 1]) for i in range(len(self.k_lens))], dtype=torch.int32)

    def kv_bytes(self) -> int:
        """Bytes of K and V (bf16) that any exact decode must read once."""
        return 2 * self.total_k * self.hkv * self.d * 2

    def hbm_bytes(self) -> int:
        """Algorithmic HBM traffic: K, V read, Q read, O written (bf16), LSE written (fp32)."""
        return self.kv_bytes() + 2 * self.total_q * self.hq * self.d * 2 + 4 * self.total_q * self.hq


def _decode_lengths(seed: int, count: int, lo: int, hi: int) -> tuple:
    g = torch.Generator().manual_seed(seed)
    return tuple(int(x) for x in torch.randint(lo, hi + 1, (count,), generator=g))


def decode8k() -> DecodeWorkload:
    return DecodeWorkload("decode8k", (1,) * 16, (8192,) * 16, 32, 8, 128, False, seed=1101)


def decode_var() -> DecodeWorkload:
    return DecodeWorkload("decode_var", (1,) * 16, _decode_lengths(1102, 16, 64, 32768), 32, 8, 128, False,
                          seed=1102, random_k=(64, 32768))


def decode_spec4() -> DecodeWorkload:
    return DecodeWorkload("decode_spec4", (4,) * 16, (4096,) * 16, 32, 8, 128, True, seed=1103)


def decode_custom(name, q_lens, k_lens, hq, hkv, d, causal, seed, scale=None) -> DecodeWorkload:
    return DecodeWorkload(name, tuple(int(x) for x in q_lens), tuple(int(x) for x in k_lens), hq, hkv, d, causal, seed,
                          scale_arg=scale)


def make_decode_inputs(w: DecodeWorkload, dtype: torch.dtype = torch.bfloat16):
    """Seeded CPU tensors q [sum Lq,Hq,d], k, v [sum Lk,Hkv,d], cu_q, cu_k (int32)."""
    g = torch.Generator().manual_seed(w.seed)
    if w.random_k is not None:
        torch.randint(w.random_k[0], w.random_k[1] + 1, (len(w.k_lens),), generator=g)   # the lengths came first
    q = torch.randn(w.total_q, w.hq, w.d, generator=g, dtype=torch.float32)
    k = torch.randn(w.total_k, w.hkv, w.d, generator=g, dtype=torch.float32)
    v = torch.randn(w.total_k, w.hkv, w.d, generator=g, dtype=torch.float32)
    if dtype != torch.float32:
        q, k, v = q.to(dtype), k.to(dtype), v.to(dtype)
    return q, k, v, w.cu_q(), w.cu_k()
