"""Seeded synthetic workloads: shapes, distributions and input generation.

This module holds no attention arithmetic; it only draws inputs.  Both the CUDA
path's tests/bench and the fp64 oracle's tests take their inputs from here.

Each workload draws Q, K, V and dO, in that order, as float32 normals from
``torch.Generator('cpu').manual_seed(seed)``, multiplies Q and K by ``qk_std``,
and rounds all four to bf16.  The oracle receives the same bf16 values upcast
exactly to float64.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    causal: bool
    qk_std: float = 1.0
    seed: int = 1000

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def fwd_flops(self) -> float:
        """4·B·Hq·N²·d, halved when causal."""
        f = 4.0 * self.B * self.Hq * self.N * self.N * self.d
        return f / 2 if self.causal else f

    def bwd_flops(self) -> float:
        return 2.5 * self.fwd_flops()

    def describe(self) -> str:
        return (f"B={self.B} Hq={self.Hq} Hkv={self.Hkv} N={self.N} d={self.d} "
                f"{'causal' if self.causal else 'non-causal'} qk_std={self.qk_std:g}")


# The five reference workloads (seed = 1000 + index); C2 runs both causal and
# non-causal.  The benchmark workload is the long causal sequence (N = 16384,
# d = 128), the largest d = 128 problem.
WORKLOADS = {
    "tiny_b1_h2_n128_d64": Workload("tiny_b1_h2_n128_d64", 1, 2, 2, 128, 64, False, 1.0, 1000),
    "train_b8_h16_n2048_d128": Workload("train_b8_h16_n2048_d128", 8, 16, 16, 2048, 128, False, 1.0, 1001),
    "train_b8_h16_n2048_d128_causal": Workload("train_b8_h16_n2048_d128_causal", 8, 16, 16, 2048, 128, True, 1.0, 1001),
    "long_b1_h16_n16384_d128_causal": Workload("long_b1_h16_n16384_d128_causal", 1, 16, 16, 16384, 128, True, 1.0, 1002),
    "gqa_b4_hq32_hkv8_n4096_d128_causal": Workload("gqa_b4_hq32_hkv8_n4096_d128_causal", 4, 32, 8, 4096, 128, True, 1.0, 1003),
    "wide_b2_h8_n8192_d256_bigqk": Workload("wide_b2_h8_n8192_d256_bigqk", 2, 8, 8, 8192, 256, False, 3.0, 1004),
    # head dimension 64: one exponential per 64 multiply-adds instead of 128,
    # the regime where the exponentials rather than the tensor cores bound
    # the forward pass
    "train_b8_h16_n2048_d64": Workload("train_b8_h16_n2048_d64", 8, 16, 16, 2048, 64, False, 1.0, 1005),
    # N not a multiple of 128: the last query and key tiles of every head are
    # partial
    "ragged_b8_h16_n2000_d128_causal": Workload("ragged_b8_h16_n2000_d128_causal", 8, 16, 16, 2000, 128, True, 1.0,
                                                1006),
}

BENCH_WORKLOAD = "long_b1_h16_n16384_d128_causal"


@dataclass(frozen=True)
class DecodeWorkload:
    """Nq query rows per head (the last Nq positions of the sequence) against
    Nk cached keys and values."""
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    d: int
    causal: bool
    seed: int

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def visible_pairs(self) -> int:
        """(query, key) pairs per head that the mask leaves visible."""
        if not self.causal:
            return self.Nq * self.Nk
        return sum(self.Nk - self.Nq + i + 1 for i in range(self.Nq))

    def fwd_flops(self) -> float:
        """4·d FLOPs per visible (query, key) pair and query head."""
        return 4.0 * self.B * self.Hq * self.d * self.visible_pairs()

    def hbm_bytes(self) -> int:
        """Bytes one call must move: K and V once, Q in, O and LSE out."""
        kv = 2 * self.B * self.Hkv * self.Nk * self.d * 2
        qo = 2 * self.B * self.Hq * self.Nq * self.d * 2
        return kv + qo + self.B * self.Hq * self.Nq * 4

    def describe(self) -> str:
        return (f"B={self.B} Hq={self.Hq} Hkv={self.Hkv} Nq={self.Nq} Nk={self.Nk} d={self.d} "
                f"{'causal' if self.causal else 'non-causal'}")


DECODE_WORKLOADS = {
    # one decoding step of a batch of 8 sequences with a 32k-token cache, GQA 4:1
    "decode_b8_hq32_hkv8_nk32768_d128": DecodeWorkload("decode_b8_hq32_hkv8_nk32768_d128", 8, 32, 8, 1, 32768, 128,
                                                      True, 1007),
    # 32 queries per head (a speculative or chunked decoding step): 128 query
    # rows per kv head share every K/V tile
    "decode_b8_hq32_hkv8_nq32_nk32768_d128": DecodeWorkload("decode_b8_hq32_hkv8_nq32_nk32768_d128", 8, 32, 8, 32,
                                                           32768, 128, True, 1008),
}


def make_decode_inputs(w: DecodeWorkload, device="cpu", seed: int | None = None):
    """Draw (q, k, v) as bf16 tensors [B,Hq,Nq,d], [B,Hkv,Nk,d], [B,Hkv,Nk,d]
    (standard normals, in that order) from the workload's seed."""
    g = torch.Generator("cpu").manual_seed(w.seed if seed is None else seed)
    q = torch.randn(w.B, w.Hq, w.Nq, w.d, generator=g, dtype=torch.float32)
    k = torch.randn(w.B, w.Hkv, w.Nk, w.d, generator=g, dtype=torch.float32)
    v = torch.randn(w.B, w.Hkv, w.Nk, w.d, generator=g, dtype=torch.float32)
    return tuple(t.to(torch.bfloat16).to(device) for t in (q, k, v))


def make_inputs(w: Workload, device="cpu", seed: int | None = None):
    """Draw (q, k, v, do) as bf16 tensors with shapes [B,Hq,N,d], [B,Hkv,N,d],
    [B,Hkv,N,d], [B,Hq,N,d] from the workload's seed, then move them to
    ``device``."""
    g = torch.Generator("cpu").manual_seed(w.seed if seed is None else seed)
    q = torch.randn(w.B, w.Hq, w.N, w.d, generator=g, dtype=torch.float32)
    k = torch.randn(w.B, w.Hkv, w.N, w.d, generator=g, dtype=torch.float32)
    v = torch.randn(w.B, w.Hkv, w.N, w.d, generator=g, dtype=torch.float32)
    do = torch.randn(w.B, w.Hq, w.N, w.d, generator=g, dtype=torch.float32)
    if w.qk_std != 1.0:
        q.mul_(w.qk_std)
        k.mul_(w.qk_std)
    out = [t.to(torch.bfloat16) for t in (q, k, v, do)]
    return tuple(t.to(device) for t in out)


def shard_units(B: int, Hkv: int, rank: int, world: int):
    """Split the independent (batch, kv-head) units of a workload across
    ``world`` ranks: contiguous blocks of the flattened B·Hkv index, the first
    ``B·Hkv % world`` ranks taking one extra.  Query heads travel with their
    kv head, so no rank needs another rank's data."""
    total = B * Hkv
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    count = base + (1 if rank < extra else 0)
    return [(u // Hkv, u % Hkv) for u in range(start, start + count)]


@dataclass(frozen=True)
class VarlenWorkload:
    """A packed batch of sequences with the given lengths (sequences back to
    back along the token axis of [H, T, d] tensors)."""
    name: str
    lengths: tuple
    Hq: int
    Hkv: int
    d: int
    causal: bool
    seed: int
    qk_std: float = 1.0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def T(self) -> int:
        return int(sum(self.lengths))

    @property
    def max_seqlen(self) -> int:
        return max(1, max(self.lengths))

    def cu_seqlens(self):
        out = [0]
        for n in self.lengths:
            out.append(out[-1] + int(n))
        return out

    def fwd_flops(self) -> float:
        """4·d FLOPs per visible (query, key) pair and query head (the fixed-
        length count, summed over the sequences)."""
        pairs = sum((n * (n + 1)) // 2 if self.causal else n * n for n in self.lengths)
        return 4.0 * self.Hq * self.d * pairs

    def describe(self) -> str:
        return (f"{len(self.lengths)} sequences, T={self.T}, max len {self.max_seqlen}, Hq={self.Hq} "
                f"Hkv={self.Hkv} d={self.d} {'causal' if self.causal else 'non-causal'}")


def varlen_lengths(nseq: int, lo: int, hi: int, seed: int, include=()):
    """nseq sequence lengths drawn uniformly from [lo, hi] (seeded), with the
    values in ``include`` placed first."""
    g = torch.Generator("cpu").manual_seed(seed)
    extra = torch.randint(lo, hi + 1, (max(0, nseq - len(include)),), generator=g).tolist()
    return tuple(list(include) + extra)


def make_varlen_inputs(w: VarlenWorkload, device="cpu"):
    """Draw (q, k, v, do, cu_seqlens): q, do bf16 [Hq, T, d], k, v bf16
    [Hkv, T, d] (standard normals in the order q, k, v, do; q and k times
    qk_std) and cu_seqlens int32 [nseq + 1]."""
    g = torch.Generator("cpu").manual_seed(w.seed)
    T = w.T
    q = torch.randn(w.Hq, T, w.d, generator=g, dtype=torch.float32)
    k = torch.randn(w.Hkv, T, w.d, generator=g, dtype=torch.float32)
    v = torch.randn(w.Hkv, T, w.d, generator=g, dtype=torch.float32)
    do = torch.randn(w.Hq, T, w.d, generator=g, dtype=torch.float32)
    if w.qk_std != 1.0:
        q.mul_(w.qk_std)
        k.mul_(w.qk_std)
    out = [t.to(torch.bfloat16).to(device) for t in (q, k, v, do)]
    cu = torch.tensor(w.cu_seqlens(), dtype=torch.int32, device=device)
    return (*out, cu)


# A packed batch for the benchmark: 16 causal sequences of 256 .. 4096 tokens
# (seeded), 16 heads, d = 128 -- a training batch of documents of mixed length.
VARLEN_WORKLOADS = {
    "varlen_16seq_256to4096_h16_d128_causal": VarlenWorkload(
        "varlen_16seq_256to4096_h16_d128_causal", varlen_lengths(16, 256, 4096, 1009), 16, 16, 128, True, 1009),
}
