"""Seeded synthetic workloads for the measured shapes.

This module only draws random numbers: it holds none of the method's
arithmetic (no rotation, no softmax, no scoring).  Tests, the benchmark and
the smoke check use it to give the CUDA library and the CPU oracle the very
same inputs.

Recipe: one ``torch.Generator`` per workload, seeded with ``20260000 + index``
(index = position of the workload in the list below, the tiny case first).
Values are fp32 N(0, 1) rounded to bf16 (round-to-nearest-even, torch's
conversion); indexer head weights are fp32 U(0, 1); ragged cache lengths are
``randint(lo, hi + 1)`` drawn from a CPU generator so that they do not depend
on the device the tensors are drawn on.  Cache rows past a sequence's length
are filled with random values too (the kernels must ignore them).
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field

import torch

SEED_BASE = 20260000

# RoPE frequency-scaling modes, numbered as in the C header.
ROPE_NONE, ROPE_PI, ROPE_NTK, ROPE_YARN, ROPE_DYN_NTK = 0, 1, 2, 3, 4


@dataclass(frozen=True)
class RopeSpec:
    base: float = 10000.0
    scaling: int = ROPE_NONE
    s: float = 1.0
    L_train: float = 0.0
    alpha: float = 1.0
    beta: float = 32.0
    L_cur: float = 0.0
    pair_style: int = 0  # 0: adjacent pairs (2i, 2i+1); 1: half-split (i, i + d/2)


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    index: int
    B: int
    H: int
    Hk: int
    d: int
    T_max: int
    T_lo: int  # lengths drawn uniformly in [T_lo, T_hi]; T_lo == T_hi means fixed
    T_hi: int
    rope: RopeSpec = field(default_factory=RopeSpec)

    @property
    def g(self) -> int:
        return self.H // self.Hk

    @property
    def scale(self) -> float:
        return self.d ** -0.5


@dataclass(frozen=True)
class PrefillWorkload:
    name: str
    index: int
    B: int
    T: int
    H: int
    Hk: int
    d: int
    rope: RopeSpec = field(default_factory=RopeSpec)

    @property
    def scale(self) -> float:
        return self.d ** -0.5


@dataclass(frozen=True)
class DsaWorkload:
    name: str
    index: int
    B: int
    L: int
    HI: int  # indexer heads
    dI: int  # indexer key/query width
    k: int  # rows kept per query
    Hq: int  # attention heads
    Dk: int  # latent row width (keys)
    Dv: int  # value width (first Dv columns of a latent row)
    sparse_scale: float = 192 ** -0.5  # 1/sqrt(d_h + d_h^R) with d_h = 128, d_h^R = 64


@dataclass(frozen=True)
class QsaWorkload:
    """Block-level indexer over 4-token groups, then sparse GQA decode."""
    name: str
    index: int
    B: int
    L: int        # cache capacity (tokens); lengths are drawn in [L_lo, L]
    L_lo: int
    HI: int       # indexer heads
    dI: int       # indexer key/query width
    n_top: int    # groups kept
    H: int        # attention heads
    Hk: int       # KV heads
    d: int        # head width
    rope: RopeSpec = field(default_factory=lambda: RopeSpec(base=500000.0))

    @property
    def scale(self) -> float:
        return self.d ** -0.5


TINY_GQA = DecodeWorkload("tiny_gqa_decode_B2_H8_Hk2_d64_T256", 0, B=2, H=8, Hk=2, d=64, T_max=256,
                          T_lo=256, T_hi=256, rope=RopeSpec(base=10000.0))
LLAMA3_8B_DECODE = DecodeWorkload("llama3_8b_decode_B16_H32_Hk8_d128_ragged1024-8192", 1, B=16, H=32,
                                  Hk=8, d=128, T_max=8192, T_lo=1024, T_hi=8192,
                                  rope=RopeSpec(base=500000.0))
_YARN4 = RopeSpec(base=10000.0, scaling=ROPE_YARN, s=4.0, L_train=8192.0, alpha=1.0, beta=32.0)
LLAMA2_70B_GQA_32K = DecodeWorkload("llama2_70b_decode_gqa_B16_H64_Hk8_d128_T32768_yarn4", 2, B=16,
                                    H=64, Hk=8, d=128, T_max=32768, T_lo=32768, T_hi=32768,
                                    rope=_YARN4)
LLAMA2_70B_MQA_32K = dataclasses.replace(LLAMA2_70B_GQA_32K,
                                         name="llama2_70b_decode_mqa_B16_H64_Hk1_d128_T32768_yarn4",
                                         Hk=1)
LLAMA2_70B_MHA_32K = dataclasses.replace(LLAMA2_70B_GQA_32K,
                                         name="llama2_70b_decode_mha_B4_H64_Hk64_d128_T32768_yarn4",
                                         B=4, Hk=64)
PREFILL_8K = PrefillWorkload("causal_prefill_B2_T8192_H32_Hk8_d128", 3, B=2, T=8192, H=32, Hk=8,
                             d=128, rope=RopeSpec(base=500000.0))
DSA_128K = DsaWorkload("dsa_sparse_decode_B8_L131072_HI64_dI128_k2048_Hq128_576-512", 4, B=8,
                       L=131072, HI=64, dI=128, k=2048, Hq=128, Dk=576, Dv=512)

QSA_128K = QsaWorkload("qsa_block_sparse_decode_B8_L131072_HI64_dI128_top512x4_H32_Hk8_d128", 5, B=8, L=131072,
                       L_lo=65536, HI=64, dI=128, n_top=512, H=32, Hk=8, d=128)

DECODE_WORKLOADS = [TINY_GQA, LLAMA3_8B_DECODE, LLAMA2_70B_GQA_32K, LLAMA2_70B_MQA_32K,
                    LLAMA2_70B_MHA_32K]


def generator(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal_bf16(shape, gen: torch.Generator, device="cpu") -> torch.Tensor:
    """fp32 N(0,1) draws rounded to bf16 (nearest-even)."""
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)


def uniform_f32(shape, gen: torch.Generator, device="cpu") -> torch.Tensor:
    return torch.rand(shape, generator=gen, device=device, dtype=torch.float32)


def lengths(B: int, lo: int, hi: int, seed: int) -> torch.Tensor:
    """Cache lengths: fixed when lo == hi, else uniform integers in [lo, hi]."""
    if lo == hi:
        return torch.full((B,), lo, dtype=torch.int32)
    g = generator(seed + 7_777)
    return torch.randint(lo, hi + 1, (B,), generator=g, dtype=torch.int64).to(torch.int32)


def decode_inputs(w: DecodeWorkload, device="cpu", seed: int | None = None, B: int | None = None,
                  T_max: int | None = None, lens: torch.Tensor | None = None) -> dict:
    """Raw (pre-RoPE) decode inputs.

    q [B, H, d] -- the new token's query, at position seq_lens[b];
    k, v [B, Hk, T_max, d] -- cache rows, row t at position t;
    seq_lens int32 [B]; k_pos int32 [B, T_max] (= t); q_pos int32 [B, 1].
    ``B``/``T_max`` shrink the workload for oracle-sized tests.
    """
    seed = SEED_BASE + w.index if seed is None else seed
    B = w.B if B is None else B
    T_max = w.T_max if T_max is None else T_max
    if lens is None:
        lens = lengths(B, min(w.T_lo, T_max), min(w.T_hi, T_max), seed)
    gen = generator(seed, device)
    q = normal_bf16((B, w.H, w.d), gen, device)
    k = normal_bf16((B, w.Hk, T_max, w.d), gen, device)
    v = normal_bf16((B, w.Hk, T_max, w.d), gen, device)
    k_pos = torch.arange(T_max, dtype=torch.int32).repeat(B, 1)
    q_pos = lens.clone().reshape(B, 1)
    return dict(q=q, k=k, v=v, seq_lens=lens.to(torch.int32), k_pos=k_pos, q_pos=q_pos)


def prefill_inputs(w: PrefillWorkload, device="cpu", seed: int | None = None, B: int | None = None,
                   T: int | None = None) -> dict:
    """q [B, T, H, d]; k, v [B, Hk, T, d]; positions 0 .. T-1 for every batch."""
    seed = SEED_BASE + w.index if seed is None else seed
    B = w.B if B is None else B
    T = w.T if T is None else T
    gen = generator(seed, device)
    q = normal_bf16((B, T, w.H, w.d), gen, device)
    k = normal_bf16((B, w.Hk, T, w.d), gen, device)
    v = normal_bf16((B, w.Hk, T, w.d), gen, device)
    pos = torch.arange(T, dtype=torch.int32).repeat(B, 1)
    return dict(q=q, k=k, v=v, pos=pos)


def dsa_inputs(w: DsaWorkload, device="cpu", seed: int | None = None, B: int | None = None,
               L: int | None = None, with_latent: bool = True) -> dict:
    """q_idx [B, HI, dI] bf16, w [B, HI] fp32 U(0,1), k_idx [B, L, dI] bf16,
    q [B, Hq, Dk] bf16, latent [B, L, Dk] bf16, seq_lens int32 [B] (= L)."""
    seed = SEED_BASE + w.index if seed is None else seed
    B = w.B if B is None else B
    L = w.L if L is None else L
    gen = generator(seed, device)
    out = dict(q_idx=normal_bf16((B, w.HI, w.dI), gen, device),
               w=uniform_f32((B, w.HI), gen, device),
               k_idx=normal_bf16((B, L, w.dI), gen, device))
    if with_latent:
        out["q"] = normal_bf16((B, w.Hq, w.Dk), gen, device)
        out["latent"] = normal_bf16((B, L, w.Dk), gen, device)
    out["seq_lens"] = torch.full((B,), L, dtype=torch.int32)
    return out


def qsa_inputs(w: QsaWorkload, device="cpu", seed: int | None = None, B: int | None = None,
               L: int | None = None, L_lo: int | None = None, with_cache: bool = True) -> dict:
    """q_idx [B, HI, dI] bf16, w [B, HI] fp32 U(0,1), k_idx [B, L, dI] bf16 (the
    indexer keys), q [B, H, d], k/v [B, Hk, L, d] bf16, seq_lens int32 [B] drawn
    uniformly in [L_lo, L] (every residue mod 4 occurs: the trailing partial group)."""
    seed = SEED_BASE + w.index if seed is None else seed
    B = w.B if B is None else B
    if L_lo is None:
        L_lo = w.L_lo if L is None else L // 2
    L = w.L if L is None else L
    gen = generator(seed, device)
    out = dict(q_idx=normal_bf16((B, w.HI, w.dI), gen, device),
               w=uniform_f32((B, w.HI), gen, device),
               k_idx=normal_bf16((B, L, w.dI), gen, device))
    if with_cache:
        out["q"] = normal_bf16((B, w.H, w.d), gen, device)
        out["k"] = normal_bf16((B, w.Hk, L, w.d), gen, device)
        out["v"] = normal_bf16((B, w.Hk, L, w.d), gen, device)
    out["seq_lens"] = lengths(B, L_lo, L, seed)
    return out


def bf16_bits(t: torch.Tensor):
    """numpy uint16 view of a bf16 tensor's bit patterns (copied to host)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")
