"""Seeded synthetic workloads (shared by the tests, the benchmark and the CPU oracle).

This module holds none of the method's arithmetic: it only draws random fp16 inputs of
the shapes and value distributions of the method's target workloads (LLM prefill,
video-DiT attention with channel outliers in K, long-sequence sweeps, packed varlen).

Recipe (all draws on the CPU from ``torch.Generator().manual_seed(seed)``, in this order):

1. (varlen only) the sequence lengths, ``randint(lo, hi + 1)`` each;
2. Q, K, V as fp32 standard normals in the layout's shape (Q with its own length when
   the queries are fewer than the keys);
3. the K channel offset: one length-d vector added to every token of every head. With
   ``offset_channels = c`` only c channels (``randperm(d)[:c]``) get an offset, drawn
   after the permutation. ``N(0, s^2)`` is read as variance s^2 (std s);
4. cast to fp16 (round to nearest even).

The channel offset reproduces the outlier structure that motivates smoothing K: a
shared per-channel bias across all tokens.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional, Tuple

import torch

SWEEP_N = (1024, 2048, 4096, 8192, 16384, 32768)


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    B: int
    H: int
    N: int
    d: int
    causal: bool
    offset_std: float
    offset_channels: Optional[int] = None
    pv_modes: Tuple[str, ...] = ("fp16",)
    nseq: int = 0                  # > 0: packed varlen with nseq sequences
    len_lo: int = 512
    len_hi: int = 16384
    nq: int = 0                    # > 0: queries per sequence when fewer than the N keys


def tiny() -> Workload:
    return Workload("tiny B1 H2 N256 d64 non-causal", 1000, 1, 2, 256, 64, False, 2.0)


def llm_prefill() -> Workload:
    return Workload("LLM causal prefill B4 H32 N4096 d128", 1001, 4, 32, 4096, 128, True, 1.0)


def video_dit() -> Workload:
    return Workload("video-DiT B1 H30 N17550 d64 non-causal", 1002, 1, 30, 17550, 64, False, 3.0,
                    offset_channels=4, pv_modes=("fp16", "fp8"))


def sweep(N: int, d: int, causal: bool) -> Workload:
    B = max(1, 32768 // N)
    return Workload(f"sweep B{B} H32 N{N} d{d} {'causal' if causal else 'non-causal'}", 1003,
                    B, 32, N, d, causal, 1.0)


def prefill_kv() -> Workload:
    """The last 2048 tokens of 8192-token sequences attending to all their keys (chunked
    prefill against cached keys), causal."""
    return Workload("LLM chunked prefill B2 H32 Nq2048 Nk8192 d128 causal", 1005, 2, 32, 8192,
                    128, True, 1.0, nq=2048)


def decode() -> Workload:
    """One decode step: one new query per sequence attending to 32768 cached keys, B=8 H=32
    d=128 (causal, which for the last position is every key)."""
    return Workload("LLM decode B8 H32 Nq1 Nk32768 d128 causal", 1006, 8, 32, 32768, 128, True,
                    1.0, nq=1)


def varlen() -> Workload:
    return Workload("packed varlen causal 8 seqs H32 d128", 1004, 0, 32, 0, 128, True, 2.0,
                    pv_modes=("fp8",), nseq=8)


def _offset(g: torch.Generator, d: int, std: float, channels: Optional[int]) -> torch.Tensor:
    if channels is None:
        return torch.randn(d, generator=g) * std
    perm = torch.randperm(d, generator=g)[:channels]
    off = torch.zeros(d)
    off[perm] = torch.randn(channels, generator=g) * std
    return off


def make_dense(w: Workload, B: Optional[int] = None, N: Optional[int] = None,
               Nq: Optional[int] = None):
    """fp16 CPU tensors q [B, H, Nq, d] and k, v [B, H, N, d] (B, N and Nq may be
    overridden; Nq defaults to the workload's nq, else N)."""
    B = w.B if B is None else B
    N = w.N if N is None else N
    Nq = (w.nq or N) if Nq is None else Nq
    g = torch.Generator().manual_seed(w.seed)
    shape = (B, w.H, N, w.d)
    q = torch.randn((B, w.H, Nq, w.d), generator=g)
    k = torch.randn(shape, generator=g)
    v = torch.randn(shape, generator=g)
    k += _offset(g, w.d, w.offset_std, w.offset_channels)
    return q.half(), k.half(), v.half()


def make_varlen(w: Workload, nseq: Optional[int] = None, len_lo: Optional[int] = None,
                len_hi: Optional[int] = None, lens=None):
    """Packed fp16 q, k, v of shape [T, H, d] and int32 cu_seqlens [nseq+1]."""
    g = torch.Generator().manual_seed(w.seed)
    nseq = w.nseq if nseq is None else nseq
    lo = w.len_lo if len_lo is None else len_lo
    hi = w.len_hi if len_hi is None else len_hi
    if lens is None:
        lens = torch.randint(lo, hi + 1, (nseq,), generator=g)
    else:
        lens = torch.as_tensor(lens, dtype=torch.int64)
    cu = torch.zeros(len(lens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(lens, 0).to(torch.int32)
    T = int(cu[-1])
    shape = (T, w.H, w.d)
    q = torch.randn(shape, generator=g)
    k = torch.randn(shape, generator=g)
    v = torch.randn(shape, generator=g)
    k += _offset(g, w.d, w.offset_std, w.offset_channels)
    return q.half(), k.half(), v.half(), cu


def make_varlen_kv(w: Workload, lens_q, lens_k):
    """Packed q [Tq, H, d], k and v [Tk, H, d] with their own per-sequence lengths, and
    int32 cu_seqlens_q, cu_seqlens_k."""
    g = torch.Generator().manual_seed(w.seed)
    cq = torch.zeros(len(lens_q) + 1, dtype=torch.int32)
    ck = torch.zeros(len(lens_k) + 1, dtype=torch.int32)
    cq[1:] = torch.cumsum(torch.as_tensor(lens_q, dtype=torch.int64), 0).to(torch.int32)
    ck[1:] = torch.cumsum(torch.as_tensor(lens_k, dtype=torch.int64), 0).to(torch.int32)
    q = torch.randn((int(cq[-1]), w.H, w.d), generator=g)
    k = torch.randn((int(ck[-1]), w.H, w.d), generator=g)
    v = torch.randn((int(ck[-1]), w.H, w.d), generator=g)
    k += _offset(g, w.d, w.offset_std, w.offset_channels)
    return q.half(), k.half(), v.half(), cq, ck


def attention_ops(B: int, H: int, N: int, d: int, causal: bool) -> float:
    """Operation count of one attention forward: 4 B H N^2 d, halved for causal."""
    ops = 4.0 * B * H * N * N * d
    return ops / 2 if causal else ops


def attention_ops_kv(B: int, H: int, Nq: int, Nk: int, d: int, causal: bool) -> float:
    """4 d per visible (query, key) pair: B H Nq Nk 4d, or with the bottom-right causal
    mask B H 4d times the visible pairs sum over i of min(Nk, max(0, i + 1 + Nk - Nq))."""
    if not causal:
        return 4.0 * B * H * Nq * Nk * d
    off = Nk - Nq
    lo = max(0, -off)                  # first query that sees a key
    full = max(lo, min(Nq, Nk - off))  # queries from here on see all Nk keys
    pairs = sum(i + 1 + off for i in range(lo, full)) + (Nq - full) * Nk
    return 4.0 * B * H * pairs * d


def varlen_ops(lens, H: int, d: int, causal: bool) -> float:
    return sum(attention_ops(1, H, int(n), d, causal) for n in lens)
