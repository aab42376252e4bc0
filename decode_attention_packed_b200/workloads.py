"""Seeded synthetic inputs for paged GQA decode attention.

This module only draws and lays out inputs; it holds none of the attention
arithmetic.  The same generator feeds the CUDA path, the benchmark and the
CPU oracle, so that all three see bit-identical inputs.

Five named workloads are shaped like the decode problems the source pages
describe: Qwen3-class grouped-query attention with 2/4/8 query heads per KV
head, head_dim 64 or 128, KV lengths up to 16K, paged caches
("MXFlashAttn 1.4.0" project page, 能力矩阵 capability matrix), small-qLen
speculative/MTP queries with non power-of-two KV lengths ("SmallQ
FlashAttention (Vector)" README, 支持范围 support range), and a low-batch
long-context case that needs the KV axis split ("Flash-Attention GQA
性能调优: pack_gqa 与 num_splits", section "为什么 GQA 推理会喂不饱 SM").

Recipe (per workload index i): ``numpy.random.default_rng(1000 + i)``
(PCG64); KV lengths are drawn first, then the page permutation, then Q, K and
V as N(0, 1) in float32 (K optionally multiplied by ``k_scale``), each rounded
to the storage dtype with round-to-nearest-even.  Paged pools hold exactly
``sum_b ceil(L_b / page)`` pages; a seeded permutation of the page ids is
dealt out to the rows in order; unused block-table slots are 0 and never
read.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Optional

import numpy as np
import torch

DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    q_len: int
    Hq: int
    Hkv: int
    D: int
    dtype: str            # "f16" or "bf16"
    page_size: int        # 0 = contiguous KV ([B, max_seqlen_k, Hkv, D], no block table)
    causal: bool
    lengths: str          # "const:<L>", "uniform:<lo>:<hi>", "cycle:<a>,<b>,...", "loguniform:<lo>:<hi>"
    k_scale: float = 1.0
    num_splits: int = 0   # 0 = let the planner choose
    seed: int = 0

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def M(self) -> int:
        """Packed query rows per KV head: qLen x group."""
        return self.q_len * self.G

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)


WORKLOADS = [
    Workload("tiny_mqa_decode", B=1, q_len=1, Hq=4, Hkv=1, D=64, dtype="f16",
             page_size=0, causal=False, lengths="const:256", num_splits=1, seed=1000),
    Workload("gqa_decode", B=32, q_len=1, Hq=32, Hkv=8, D=128, dtype="bf16",
             page_size=16, causal=False, lengths="uniform:1:4096", seed=1001),
    Workload("spec_mtp_small_q", B=16, q_len=4, Hq=32, Hkv=8, D=128, dtype="bf16",
             page_size=64, causal=True, lengths="cycle:8192,1023,1025,1500,3000", seed=1002),
    Workload("long_context_split_kv", B=2, q_len=1, Hq=64, Hkv=8, D=128, dtype="bf16",
             page_size=64, causal=False, lengths="const:16384", seed=1003),
    Workload("ragged_varlen", B=128, q_len=1, Hq=16, Hkv=8, D=64, dtype="f16",
             page_size=16, causal=False, lengths="loguniform:1:16384", k_scale=3.0, seed=1004),
]

# Other readings of the workloads above, benchmarked for context only: the
# speculative step with every row at 8192 keys (the spec/MTP lengths read as
# "all rows 8192" instead of the cycle through the non-power-of-two lengths);
# and head dim 256, the wider head a model family of the MXFlashAttn page
# uses (its split-KV kernel hands that shape back to a fallback path), as a
# GQA decode batch: groups of 4, 16-slot pages in a seeded permutation.
CONTEXT_WORKLOADS = [
    Workload("spec_mtp_small_q_all8192", B=16, q_len=4, Hq=32, Hkv=8, D=128, dtype="bf16",
             page_size=64, causal=True, lengths="const:8192", seed=1012),
    Workload("gqa_decode_hd256", B=32, q_len=1, Hq=16, Hkv=4, D=256, dtype="bf16",
             page_size=16, causal=False, lengths="uniform:1:4096", seed=1013),
]

BY_NAME = {w.name: w for w in WORKLOADS + CONTEXT_WORKLOADS}


def workload(name_or_index) -> Workload:
    if isinstance(name_or_index, int):
        return WORKLOADS[name_or_index]
    return BY_NAME[name_or_index]


def draw_lengths(w: Workload, rng: np.random.Generator) -> np.ndarray:
    kind, _, arg = w.lengths.partition(":")
    if kind == "const":
        L = np.full(w.B, int(arg), dtype=np.int64)
    elif kind == "uniform":
        lo, hi = (int(x) for x in arg.split(":"))
        L = rng.integers(lo, hi + 1, size=w.B)
    elif kind == "cycle":
        vals = [int(x) for x in arg.split(",")]
        L = np.array([vals[b % len(vals)] for b in range(w.B)], dtype=np.int64)
    elif kind == "loguniform":
        lo, hi = (int(x) for x in arg.split(":"))
        u = rng.uniform(math.log(lo), math.log(hi), size=w.B)
        L = np.clip(np.rint(np.exp(u)), lo, hi).astype(np.int64)
    elif kind == "list":
        L = np.array([int(x) for x in arg.split(",")], dtype=np.int64)
        assert L.size == w.B
    else:
        raise ValueError(f"unknown length recipe {w.lengths!r}")
    return L.astype(np.int32)


@dataclass
class Inputs:
    w: Workload
    q: torch.Tensor                 # [B, q_len, Hq, D] dtype
    k_cache: torch.Tensor           # [num_pages, page, Hkv, D] or [B, max_seqlen_k, Hkv, D]
    v_cache: torch.Tensor
    block_table: Optional[torch.Tensor]   # [B, max_pages_per_seq] int32, or None
    cache_seqlens: torch.Tensor     # [B] int32
    page_size: int                  # slots per page (max_seqlen_k when contiguous)
    max_seqlen_k: int

    @property
    def max_pages_per_seq(self) -> int:
        return 1 if self.block_table is None else int(self.block_table.shape[1])

    @property
    def num_pages(self) -> int:
        return int(self.k_cache.shape[0])

    def kv_bytes(self) -> int:
        """Algorithmic K+V bytes one pass reads: sum_b L_b * Hkv * 2 * D * elem."""
        es = self.q.element_size()
        return int(self.cache_seqlens.to(torch.int64).sum()) * self.w.Hkv * 2 * self.w.D * es


def _round(x: np.ndarray, dtype: str) -> torch.Tensor:
    # float32 -> 16-bit storage, round-to-nearest-even (torch's cast)
    return torch.from_numpy(x).to(DTYPES[dtype])


def make_inputs(w: Workload, seed: Optional[int] = None,
                lengths: Optional[np.ndarray] = None,
                max_seqlen_k: Optional[int] = None) -> Inputs:
    """Draw one seeded problem instance on the host (torch CPU tensors)."""
    rng = np.random.default_rng(w.seed if seed is None else seed)
    L = draw_lengths(w, rng) if lengths is None else np.asarray(lengths, dtype=np.int32)
    assert L.shape == (w.B,) and (L >= 0).all()
    Lmax = int(L.max()) if L.size else 0
    if max_seqlen_k is None:
        max_seqlen_k = max(Lmax, 1)
    assert max_seqlen_k >= Lmax

    if w.page_size == 0:
        page = max_seqlen_k
        pool_shape = (w.B, page, w.Hkv, w.D)
        block_table = None
    else:
        page = w.page_size
        pages_per_seq = [(int(l) + page - 1) // page for l in L]
        num_pages = max(sum(pages_per_seq), 1)
        perm = rng.permutation(num_pages).astype(np.int32)
        max_pages = max(max(pages_per_seq, default=0), 1)
        bt = np.zeros((w.B, max_pages), dtype=np.int32)
        pos = 0
        for b, n in enumerate(pages_per_seq):
            bt[b, :n] = perm[pos:pos + n]
            pos += n
        block_table = torch.from_numpy(bt)
        pool_shape = (num_pages, page, w.Hkv, w.D)

    q = rng.standard_normal((w.B, w.q_len, w.Hq, w.D), dtype=np.float32)
    k = rng.standard_normal(pool_shape, dtype=np.float32)
    if w.k_scale != 1.0:
        k *= np.float32(w.k_scale)
    v = rng.standard_normal(pool_shape, dtype=np.float32)
    return Inputs(w=w, q=_round(q, w.dtype), k_cache=_round(k, w.dtype),
                  v_cache=_round(v, w.dtype), block_table=block_table,
                  cache_seqlens=torch.from_numpy(L.copy()), page_size=page,
                  max_seqlen_k=max_seqlen_k)


def make_varlen_queries(q_lens, Hq: int, D: int, dtype: str, seed: int):
    """Queries of rows with their own query counts, packed: q [total_q, Hq, D]
    (N(0, 1) rounded to `dtype`) and the offsets cu [B + 1] int32 (0, then the
    running totals of q_lens)."""
    rng = np.random.default_rng(seed)
    ql = np.asarray(q_lens, dtype=np.int64)
    assert ql.ndim == 1 and (ql >= 0).all()
    cu = np.concatenate([[0], np.cumsum(ql)]).astype(np.int32)
    q = rng.standard_normal((int(cu[-1]), Hq, D), dtype=np.float32)
    return _round(q, dtype), torch.from_numpy(cu)


def small_variant(w: Workload, **changes) -> Workload:
    """The same recipe with some fields changed (used for parity cases the
    oracle finishes in seconds)."""
    return replace(w, **changes)


def shard_rows(B: int, rank: int, world: int) -> range:
    """Contiguous batch rows owned by `rank` when B rows are spread over
    `world` processes.  Decode rows are independent, so sharding needs no
    exchange between ranks."""
    base, extra = divmod(B, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))
