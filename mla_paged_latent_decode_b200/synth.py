"""Seeded synthetic decode workloads for MLA over a paged latent cache.

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic.  The same inputs feed the CUDA path and the fp64 oracle.

Layouts (all row-major, contiguous):
  q             [b, s_q, h_q, 576]  bf16   query heads: 512 latent + 64 rope dims
  kcache        [nblk, 64, 576]     bf16   one latent row per cached token, 64-token pages
  block_table   [b, max_pages]      int32  physical page of each logical page
  cache_seqlens [b]                 int32  tokens cached per sequence

The page size of 64 and the bf16 cache follow "OpenSourceWeek Day 1: FlashMLA",
"Key Highlights" (BF16, paged KV cache with block size 64).  The 576-dim row with
its first 512 dims as the value is the absorbed-weight MLA form; the pages state
only that one latent vector per token is cached and that K and V are derived
from it ("How MLA Optimizes Memory Usage").

Draw order for a given seed (a torch CPU generator):
  1. cache_seqlens (when random),
  2. a permutation of the page pool; sequence i takes the next ceil(L_i/64) pages,
  3. q ~ N(0, 1) rounded to bf16,
  4. kcache ~ N(0, 1) rounded to bf16.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

PAGE = 64
D_QK = 576
D_V = 512
# 1/sqrt(192): DeepSeek-V3's per-head qk width (128 nope + 64 rope), rounded to fp32.
DEFAULT_SCALE = float(torch.tensor(1.0 / math.sqrt(192.0), dtype=torch.float32).item())
POISON = 3.0e4


@dataclass(frozen=True)
class Workload:
    """A named decode workload: shapes plus how its sequence lengths are drawn."""

    name: str
    batch: int
    s_q: int
    h_q: int
    seqlens: tuple | None = None      # fixed lengths, or None to draw uniformly
    seqlen_range: tuple | None = None  # inclusive (lo, hi) for the uniform draw
    causal: bool = False
    pool_pages: int | None = None     # page-pool size; default = pages in use
    scale: float = DEFAULT_SCALE
    description: str = field(default="", compare=False)


WORKLOADS = {
    "tiny": Workload(
        "tiny", 2, 1, 16, seqlens=(37, 130),
        description="batch 2, s_q 1, 16 heads, seqlens {37, 130}, non-causal"),
    "dsv3_decode": Workload(
        "dsv3_decode", 64, 1, 128, seqlens=(4096,) * 64,
        description="DeepSeek-V3-shaped decode: batch 64, s_q 1, 128 heads, every seqlen 4096"),
    "varlen_h16": Workload(
        "varlen_h16", 128, 1, 16, seqlen_range=(1, 8192),
        description="memory-bound variable length: batch 128, 16 heads, seqlens U[1, 8192]"),
    "spec_causal": Workload(
        "spec_causal", 32, 2, 128, seqlen_range=(2048, 16384), causal=True,
        description="speculative decode: batch 32, s_q 2 causal, 128 heads, seqlens U[2048, 16384]"),
    "skewed_long": Workload(
        "skewed_long", 16, 1, 128, seqlens=(32768,) * 15 + (1,), pool_pages=8192,
        description="skewed long context: 15 x 32768 + 1 token, 128 heads, 512K-token page pool"),
}


@dataclass
class DecodeInputs:
    workload: Workload
    seed: int
    q: torch.Tensor
    kcache: torch.Tensor
    block_table: torch.Tensor
    cache_seqlens: torch.Tensor
    scale: float
    causal: bool
    poison_page: int | None = None

    @property
    def batch(self) -> int:
        return self.q.shape[0]

    @property
    def s_q(self) -> int:
        return self.q.shape[1]

    @property
    def h_q(self) -> int:
        return self.q.shape[2]


def pages_for(seqlen: int) -> int:
    return (int(seqlen) + PAGE - 1) // PAGE


def draw_seqlens(w: Workload, gen: torch.Generator) -> torch.Tensor:
    if w.seqlens is not None:
        assert len(w.seqlens) == w.batch
        return torch.tensor(w.seqlens, dtype=torch.int32)
    lo, hi = w.seqlen_range
    return torch.randint(lo, hi + 1, (w.batch,), generator=gen, dtype=torch.int32)


def make_inputs(w: Workload | str, seed: int = 0, poison: bool = False,
                seqlens: list | None = None) -> DecodeInputs:
    """Draw the inputs of workload `w` from `seed`.

    poison=True appends one extra page filled with +-3e4, points every unused
    block-table entry at it, and overwrites the rows past each sequence's end in
    its last page with the same pattern.  Those values must not reach any output.
    `seqlens` overrides the workload's lengths (same batch size).
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    gen = torch.Generator().manual_seed(seed)
    if seqlens is not None:
        lens = torch.tensor(list(seqlens), dtype=torch.int32)
        assert lens.numel() == w.batch
    else:
        lens = draw_seqlens(w, gen)
    n_pages = [pages_for(v) for v in lens.tolist()]
    used = sum(n_pages)
    pool = max(used, 1) if w.pool_pages is None else w.pool_pages
    assert pool >= used, "page pool smaller than the pages in use"
    perm = torch.randperm(pool, generator=gen).to(torch.int32)
    max_pages = max(max(n_pages), 1)
    block_table = torch.zeros((w.batch, max_pages), dtype=torch.int32)
    cursor = 0
    for i, n in enumerate(n_pages):
        block_table[i, :n] = perm[cursor:cursor + n]
        cursor += n
    q = torch.randn((w.batch, w.s_q, w.h_q, D_QK), generator=gen).to(torch.bfloat16)
    kcache = torch.randn((pool, PAGE, D_QK), generator=gen).to(torch.bfloat16)
    poison_page = None
    if poison:
        pattern = torch.full((PAGE, D_QK), POISON)
        pattern[:, 1::2] = -POISON
        pattern = pattern.to(torch.bfloat16)
        kcache = torch.cat([kcache, pattern[None]], dim=0)
        poison_page = pool
        for i, n in enumerate(n_pages):
            block_table[i, n:] = poison_page
            tail = int(lens[i]) - (n - 1) * PAGE if n > 0 else 0
            if n > 0 and tail < PAGE:
                kcache[int(block_table[i, n - 1]), tail:] = pattern[tail:]
    return DecodeInputs(w, seed, q.contiguous(), kcache.contiguous(), block_table.contiguous(),
                        lens.contiguous(), w.scale, w.causal, poison_page)


def custom_workload(batch: int, s_q: int, h_q: int, seqlens, causal: bool = False,
                    scale: float = DEFAULT_SCALE, pool_pages: int | None = None,
                    name: str = "custom") -> Workload:
    """A workload with explicit lengths, for edge-case and parity tests."""
    return Workload(name, batch, s_q, h_q, seqlens=tuple(int(v) for v in seqlens),
                    causal=causal, pool_pages=pool_pages, scale=scale)


def algorithmic_work(inp: DecodeInputs, kv_bytes_per_token: int = D_QK * 2) -> tuple[int, int]:
    """(bytes, flops) the method must move or compute for one call.

    kv_bytes_per_token: bytes of one cached row (1152 for bf16; 580 for 576
    E4M3 codes plus a 4-byte scale).
    bytes: every visible-or-not cached row once (576 values, read once because
    the value is the first 512 dims of the same row), q in, out and lse out,
    seqlens and the used block-table entries.
    flops: 2 * (576 + 512) per (query row, visible key) pair.
    """
    b, s_q, h_q = inp.batch, inp.s_q, inp.h_q
    lens = inp.cache_seqlens.tolist()
    total_tokens = sum(lens)
    n_pages = sum(pages_for(v) for v in lens)
    nbytes = (total_tokens * kv_bytes_per_token + b * s_q * h_q * (D_QK * 2 + D_V * 2)
              + b * h_q * s_q * 4 + 4 * (b + n_pages))
    pairs = 0
    for L in lens:
        for j in range(s_q):
            vis = L - s_q + j + 1 if inp.causal else L
            pairs += max(0, min(vis, L))
    flops = 2 * (D_QK + D_V) * h_q * pairs
    return nbytes, flops


def make_sparse_indices(inp: DecodeInputs, topk: int, seed: int = 0, pad_frac: float = 0.0):
    """indices [b, s_q, topk] int32 for the sparse decode: for each query
    position, min(topk, L) distinct positions drawn uniformly from [0, L) in
    random order, the rest -1.  With pad_frac > 0 that fraction of the drawn
    entries is replaced by -1 or by positions past the sequence's end."""
    gen = torch.Generator().manual_seed(seed)
    b, s_q = inp.batch, inp.s_q
    idx = torch.full((b, s_q, topk), -1, dtype=torch.int32)
    for i, L in enumerate(inp.cache_seqlens.tolist()):
        for j in range(s_q):
            k = min(topk, L)
            if k > 0:
                idx[i, j, :k] = torch.randperm(L, generator=gen)[:k].to(torch.int32)
    if pad_frac > 0:
        drop = torch.rand((b, s_q, topk), generator=gen) < pad_frac
        far = torch.rand((b, s_q, topk), generator=gen) < 0.5
        idx = torch.where(drop & far, torch.full_like(idx, 1 << 30), idx)
        idx = torch.where(drop & ~far, torch.full_like(idx, -1), idx)
    return idx.contiguous()


def sparse_algorithmic_work(inp: DecodeInputs, indices: torch.Tensor) -> tuple[int, int]:
    """(bytes, flops) of one sparse decode call: every used entry's cached row
    once (1152 bytes), q in, out and lse out, and the index lists; 2 * (576 +
    512) flops per (head, used entry)."""
    b, s_q, h_q = inp.batch, inp.s_q, inp.h_q
    lens = inp.cache_seqlens.tolist()
    used = 0
    for i in range(b):
        for j in range(s_q):
            lim = min(lens[i] - s_q + j + 1, lens[i]) if inp.causal else lens[i]
            row = indices[i, j]
            used += int(((row >= 0) & (row < lim)).sum())
    nbytes = (used * D_QK * 2 + b * s_q * h_q * (D_QK * 2 + D_V * 2) + b * h_q * s_q * 4
              + indices.numel() * 4)
    return nbytes, 2 * (D_QK + D_V) * h_q * used
