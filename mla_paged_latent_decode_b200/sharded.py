"""Decode over a latent cache sharded across GPUs by token ranges, merged by lse.

Each of `world` ranks holds a contiguous run of every sequence's 64-token pages
in its own page pool.  Every rank decodes the same queries over the pages it
holds, the ranks all-gather their (out, lse) pairs, and each merges them with
mla_merge_partials:
    lse = ln sum_r exp(lse_r),  out = sum_r exp(lse_r - lse) out_r.
This is the partition-then-combine form of multi-device latent attention
("TPLA: Tensor Parallel Latent Attention...", abstract), applied to the cached
tokens rather than to the latent dims, so the result is the exact attention of
the unsharded decode (within bf16 rounding of the exchanged outputs).

Causal decode (query j of a sequence of L tokens sees tokens t <= L - s_q + j)
stays exact because the last rank always holds the sequence's last page and,
when the sequence has two or more pages, at least its last two: with s_q <= 64
every token before that run is visible to every query, so the other ranks run
without the mask and only the last rank applies it to its own (local) length.

Only the exchange uses torch.distributed (NCCL between GPUs): one all-gather of
the bf16 outputs and one of the fp32 lse values.  Both decode and merge run in
the library's kernels.
"""
from __future__ import annotations

import torch

from . import binding

PAGE = binding.PAGE


def split_pages(npages: int, world: int) -> list[int]:
    """Pages of one sequence per rank: as even as possible, extra pages on the
    last ranks, and the last rank holding at least min(npages, 2)."""
    q, rem = divmod(npages, world)
    sizes = [q + (1 if r >= world - rem else 0) for r in range(world)]
    need = min(npages, 2)
    r = world - 2
    while sizes[-1] < need and r >= 0:
        if sizes[r] > 0:
            sizes[r] -= 1
            sizes[-1] += 1
        else:
            r -= 1
    return sizes


def shard_plan(cache_seqlens, world: int):
    """Per rank and sequence: (first page, page count, local token count)."""
    lens = [int(v) for v in (cache_seqlens.tolist() if hasattr(cache_seqlens, "tolist")
                             else cache_seqlens)]
    plan = [[] for _ in range(world)]
    for L in lens:
        n = (L + PAGE - 1) // PAGE if L > 0 else 0
        start = 0
        for r, size in enumerate(split_pages(n, world)):
            tokens = max(0, min(L, (start + size) * PAGE) - start * PAGE) if size > 0 else 0
            plan[r].append((start, size, tokens))
            start += size
    return plan


def shard_inputs(block_table: torch.Tensor, cache_seqlens: torch.Tensor, world: int, rank: int):
    """This rank's block table [b, max local pages] (entries of the global one)
    and local lengths [b], from the global block table and lengths (host tensors
    or device tensors; computed on the host)."""
    plan = shard_plan(cache_seqlens.cpu(), world)[rank]
    bt = block_table.cpu()
    width = max(1, max(size for _, size, _ in plan))
    local_bt = torch.zeros((len(plan), width), dtype=torch.int32)
    local_len = torch.zeros((len(plan),), dtype=torch.int32)
    for i, (start, size, tokens) in enumerate(plan):
        local_bt[i, :size] = bt[i, start:start + size]
        local_len[i] = tokens
    return local_bt.to(block_table.device), local_len.to(cache_seqlens.device)


def gather_parts(out_local: torch.Tensor, lse_local: torch.Tensor, group=None):
    """All-gather every rank's (out, lse): returns outs [world, ...] and lses
    [world, ...] in rank order (NCCL on GPUs; any backend works)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    # ranks' tensors concatenated along dim 0, then viewed as [world, ...]
    outs = torch.empty((world * out_local.shape[0], *out_local.shape[1:]), dtype=out_local.dtype,
                       device=out_local.device)
    lses = torch.empty((world * lse_local.shape[0], *lse_local.shape[1:]), dtype=lse_local.dtype,
                       device=lse_local.device)
    dist.all_gather_into_tensor(outs, out_local.contiguous(), group=group)
    dist.all_gather_into_tensor(lses, lse_local.contiguous(), group=group)
    return outs.view(world, *out_local.shape), lses.view(world, *lse_local.shape)


def sharded_decode(q: torch.Tensor, kcache: torch.Tensor, local_block_table: torch.Tensor,
                   local_seqlens: torch.Tensor, softmax_scale: float, causal: bool = False,
                   group=None):
    """Decode over this rank's shard of the cache, then exchange and merge.
    q [b, s_q, h_q, 576] is the same on every rank; kcache is this rank's page
    pool and local_block_table / local_seqlens its shard (see shard_inputs).
    Returns the full (out [b, s_q, h_q, 512] bf16, lse [b, h_q, s_q] fp32) on
    every rank."""
    import torch.distributed as dist
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    s_q, h_q = q.shape[1], q.shape[2]
    if causal and s_q > 64:
        raise ValueError("causal sharded decode needs s_q <= 64")
    md, ns = binding.get_mla_metadata(local_seqlens, h_q, s_q)
    out, lse = binding.mla_decode_kvcache(q, kcache, local_block_table, local_seqlens, binding.D_V,
                                          md, ns, softmax_scale,
                                          causal=bool(causal) and rank == world - 1)
    outs, lses = gather_parts(out, lse, group)
    return binding.merge_partials(outs, lses)
