"""The host side of the sharded decode (no GPU): how pages are split over ranks,
that the split keeps causal decode exact, and the all-gather of the ranks'
results over gloo (world size 2).

The per-rank decodes and the merge here are the oracle's (this checks the
sharding rule and the exchange, not the kernels; the GPU test runs the
library's decode and merge kernels on emulated ranks).
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from mla_paged_latent_decode_b200 import synth
from mla_paged_latent_decode_b200.sharded import shard_inputs, shard_plan, split_pages

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("world", [1, 2, 3, 4, 7])
def test_split_pages(world):
    for n in range(0, 40):
        sizes = split_pages(n, world)
        assert len(sizes) == world and sum(sizes) == n and min(sizes) >= 0
        assert sizes[-1] >= min(n, 2)
        assert max(sizes) - min(s for s in sizes[:-1] or [sizes[-1]]) <= 2


@pytest.mark.parametrize("world", [1, 2, 3, 5])
def test_shard_plan_covers_every_token_once(world):
    lens = [0, 1, 63, 64, 65, 128, 129, 1000, 4096]
    plan = shard_plan(lens, world)
    for i, L in enumerate(lens):
        start_expect, total = 0, 0
        for r in range(world):
            start, size, tokens = plan[r][i]
            assert start == start_expect
            start_expect += size
            total += tokens
            if size > 0:
                assert tokens > 0 and tokens <= size * 64
        assert total == L and start_expect == (L + 63) // 64
        # the last rank holds the last page (and, from two pages on, the last two)
        n = (L + 63) // 64
        assert plan[world - 1][i][1] >= min(n, 2)


def oracle_sharded(inp, world):
    """Every rank's decode by the oracle, merged by the oracle's combine."""
    parts = []
    for r in range(world):
        bt, sl = shard_inputs(inp.block_table, inp.cache_seqlens, world, r)
        parts.append(oracle.decode(inp.q, inp.kcache, bt, sl, inp.scale,
                                   inp.causal and r == world - 1))
    b, s_q, h_q = inp.batch, inp.s_q, inp.h_q
    out = np.zeros((b, s_q, h_q, 512))
    lse = np.zeros((b, h_q, s_q))
    for i in range(b):
        for j in range(s_q):
            for h in range(h_q):
                o, l = oracle.combine([p[0][i, j, h] for p in parts], [p[1][i, h, j] for p in parts])
                out[i, j, h], lse[i, h, j] = o, l
    return out, lse


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("s_q,causal", [(1, False), (2, True), (3, True), (2, False)])
def test_sharding_keeps_the_decode_exact(world, s_q, causal):
    # lengths that put a page boundary right at the causal limit, a last page
    # with one token, a sequence shorter than s_q, and fewer pages than ranks
    w = synth.custom_workload(6, s_q, 2, [1, 2, 65, 129, 300, 64 * 5 + 1], causal=causal)
    inp = synth.make_inputs(w, seed=50 + world)
    want_out, want_lse = oracle.decode(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens,
                                       inp.scale, inp.causal)
    got_out, got_lse = oracle_sharded(inp, world)
    np.testing.assert_allclose(got_out, want_out, rtol=1e-10, atol=1e-12)
    fin = np.isfinite(want_lse)
    assert np.array_equal(fin, np.isfinite(got_lse))
    np.testing.assert_allclose(got_lse[fin], want_lse[fin], rtol=1e-12, atol=1e-12)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    import oracle as orc
    from mla_paged_latent_decode_b200 import synth as sy
    from mla_paged_latent_decode_b200.sharded import gather_parts, shard_inputs as si
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = sy.custom_workload(3, 2, 4, [130, 1, 700], causal=True)
        inp = sy.make_inputs(w, seed=61)
        bt, sl = si(inp.block_table, inp.cache_seqlens, world, rank)
        o, l = orc.decode(inp.q, inp.kcache, bt, sl, inp.scale, rank == world - 1)
        outs, lses = gather_parts(torch.from_numpy(o), torch.from_numpy(l))
        if rank == 0:
            want_o, want_l = orc.decode(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens,
                                        inp.scale, True)
            err = 0.0
            for i in range(3):
                for j in range(2):
                    for h in range(4):
                        mo, ml = orc.combine(outs[:, i, j, h].numpy(), lses[:, i, h, j].numpy())
                        err = max(err, float(np.abs(mo - want_o[i, j, h]).max()),
                                  abs(ml - want_l[i, h, j]))
            q.put(err)
    finally:
        dist.destroy_process_group()


def test_gather_parts_over_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gloo_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs)
    assert q.get(timeout=5) < 1e-10
