"""GPU parity of the sharded decode's kernels on emulated ranks (one GPU).

Each rank's shard is decoded by the library over the pages that rank would
hold (its own block table and lengths, see sharded.shard_inputs); the results
are stacked in rank order, as the all-gather delivers them, and merged by the
library's merge kernel.  The result must match the oracle's unsharded decode
within the decode's tolerance.  The exchange itself (NCCL all-gather) needs
several GPUs; its host side runs over gloo in test_sharded_host.py.
"""
import numpy as np
import pytest
import torch

import oracle
from mla_paged_latent_decode_b200 import binding, synth
from mla_paged_latent_decode_b200.sharded import shard_inputs
from parity import assert_close_lse, assert_close_out

pytestmark = pytest.mark.gpu


def emulated(inp, world, dev):
    q, kc = inp.q.to(dev), inp.kcache.to(dev)
    outs, lses = [], []
    for r in range(world):
        bt, sl = shard_inputs(inp.block_table, inp.cache_seqlens, world, r)
        bt, sl = bt.to(dev), sl.to(dev)
        md, ns = binding.get_mla_metadata(sl, inp.h_q, inp.s_q)
        o, l = binding.mla_decode_kvcache(q, kc, bt, sl, 512, md, ns, inp.scale,
                                          inp.causal and r == world - 1)
        outs.append(o)
        lses.append(l)
    out, lse = binding.merge_partials(torch.stack(outs), torch.stack(lses))
    torch.cuda.synchronize(dev)
    return out.float().cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("world", [1, 2, 4, 8])
@pytest.mark.parametrize("s_q,h_q,causal", [(1, 16, False), (1, 128, False), (2, 128, True)])
def test_sharded_decode_matches_oracle(cuda_device, world, s_q, h_q, causal):
    w = synth.custom_workload(5, s_q, h_q, [1, 130, 4096, 64 * 9 + 1, 2000], causal=causal)
    inp = synth.make_inputs(w, seed=70 + world)
    out, lse = emulated(inp, world, cuda_device)
    ref_out, ref_lse = oracle.decode(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens,
                                     inp.scale, inp.causal)
    assert_close_out(out, ref_out, f"sharded out (world {world})")
    assert_close_lse(lse, ref_lse, f"sharded lse (world {world})")


def test_merge_of_empty_and_single_parts(cuda_device):
    # a part with lse = -inf weighs nothing; all parts empty gives 0 and -inf;
    # one part is returned as it is (bit for bit)
    g = torch.Generator().manual_seed(3)
    b, s_q, h_q, R = 3, 2, 8, 3
    outs = torch.randn((R, b, s_q, h_q, 512), generator=g).to(torch.bfloat16)
    lses = torch.randn((R, b, h_q, s_q), generator=g, dtype=torch.float64).float()
    lses[1] = -float("inf")           # part 1 empty everywhere
    lses[:, 2] = -float("inf")        # sequence 2 empty in every part
    out, lse = binding.merge_partials(outs.to(cuda_device), lses.to(cuda_device))
    torch.cuda.synchronize(cuda_device)
    out, lse = out.float().cpu().numpy(), lse.cpu().numpy()
    for i in range(b):
        for j in range(s_q):
            for h in range(h_q):
                o, l = oracle.combine(outs[:, i, j, h].double().numpy(),
                                      lses[:, i, h, j].double().numpy())
                assert np.all(np.abs(out[i, j, h] - o) <= 1e-2 + 1e-2 * np.abs(o))
                assert (np.isneginf(l) and np.isneginf(lse[i, h, j])) or abs(lse[i, h, j] - l) <= 1e-5
    assert np.all(out[2] == 0) and np.all(np.isneginf(lse[2]))
    one, one_lse = binding.merge_partials(outs[:1].to(cuda_device), lses[:1].to(cuda_device))
    torch.cuda.synchronize(cuda_device)
    assert torch.equal(one.cpu()[:2], outs[0][:2])
    assert torch.equal(one_lse.cpu()[:2], lses[0][:2])
