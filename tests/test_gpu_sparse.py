"""GPU parity of the sparse (top-k) decode through the C ABI against the CPU
statement in oracle/sparse.py: |out - ref| <= 1e-2 + 1e-2 |ref| on the bf16
output and |lse - ref| <= 1e-3, as for the dense decode.  Index lists carry
padding (-1 and positions past the sequence), repeats, and positions past the
causal limit; some query positions select nothing."""
import numpy as np
import pytest
import torch

from oracle import sparse
from mla_paged_latent_decode_b200 import synth
from parity import assert_close_lse, assert_close_out

pytestmark = pytest.mark.gpu


def run_sparse(inp, idx, dev):
    from mla_paged_latent_decode_b200 import binding
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    out, lse = binding.mla_decode_sparse(inp.q.to(dev), inp.kcache.to(dev),
                                         inp.block_table.to(dev), inp.cache_seqlens.to(dev),
                                         idx.to(dev), inp.scale, inp.causal, device_status=status)
    torch.cuda.synchronize(dev)
    assert int(status.item()) == 0
    return out.float().cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("h_q", [16, 128])
@pytest.mark.parametrize("s_q,causal", [(1, False), (2, True), (3, False)])
@pytest.mark.parametrize("topk", [1, 100, 300])
def test_sparse_small(cuda_device, h_q, s_q, causal, topk):
    w = synth.custom_workload(4, s_q, h_q, [1, 63, 200, 700], causal=causal)
    inp = synth.make_inputs(w, seed=70 + h_q + s_q + topk)
    idx = synth.make_sparse_indices(inp, topk, seed=topk, pad_frac=0.2)
    out, lse = run_sparse(inp, idx, cuda_device)
    ref_out, ref_lse = sparse.decode(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens, idx,
                                     inp.scale, inp.causal)
    assert_close_out(out, ref_out, "sparse out")
    assert_close_lse(lse, ref_lse, "sparse lse")


def test_sparse_repeats_and_empty_positions(cuda_device):
    w = synth.custom_workload(3, 2, 16, [50, 80, 5], causal=True)
    inp = synth.make_inputs(w, seed=75)
    idx = torch.full((3, 2, 8), -1, dtype=torch.int32)
    idx[0, 0, :4] = torch.tensor([3, 3, 7, 49])      # 49 is past the causal limit of j = 0
    idx[0, 1, :3] = torch.tensor([49, 0, 0])
    idx[1, 1, :2] = torch.tensor([79, 1 << 20])       # position 0 of sequence 1 selects nothing
    idx[2, 0, :1] = torch.tensor([4])                 # causal limit of j = 0 is 3: nothing used
    idx[2, 1, :2] = torch.tensor([4, 2])
    out, lse = run_sparse(inp, idx, cuda_device)
    ref_out, ref_lse = sparse.decode(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens, idx,
                                     inp.scale, True)
    assert_close_out(out, ref_out, "sparse out")
    assert_close_lse(lse, ref_lse, "sparse lse")
    assert not out[1, 0].any() and np.all(np.isneginf(lse[1, :, 0]))
    assert not out[2, 0].any() and np.all(np.isneginf(lse[2, :, 0]))


def test_sparse_dsa_shaped(cuda_device):
    # 2048 selected tokens per query position out of 8192, 128 heads
    w = synth.custom_workload(4, 1, 128, [8192, 8192, 3000, 8192])
    inp = synth.make_inputs(w, seed=76)
    idx = synth.make_sparse_indices(inp, 2048, seed=76)
    out, lse = run_sparse(inp, idx, cuda_device)
    ref_out, ref_lse = sparse.decode(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens, idx,
                                     inp.scale, False)
    assert_close_out(out, ref_out, "sparse out")
    assert_close_lse(lse, ref_lse, "sparse lse")


def test_sparse_full_list_equals_dense(cuda_device):
    # every position in order: the sparse path must agree with the dense one
    from parity import run_cuda
    w = synth.custom_workload(3, 2, 64, [130, 64, 257], causal=True)
    inp = synth.make_inputs(w, seed=77)
    idx = torch.full((3, 2, 257), -1, dtype=torch.int32)
    for i, L in enumerate(inp.cache_seqlens.tolist()):
        idx[i, :, :L] = torch.arange(L, dtype=torch.int32)
    out, lse = run_sparse(inp, idx, cuda_device)
    dense = run_cuda(inp, cuda_device)
    np.testing.assert_allclose(out, dense["out"], atol=1e-2, rtol=1e-2)
    np.testing.assert_allclose(lse, dense["lse"], atol=1e-3)


@pytest.mark.parametrize("s_q,causal", [(1, False), (2, True)])
def test_sparse_full_list_equals_dense_on_pairs(cuda_device, s_q, causal):
    # 128 heads: the pair kernel copies the listed rows itself; with every
    # position listed, in order, it must agree with the dense decode
    from parity import run_cuda
    w = synth.custom_workload(3, s_q, 128, [130, 64, 1000], causal=causal)
    inp = synth.make_inputs(w, seed=78 + s_q)
    idx = torch.full((3, s_q, 1000), -1, dtype=torch.int32)
    for i, L in enumerate(inp.cache_seqlens.tolist()):
        idx[i, :, :L] = torch.arange(L, dtype=torch.int32)
    out, lse = run_sparse(inp, idx, cuda_device)
    dense = run_cuda(inp, cuda_device)
    np.testing.assert_allclose(out, dense["out"], atol=1e-2, rtol=1e-2)
    np.testing.assert_allclose(lse, dense["lse"], atol=1e-3)


@pytest.mark.parametrize("h_q", [16, 128])
def test_sparse_entry_on_a_page_outside_the_cache(cuda_device, h_q):
    # a used entry whose block-table page lies outside the cache is read as a
    # zero row and reported; the rest of the result is exact
    from mla_paged_latent_decode_b200 import binding
    w = synth.custom_workload(2, 1, h_q, [300, 200])
    inp = synth.make_inputs(w, seed=79)
    nb = inp.kcache.shape[0]
    idx = synth.make_sparse_indices(inp, 40, seed=79)
    idx[0, 0, 0] = 70                      # token 70 lives in logical page 1 of sequence 0
    bad_bt = inp.block_table.clone()
    bad_bt[0, 1] = nb + 5                  # ... which now points past the cache
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out, lse = binding.mla_decode_sparse(inp.q.to(cuda_device), inp.kcache.to(cuda_device),
                                         bad_bt.to(cuda_device), inp.cache_seqlens.to(cuda_device),
                                         idx.to(cuda_device), inp.scale, False,
                                         device_status=status)
    torch.cuda.synchronize(cuda_device)
    assert int(status.item()) == binding.MLA_ERR_DEVICE_CHECK
    # the oracle on a cache with one more page, all zeros, in place of the bad one
    kc = torch.cat([inp.kcache, torch.zeros((1, 64, 576), dtype=torch.bfloat16)])
    zero_bt = inp.block_table.clone()
    zero_bt[0, 1] = nb
    ref_out, ref_lse = sparse.decode(inp.q, kc, zero_bt, inp.cache_seqlens, idx, inp.scale, False)
    assert_close_out(out.float().cpu().numpy(), ref_out, "sparse out")
    assert_close_lse(lse.cpu().numpy(), ref_lse, "sparse lse")
