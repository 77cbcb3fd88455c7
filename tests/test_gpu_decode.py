"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Tolerance of the decode: |out - ref| <= 1e-2 + 1e-2 |ref| on the bf16 output,
|lse - ref| <= 1e-3, and the split metadata bit-exact against the CPU
restatement of the partition rule.
"""
import numpy as np
import pytest
import torch

from mla_paged_latent_decode_b200 import synth
from parity import (check_metadata, full_parity, full_size_parity, run_cuda, assert_close_out,
                    assert_close_lse, expected_workers)

pytestmark = pytest.mark.gpu


def test_tiny_workload(cuda_device):
    inp = synth.make_inputs("tiny", seed=0)
    full_parity(inp, cuda_device)


@pytest.mark.parametrize("h_q", [1, 16, 64, 128])
@pytest.mark.parametrize("s_q,causal", [(1, False), (2, True), (2, False)])
def test_small_shapes(cuda_device, h_q, s_q, causal):
    # several pages, ragged tails, one sequence shorter than a page
    w = synth.custom_workload(4, s_q, h_q, [1, 63, 130, 257], causal=causal)
    inp = synth.make_inputs(w, seed=100 + h_q + s_q)
    full_parity(inp, cuda_device)


@pytest.mark.parametrize("s_q,h_q,causal", [(1, 1, False), (1, 4, False), (2, 8, True),
                                             (1, 16, False), (4, 4, True), (3, 5, False)])
def test_narrow_rows(cuda_device, s_q, h_q, causal):
    # few query rows per sequence (1 to 16): most of the single-CTA kernel's
    # 64-row block is padding, whose rows must never reach the output
    w = synth.custom_workload(5, s_q, h_q, [1, 63, 64, 130, 2000], causal=causal)
    inp = synth.make_inputs(w, seed=400 + s_q * h_q)
    full_parity(inp, cuda_device)
    full_parity(inp, cuda_device, num_workers=9)


@pytest.mark.parametrize("num_workers", [1, 2, 7, 148, 600])
def test_few_rows_forced_splits_and_poison(cuda_device, num_workers):
    w = synth.custom_workload(3, 1, 16, [700, 5, 1100])
    inp = synth.make_inputs(w, seed=17, poison=True)
    full_parity(inp, cuda_device, num_workers=num_workers)


@pytest.mark.parametrize("num_workers", [1, 3, 17, 148, 600])
def test_forced_splits(cuda_device, num_workers):
    # num_workers controls how finely sequences are cut: 1 = no splits at all,
    # 600 = a piece per page; every plan must give the same answer
    w = synth.custom_workload(3, 2, 32, [700, 5, 1100], causal=True)
    inp = synth.make_inputs(w, seed=7)
    full_parity(inp, cuda_device, num_workers=num_workers)


@pytest.mark.parametrize("num_workers", [1, 2, 5, 37, 74, 300])
def test_forced_splits_pairs(cuda_device, num_workers):
    # more than 64 query rows run on CTA pairs: two 128-row blocks per worker,
    # every split plan
    w = synth.custom_workload(3, 2, 128, [700, 5, 1100], causal=True)
    inp = synth.make_inputs(w, seed=8)
    full_parity(inp, cuda_device, num_workers=num_workers)


@pytest.mark.parametrize("s_q,h_q,causal", [(3, 32, True), (1, 96, False), (4, 128, True),
                                             (2, 96, True), (1, 65, False)])
def test_pair_row_blocks(cuda_device, s_q, h_q, causal):
    # query-row counts on the CTA-pair path: a second CTA with some or no valid
    # rows (96, 65 rows), several 128-row blocks per worker (192, 384, 512 rows)
    w = synth.custom_workload(3, s_q, h_q, [900, 3, 200], causal=causal)
    inp = synth.make_inputs(w, seed=20 + s_q * h_q)
    full_parity(inp, cuda_device)
    full_parity(inp, cuda_device, num_workers=7)


def test_pair_split_reuses_workspace(cuda_device):
    # leftovers of an earlier call on the same workspace, or arbitrary bytes in
    # it, must not change the result
    from mla_paged_latent_decode_b200 import binding
    w = synth.custom_workload(4, 1, 128, [3000, 64, 1900, 700])
    inp = synth.make_inputs(w, seed=12)
    q, kc, bt, sl = (t.to(cuda_device) for t in (inp.q, inp.kcache, inp.block_table, inp.cache_seqlens))
    md, ns = binding.get_mla_metadata(sl, inp.h_q, inp.s_q, 40)
    assert int(ns[-1].item()) > inp.batch  # some sequence is split
    ws = torch.full((binding.workspace_size(inp.batch, inp.s_q, inp.h_q, 40),), 0xFF,
                    dtype=torch.uint8, device=cuda_device)
    outs = []
    for _ in range(3):
        out, lse = binding.mla_decode_kvcache(q, kc, bt, sl, 512, md, ns, inp.scale, inp.causal,
                                              workspace=ws)
        torch.cuda.synchronize(cuda_device)
        outs.append((out.float().cpu().numpy(), lse.cpu().numpy()))
    for o, l in outs[1:]:
        np.testing.assert_array_equal(o, outs[0][0])
        np.testing.assert_array_equal(l, outs[0][1])
    full_parity(inp, cuda_device, num_workers=40)


def test_empty_and_degenerate_sequences(cuda_device):
    # L = 0 (nothing visible), L = 1 < s_q (first query empty under causal), exact pages
    w = synth.custom_workload(5, 2, 16, [0, 1, 64, 128, 2], causal=True)
    inp = synth.make_inputs(w, seed=3)
    res, ref_out, ref_lse = full_parity(inp, cuda_device)
    assert np.all(res["out"][0] == 0) and np.all(np.isneginf(res["lse"][0]))
    assert np.all(res["out"][1, 0] == 0) and np.all(np.isneginf(res["lse"][1, :, 0]))


def test_poisoned_tails_and_pad_pages(cuda_device):
    w = synth.custom_workload(4, 2, 128, [37, 130, 64, 300], causal=True)
    inp = synth.make_inputs(w, seed=5, poison=True)
    full_parity(inp, cuda_device)
    full_parity(inp, cuda_device, num_workers=50)


def test_page_permutation_bit_exact(cuda_device):
    w = synth.custom_workload(3, 1, 128, [500, 64, 1000])
    inp = synth.make_inputs(w, seed=9)
    a = run_cuda(inp, cuda_device)
    nb = inp.kcache.shape[0]
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(1))
    moved = torch.empty_like(inp.kcache)
    moved[perm] = inp.kcache
    inp.kcache = moved
    inp.block_table = perm[inp.block_table.long()].to(torch.int32)
    b = run_cuda(inp, cuda_device)
    np.testing.assert_array_equal(a["out"], b["out"])
    np.testing.assert_array_equal(a["lse"], b["lse"])


def test_dominant_key_and_large_logits(cuda_device):
    # a key whose logit dominates by ~74 must be selected exactly; logits far
    # above the rescale threshold exercise the running-max correction
    L = 4000
    w = synth.custom_workload(2, 1, 64, [L, L])
    inp = synth.make_inputs(w, seed=11)
    inp.q[..., 575] = 1.0
    inp.kcache[..., 575] = 0.0
    for i, t_star in enumerate([3900, 17]):
        page = int(inp.block_table[i, t_star // 64])
        inp.kcache[page, t_star % 64, 575] = 1024.0
    # growing logits along the sequence force repeated rescales
    for t in range(0, L, 64):
        page = int(inp.block_table[1, t // 64])
        inp.kcache[page, :, 574] = float(t) / 16.0
    inp.q[1, :, :, 574] = 1.0
    full_parity(inp, cuda_device)


@pytest.mark.parametrize("name", ["dsv3_decode", "varlen_h16", "spec_causal", "skewed_long"])
def test_full_size_workloads(cuda_device, name):
    # every element of out and lse, in the launch configuration the benchmark times
    inp = synth.make_inputs(name, seed=0)
    full_size_parity(inp, cuda_device)


def test_default_workers_match_formula(cuda_device):
    from mla_paged_latent_decode_b200 import binding
    sms = torch.cuda.get_device_properties(cuda_device).multi_processor_count
    for s_q, h_q in [(1, 16), (1, 64), (1, 1), (1, 128), (2, 128), (4, 128), (3, 64)]:
        nw, stride = binding.metadata_shape(8, h_q, s_q)
        assert stride == 8
        if s_q * h_q <= 64:
            assert nw == sms
        else:
            # pairs: never more than fit on the device at once, and at most SMs / 2 per block
            assert 1 <= nw <= expected_workers(cuda_device, s_q, h_q)
            assert nw >= expected_workers(cuda_device, s_q, h_q) // 2


def test_metadata_bit_exact_many_shapes(cuda_device):
    from mla_paged_latent_decode_b200 import binding
    g = torch.Generator().manual_seed(0)
    for b in (1, 2, 7, 128, 1000, 3000):
        lens = torch.randint(0, 20000, (b,), generator=g, dtype=torch.int32)
        lens[::5] = 0
        sl = lens.to(cuda_device)
        # both per-sequence costs: single-CTA rows (16 heads) and CTA-pair rows (128)
        for h_q in (16, 128) if b <= 1000 else (16,):
            for W in (1, 5, 74, 148, 2000):
                tile_md, num_splits = binding.get_mla_metadata(sl, h_q, 1, W)
                torch.cuda.synchronize()
                res = {"tile_md": tile_md.cpu(), "num_splits": num_splits.cpu()}

                class _I:
                    cache_seqlens = lens
                    s_q = 1
                _I.h_q = h_q
                check_metadata(_I, res, W)


def test_host_validation_rejects_bad_arguments(cuda_device):
    from mla_paged_latent_decode_b200 import binding
    inp = synth.make_inputs("tiny", seed=0)
    q = inp.q.to(cuda_device)
    kc = inp.kcache.to(cuda_device)
    bt = inp.block_table.to(cuda_device)
    sl = inp.cache_seqlens.to(cuda_device)
    md, ns = binding.get_mla_metadata(sl, inp.h_q, inp.s_q)
    with pytest.raises(binding.MLAError) as e:
        binding.mla_decode_kvcache(q, kc, bt, sl, 256, md, ns, inp.scale)
    assert e.value.code == binding.MLA_ERR_UNSUPPORTED
    small_ws = torch.empty(16, dtype=torch.uint8, device=cuda_device)
    with pytest.raises(binding.MLAError) as e:
        binding.mla_decode_kvcache(q, kc, bt, sl, 512, md, ns, inp.scale, workspace=small_ws)
    assert e.value.code == binding.MLA_ERR_INVALID_ARG


def test_overlong_sequence_is_reported_not_read(cuda_device):
    # a length beyond the block-table row is flagged on the device; the kernel
    # reads no entry past the row
    w = synth.custom_workload(2, 1, 16, [100, 64])
    inp = synth.make_inputs(w, seed=2)
    inp.cache_seqlens[1] = 64 * inp.block_table.shape[1] + 50
    res = run_cuda(inp, cuda_device)
    from mla_paged_latent_decode_b200 import binding
    assert res["status"] == binding.MLA_ERR_DEVICE_CHECK


@pytest.mark.parametrize("h_q", [16, 128])
def test_large_batch_of_short_sequences(cuda_device, h_q):
    # many more sequences than workers: every worker runs many pieces, the
    # scheduler's worker rows span thousands of sequences
    g = torch.Generator().manual_seed(5)
    b = 3000 if h_q == 16 else 600
    lens = torch.randint(0, 300, (b,), generator=g).tolist()
    w = synth.custom_workload(b, 1, h_q, lens)
    inp = synth.make_inputs(w, seed=81)
    full_parity(inp, cuda_device)
