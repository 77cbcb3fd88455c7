"""GPU parity of the FP8 latent cache: the quantising append and the decode over
E4M3 codes with per-token scales, through the C ABI, against the oracle.

- Append: bit-exact.  The codes and scale of every token a sequence can see,
  the lengths, the free count and the block-table entries must equal the CPU
  statement (oracle/fp8_cache.py encodes the rows, oracle/paged_cache.py does
  the bookkeeping).
- Decode: the decode oracle on the dequantised cache (code * scale, exact in
  bf16), within the decode's tolerance: |out - ref| <= 1e-2 + 1e-2 |ref|,
  |lse - ref| <= 1e-3.  Split metadata bit-exact as for the bf16 cache.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import fp8_cache as f8
from oracle import paged_cache as pc
from mla_paged_latent_decode_b200 import synth
from parity import (assert_close_lse, assert_close_out, check_metadata, expected_workers)

pytestmark = pytest.mark.gpu

PAGE = 64


def encode_cache(kcache_bf16, pages_per_block=128):
    """Oracle encoding of a whole bf16 cache: (codes uint8 [nblk, 64, 576], scales fp32)."""
    nblk = kcache_bf16.shape[0]
    codes = torch.empty((nblk, PAGE, 576), dtype=torch.uint8)
    scales = torch.empty((nblk, PAGE), dtype=torch.float32)
    for p0 in range(0, nblk, pages_per_block):
        c, s = f8.encode_rows(kcache_bf16[p0:p0 + pages_per_block].double().numpy())
        codes[p0:p0 + pages_per_block] = torch.from_numpy(c)
        scales[p0:p0 + pages_per_block] = torch.from_numpy(s.astype(np.float32))
    return codes, scales


def dequantized(codes, scales, pages_per_block=128):
    """code * scale for the whole cache, as bf16 (checked exact)."""
    out = torch.empty(codes.shape, dtype=torch.bfloat16)
    for p0 in range(0, codes.shape[0], pages_per_block):
        t = torch.from_numpy(f8.dequantize(codes[p0:p0 + pages_per_block].numpy(),
                                           scales[p0:p0 + pages_per_block].double().numpy()))
        b = t.to(torch.bfloat16)
        assert torch.equal(b.double(), t), "dequantised cache not exact in bf16"
        out[p0:p0 + pages_per_block] = b
    return out


def run_fp8(inp, codes, scales, dev, num_workers=None):
    from mla_paged_latent_decode_b200 import binding
    q, bt, sl = inp.q.to(dev), inp.block_table.to(dev), inp.cache_seqlens.to(dev)
    md, ns = binding.get_mla_metadata(sl, inp.h_q, inp.s_q, num_workers)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    out, lse = binding.mla_decode_kvcache_fp8(q, codes.to(dev), scales.to(dev), bt, sl, 512, md,
                                              ns, inp.scale, inp.causal, device_status=status)
    torch.cuda.synchronize(dev)
    assert int(status.item()) == 0
    return out.float().cpu().numpy(), lse.cpu().numpy(), md.cpu(), ns.cpu()


@pytest.mark.parametrize("h_q,s_q,causal", [(16, 1, False), (1, 1, False), (32, 2, True),
                                             (64, 1, False), (16, 4, True)])
def test_fp8_decode_small(cuda_device, h_q, s_q, causal):
    w = synth.custom_workload(4, s_q, h_q, [1, 63, 130, 257], causal=causal)
    inp = synth.make_inputs(w, seed=300 + h_q + s_q)
    codes, scales = encode_cache(inp.kcache)
    out, lse, md, ns = run_fp8(inp, codes, scales, cuda_device)
    check_metadata(inp, dict(tile_md=md, num_splits=ns), md.shape[0])
    ref_out, ref_lse = oracle.decode(inp.q, dequantized(codes, scales), inp.block_table,
                                     inp.cache_seqlens, inp.scale, inp.causal)
    assert_close_out(out, ref_out, "fp8 out")
    assert_close_lse(lse, ref_lse, "fp8 lse")


@pytest.mark.parametrize("h_q,s_q,causal", [(128, 1, False), (128, 2, True), (96, 1, False),
                                             (64, 3, True)])
def test_fp8_decode_more_than_64_rows(cuda_device, h_q, s_q, causal):
    # several 64-row blocks per worker, a last block with some or no valid rows
    w = synth.custom_workload(4, s_q, h_q, [1, 63, 700, 1300], causal=causal)
    inp = synth.make_inputs(w, seed=310 + h_q + s_q)
    codes, scales = encode_cache(inp.kcache)
    for nw in (None, 5):
        out, lse, md, ns = run_fp8(inp, codes, scales, cuda_device, nw)
        check_metadata(inp, dict(tile_md=md, num_splits=ns), md.shape[0])
        ref_out, ref_lse = oracle.decode(inp.q, dequantized(codes, scales), inp.block_table,
                                         inp.cache_seqlens, inp.scale, inp.causal)
        assert_close_out(out, ref_out, "fp8 out")
        assert_close_lse(lse, ref_lse, "fp8 lse")


@pytest.mark.parametrize("name", ["dsv3_decode", "spec_causal", "skewed_long"])
def test_fp8_full_size_128_heads(cuda_device, name):
    # the 128-head configurations over their FP8 caches, default launch
    # configuration, every element against the oracle on the dequantised cache
    inp = synth.make_inputs(name, seed=0)
    codes, scales = encode_cache(inp.kcache)
    out, lse, md, ns = run_fp8(inp, codes, scales, cuda_device)
    check_metadata(inp, dict(tile_md=md, num_splits=ns), md.shape[0])
    ref_out, ref_lse = oracle.decode(inp.q, dequantized(codes, scales), inp.block_table,
                                     inp.cache_seqlens, inp.scale, inp.causal)
    assert_close_out(out, ref_out, "fp8 out")
    assert_close_lse(lse, ref_lse, "fp8 lse")


@pytest.mark.parametrize("num_workers,h_q", [(1, 16), (3, 16), (17, 16), (600, 16), (2, 128),
                                             (9, 128), (74, 128)])
def test_fp8_decode_forced_splits(cuda_device, num_workers, h_q):
    w = synth.custom_workload(3, 2, h_q, [700, 5, 1100], causal=True)
    inp = synth.make_inputs(w, seed=31)
    codes, scales = encode_cache(inp.kcache)
    out, lse, md, ns = run_fp8(inp, codes, scales, cuda_device, num_workers)
    ref_out, ref_lse = oracle.decode(inp.q, dequantized(codes, scales), inp.block_table,
                                     inp.cache_seqlens, inp.scale, inp.causal)
    assert_close_out(out, ref_out, "fp8 out")
    assert_close_lse(lse, ref_lse, "fp8 lse")


@pytest.mark.parametrize("h_q", [16, 128])
def test_fp8_decode_ignores_stale_tail_rows(cuda_device, h_q):
    # rows past each sequence's end hold NaN codes and infinite scales: the
    # kernels must never let them reach an output (16 heads: single CTAs; 128
    # heads: CTA pairs)
    w = synth.custom_workload(3, 1, h_q, [37, 64, 100])
    inp = synth.make_inputs(w, seed=32)
    codes, scales = encode_cache(inp.kcache)
    ref_out, ref_lse = oracle.decode(inp.q, dequantized(codes, scales), inp.block_table,
                                     inp.cache_seqlens, inp.scale, False)
    for i, L in enumerate(inp.cache_seqlens.tolist()):
        n = synth.pages_for(L)
        tail = L - (n - 1) * PAGE
        if tail < PAGE:
            page = int(inp.block_table[i, n - 1])
            codes[page, tail:] = 0x7F
            scales[page, tail:] = float("inf")
    out, lse, _, _ = run_fp8(inp, codes, scales, cuda_device)
    assert np.all(np.isfinite(out))
    assert_close_out(out, ref_out, "fp8 out")
    assert_close_lse(lse, ref_lse, "fp8 lse")


def test_fp8_single_token_is_exact(cuda_device):
    """With one cached token the output is that token's value row exactly
    (weight 1, bf16 output of a bf16-exact value).  The row holds every finite
    E4M3 code, subnormals and both zeros included, under scales from 2^-124 to
    2^60: the kernel's widening must reproduce code * scale bit for bit."""
    finite = [c for c in range(256) if c not in (0x7F, 0xFF)]
    ks = [-124, -30, -7, 0, 7, 30, 60]
    b = len(ks)
    w = synth.custom_workload(b, 1, 16, [1] * b)
    inp = synth.make_inputs(w, seed=34)
    codes = torch.zeros((inp.kcache.shape[0], PAGE, 576), dtype=torch.uint8)
    scales = torch.ones((inp.kcache.shape[0], PAGE), dtype=torch.float32)
    for i, k in enumerate(ks):
        page = int(inp.block_table[i, 0])
        row = [finite[(c + 37 * i) % len(finite)] for c in range(576)]
        codes[page, 0] = torch.tensor(row, dtype=torch.uint8)
        scales[page, 0] = 2.0 ** k
    out, lse, _, _ = run_fp8(inp, codes, scales, cuda_device)
    want = dequantized(codes, scales)
    for i in range(b):
        page = int(inp.block_table[i, 0])
        v = want[page, 0, :512].float().numpy()
        for h in range(16):
            np.testing.assert_array_equal(out[i, 0, h], v)


def test_fp8_decode_dominant_key(cuda_device):
    # one key far above the rest: the output is that token's dequantised value row
    w = synth.custom_workload(2, 1, 16, [200, 77])
    inp = synth.make_inputs(w, seed=33)
    kc = inp.kcache.clone()
    for i, t in ((0, 150), (1, 3)):
        page = int(inp.block_table[i, t // PAGE])
        kc[page, t % PAGE, 512:] = (inp.q[i, 0, 0, 512:].float() * 40).to(torch.bfloat16)
    codes, scales = encode_cache(kc)
    out, lse, _, _ = run_fp8(inp, codes, scales, cuda_device)
    ref_out, ref_lse = oracle.decode(inp.q, dequantized(codes, scales), inp.block_table,
                                     inp.cache_seqlens, inp.scale, False)
    assert_close_out(out, ref_out, "fp8 out")
    assert_close_lse(lse, ref_lse, "fp8 lse")


def test_fp8_varlen_full_size(cuda_device):
    # the memory-bound variable-length workload (128 sequences, 16 heads,
    # lengths U[1, 8192]) in the default launch configuration; every element
    inp = synth.make_inputs("varlen_h16", seed=0)
    codes, scales = encode_cache(inp.kcache)
    out, lse, md, ns = run_fp8(inp, codes, scales, cuda_device)
    check_metadata(inp, dict(tile_md=md, num_splits=ns), md.shape[0])
    assert md.shape[0] == expected_workers(cuda_device, inp.s_q, inp.h_q)
    ref_out, ref_lse = oracle.decode(inp.q, dequantized(codes, scales), inp.block_table,
                                     inp.cache_seqlens, inp.scale, False)
    assert_close_out(out, ref_out, "fp8 out")
    assert_close_lse(lse, ref_lse, "fp8 lse")


def packed(codes, scales):
    """One byte row per token: 576 codes then the scale's 4 bytes (bookkeeping view)."""
    return np.concatenate([codes, np.ascontiguousarray(scales)[..., None].view(np.uint8)], axis=-1)


@pytest.mark.parametrize("L0,s_new", [((0, 1, 63, 64, 65, 200), 1), ((10, 64, 127), 2),
                                      ((5, 0, 300), 70)])
def test_fp8_append_bit_exact(cuda_device, L0, s_new):
    from mla_paged_latent_decode_b200 import binding
    b = len(L0)
    gen = torch.Generator().manual_seed(sum(L0) + s_new)
    pool = sum(pc.pages_for(L + s_new) for L in L0) + 3
    stride = max(pc.pages_for(L + s_new) for L in L0)
    start_rows = torch.randn((pool, PAGE, 576), generator=gen).to(torch.bfloat16)
    codes0, scales0 = encode_cache(start_rows)
    perm = torch.randperm(pool, generator=gen).to(torch.int32)
    bt = torch.zeros((b, stride), dtype=torch.int32)
    cur = 0
    for i, L in enumerate(L0):
        n = pc.pages_for(L)
        bt[i, :n] = perm[cur:cur + n]
        cur += n
    free = perm[cur:].clone()
    lens = torch.tensor(L0, dtype=torch.int32)
    rows = (torch.randn((b, s_new, 576), generator=gen) *
            torch.logspace(-2, 2, b * s_new, dtype=torch.float32).reshape(b, s_new, 1)).to(
                torch.bfloat16)
    # oracle: encode the new rows, then the bookkeeping over packed byte rows
    rc, rs = f8.encode_rows(rows.double().numpy())
    kc_e, bt_e, lens_e, free_e, fc_e, st = pc.append(
        packed(codes0.numpy(), scales0.numpy()), bt.numpy(), lens.numpy(), free.numpy(),
        len(free), packed(rc, rs.astype(np.float32)))
    assert st == "ok"
    # GPU
    dev = cuda_device
    kc8, ks = codes0.to(dev), scales0.to(dev)
    bt_d, lens_d, free_d = bt.to(dev), lens.to(dev), free.to(dev)
    fc_d = torch.tensor([len(free)], dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    binding.append_latent_fp8(rows.to(dev), kc8, ks, bt_d, lens_d, free_d, fc_d, status)
    torch.cuda.synchronize(dev)
    assert int(status.item()) == 0
    assert lens_d.cpu().tolist() == lens_e.tolist() and int(fc_d.item()) == fc_e
    bt_g = bt_d.cpu().numpy()
    kc_g = packed(kc8.cpu().numpy(), ks.cpu().numpy())
    for i, L in enumerate(lens_e):
        n = pc.pages_for(int(L))
        np.testing.assert_array_equal(bt_g[i, :n], bt_e[i, :n])
        np.testing.assert_array_equal(pc.sequence_rows(kc_g, bt_g, lens_e, i),
                                      pc.sequence_rows(kc_e, bt_e, lens_e, i))


def test_fp8_decode_loop_after_appends(cuda_device):
    """Append this step's rows into the FP8 cache on the GPU, then decode: the
    result matches the decode oracle over the oracle-encoded grown cache."""
    from mla_paged_latent_decode_b200 import binding
    dev = cuda_device
    L0, h_q = [63, 64, 1, 200], 16
    b = len(L0)
    gen = torch.Generator().manual_seed(77)
    pool, stride = 24, 8
    codes0, scales0 = encode_cache(torch.randn((pool, PAGE, 576), generator=gen).to(torch.bfloat16))
    perm = torch.randperm(pool, generator=gen).to(torch.int32)
    bt = torch.zeros((b, stride), dtype=torch.int32)
    cur = 0
    for i, L in enumerate(L0):
        n = pc.pages_for(L)
        bt[i, :n] = perm[cur:cur + n]
        cur += n
    state = dict(kc=packed(codes0.numpy(), scales0.numpy()), bt=bt.numpy(),
                 lens=np.array(L0, dtype=np.int32), free=perm[cur:].numpy().copy(),
                 fc=pool - cur)
    kc8, ks = codes0.to(dev), scales0.to(dev)
    bt_d, lens_d = bt.to(dev), torch.tensor(L0, dtype=torch.int32, device=dev)
    free_d = perm[cur:].to(dev)
    fc_d = torch.tensor([pool - cur], dtype=torch.int32, device=dev)
    for step in range(3):
        rows = torch.randn((b, 1, 576), generator=gen).to(torch.bfloat16)
        rc, rs = f8.encode_rows(rows.double().numpy())
        kc_e, bt_e, lens_e, free_e, fc_e, st = pc.append(
            state["kc"], state["bt"], state["lens"], state["free"], state["fc"],
            packed(rc, rs.astype(np.float32)))
        assert st == "ok"
        state = dict(kc=kc_e, bt=bt_e, lens=lens_e, free=free_e, fc=fc_e)
        binding.append_latent_fp8(rows.to(dev), kc8, ks, bt_d, lens_d, free_d, fc_d)
        q = torch.randn((b, 1, h_q, 576), generator=gen).to(torch.bfloat16)
        md, ns = binding.get_mla_metadata(lens_d, h_q, 1)
        out, lse = binding.mla_decode_kvcache_fp8(q.to(dev), kc8, ks, bt_d, lens_d, 512, md, ns,
                                                  synth.DEFAULT_SCALE, False)
        torch.cuda.synchronize(dev)
        codes_e = torch.from_numpy(np.ascontiguousarray(kc_e[..., :576]))
        scales_e = torch.from_numpy(np.ascontiguousarray(kc_e[..., 576:]).view(np.float32)[..., 0])
        ref_out, ref_lse = oracle.decode(q, dequantized(codes_e, scales_e), torch.from_numpy(bt_e),
                                         torch.from_numpy(lens_e), synth.DEFAULT_SCALE, False)
        assert_close_out(out.float().cpu().numpy(), ref_out, f"step {step} out")
        assert_close_lse(lse.cpu().numpy(), ref_lse, f"step {step} lse")
