"""mla_decode_kvcache_static_scratch: the decode for callers that cannot allocate.

Some callers cannot call cudaMalloc (an engine that owns all device memory in
its own arena, a loop that must never allocate or free), so they cannot hand
mla_decode_kvcache a workspace for split partials.  The static-scratch entry
point uses a fixed array inside the library instead.  These tests call it
through the C ABI and check that it gives bit for bit the results of the
ordinary entry point (both run the same kernels on the same split plan), and
the oracle's within the decode's tolerance, over several calls in a row: each
call finds the previous call's partials still in the shared array, including
a call with more pieces than the one after it.  A workspace larger than the
array is refused before anything runs.

The file name sorts last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from mla_paged_latent_decode_b200 import binding, synth
from parity import assert_close_lse, assert_close_out

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _static_call(inp, q, kc, bt, sl, md, ns, out, lse, status):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return binding.lib.mla_decode_kvcache_static_scratch(
        _p(q), _p(kc), kc.shape[0], _p(bt), bt.shape[1], _p(sl), inp.batch, inp.s_q, inp.h_q,
        576, 512, float(inp.scale), int(inp.causal), _p(md), _p(ns), md.shape[0], _p(out),
        _p(lse), _p(status), stream)


def test_static_scratch_matches_ordinary_entry_point(cuda_device):
    cases = [
        (synth.custom_workload(4, 2, 128, [700, 1, 3000, 64], causal=True), 20, 31),
        (synth.custom_workload(6, 1, 16, [5000, 90, 0, 4100, 64, 777]), 40, 32),
        # many more pieces than the calls before and after it leave in the array
        (synth.custom_workload(3, 1, 128, [2900, 4000, 1500]), 74, 33),
    ]
    # the first case again at the end: it reads an array that a call with more
    # pieces has just filled
    for w, num_workers, seed in cases + cases[:1]:
        inp = synth.make_inputs(w, seed=seed)
        q, kc = inp.q.to(cuda_device), inp.kcache.to(cuda_device)
        bt, sl = inp.block_table.to(cuda_device), inp.cache_seqlens.to(cuda_device)
        md, ns = binding.get_mla_metadata(sl, inp.h_q, inp.s_q, num_workers)
        ref_out, ref_lse = binding.mla_decode_kvcache(q, kc, bt, sl, 512, md, ns, inp.scale,
                                                      inp.causal)
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
        rc = _static_call(inp, q, kc, bt, sl, md, ns, out, lse, status)
        assert rc == binding.MLA_OK, binding.error_string(rc)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert int(ns[-1].item()) > inp.batch, "the case must split sequences to use the scratch"
        # same kernels, same plan: the same bits
        assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))
        assert torch.equal(lse.view(torch.int32), ref_lse.view(torch.int32))
        want_out, want_lse = oracle.decode(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens,
                                           inp.scale, inp.causal)
        assert_close_out(out.float().cpu().numpy(), want_out, "static-scratch out")
        assert_close_lse(lse.cpu().numpy(), want_lse, "static-scratch lse")


def test_static_scratch_refuses_oversized_workspace(cuda_device):
    # 1024 sequences x 128 heads need ~290 MB of partials with 74 workers: more
    # than the 48 MiB array, so the call must fail before launching anything.
    b, s_q, h_q, nw = 1024, 1, 128, 74
    assert binding.workspace_size(b, s_q, h_q, nw) > binding.STATIC_SCRATCH_BYTES
    dummy = torch.zeros(64, dtype=torch.int32, device=cuda_device)
    v = ctypes.c_void_p(dummy.data_ptr())
    rc = binding.lib.mla_decode_kvcache_static_scratch(
        v, v, 1, v, 1, v, b, s_q, h_q, 576, 512, 0.07, 0, v, v, nw, v, v, ctypes.c_void_p(0),
        ctypes.c_void_p(0))
    assert rc == binding.MLA_ERR_SCRATCH_LIMIT
    assert "static scratch" in binding.error_string(rc)
