"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
and compare it with the fp64 oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from oracle import scheduler

# Tolerances of the decode: bf16 outputs, fp32 lse (natural log).
OUT_ATOL = 1e-2
OUT_RTOL = 1e-2
LSE_ATOL = 1e-3


def to_device(inp, dev):
    return (inp.q.to(dev), inp.kcache.to(dev), inp.block_table.to(dev), inp.cache_seqlens.to(dev))


def run_cuda(inp, dev, num_workers=None, with_status=True):
    from mla_paged_latent_decode_b200 import binding
    q, kc, bt, sl = to_device(inp, dev)
    tile_md, num_splits = binding.get_mla_metadata(sl, inp.h_q, inp.s_q, num_workers)
    status = torch.zeros(1, dtype=torch.int32, device=dev) if with_status else None
    out, lse = binding.mla_decode_kvcache(q, kc, bt, sl, 512, tile_md, num_splits, inp.scale,
                                          inp.causal, device_status=status)
    torch.cuda.synchronize(dev)
    res = dict(out=out.float().cpu().numpy(), lse=lse.cpu().numpy(), tile_md=tile_md.cpu(),
               num_splits=num_splits.cpu())
    if with_status:
        res["status"] = int(status.item())
    return res


def expected_workers(dev, s_q, h_q):
    props = torch.cuda.get_device_properties(dev)
    return scheduler.num_workers_for(props.multi_processor_count, s_q, h_q)


def check_metadata(inp, res, num_workers):
    md, ns = scheduler.split_plan(inp.cache_seqlens.tolist(), num_workers,
                                  scheduler.piece_cost_for(inp.s_q, inp.h_q))
    np.testing.assert_array_equal(res["tile_md"].numpy(), np.asarray(md, dtype=np.int32))
    np.testing.assert_array_equal(res["num_splits"].numpy(), np.asarray(ns, dtype=np.int32))


def assert_close_out(got, ref, where=""):
    err = np.abs(got - ref)
    bound = OUT_ATOL + OUT_RTOL * np.abs(ref)
    bad = err > bound
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{where}: {int(bad.sum())} of {bad.size} outputs out of tolerance; "
                             f"max err {err.max():.3e}; first {idx.tolist()} "
                             f"got {got[tuple(idx[0])]:.5f} ref {ref[tuple(idx[0])]:.5f}")


def assert_close_lse(got, ref, where=""):
    both_inf = np.isneginf(got) & np.isneginf(ref)
    with np.errstate(invalid="ignore"):
        diff = np.where(both_inf, 0.0, np.abs(got - ref))
    if not np.all(diff <= LSE_ATOL):
        raise AssertionError(f"{where}: lse max err {np.nanmax(diff):.3e} "
                             f"(neg-inf mismatch: {int((np.isneginf(got) != np.isneginf(ref)).sum())})")


def workers_used(res, dev, inp, num_workers):
    W = int(res["tile_md"].shape[0])
    if num_workers is not None:
        assert W == num_workers
    else:
        assert 1 <= W <= expected_workers(dev, inp.s_q, inp.h_q)
    return W


def full_parity(inp, dev, num_workers=None):
    res = run_cuda(inp, dev, num_workers)
    assert res["status"] == 0, f"device status {res['status']}"
    W = workers_used(res, dev, inp, num_workers)
    check_metadata(inp, res, W)
    ref_out, ref_lse = oracle.decode(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens,
                                     inp.scale, inp.causal)
    assert_close_out(res["out"], ref_out, "out")
    assert_close_lse(res["lse"], ref_lse, "lse")
    return res, ref_out, ref_lse


def full_size_parity(inp, dev):
    """Full-size run in the default launch configuration (the one the benchmark
    times), every output element and every lse compared with the oracle."""
    res = run_cuda(inp, dev)
    assert res["status"] == 0, f"device status {res['status']}"
    W = workers_used(res, dev, inp, None)
    check_metadata(inp, res, W)
    ref_out, ref_lse = oracle.decode(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens,
                                     inp.scale, inp.causal)
    assert_close_out(res["out"], ref_out, "out")
    assert_close_lse(res["lse"], ref_lse, "lse")
    return res
