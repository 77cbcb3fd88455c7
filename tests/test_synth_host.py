"""Host-side input generators and work accounting (no GPU): the seeded sparse
index lists and the algorithmic bytes and flops the benchmark divides by."""
import numpy as np
import torch

from oracle import sparse
from mla_paged_latent_decode_b200 import synth


def test_sparse_indices_are_distinct_in_range_and_seeded():
    w = synth.custom_workload(4, 2, 16, [0, 5, 300, 4000], causal=True)
    inp = synth.make_inputs(w, seed=3)
    idx = synth.make_sparse_indices(inp, 256, seed=9)
    assert idx.dtype == torch.int32 and tuple(idx.shape) == (4, 2, 256)
    for i, L in enumerate(inp.cache_seqlens.tolist()):
        for j in range(2):
            row = idx[i, j]
            picked = row[row >= 0].tolist()
            assert len(picked) == min(256, L)
            assert len(set(picked)) == len(picked) and all(0 <= t < L for t in picked)
            assert torch.all(row[len(picked):] == -1)
    assert torch.equal(idx, synth.make_sparse_indices(inp, 256, seed=9))
    assert not torch.equal(idx, synth.make_sparse_indices(inp, 256, seed=10))


def test_sparse_padding_replaces_entries():
    inp = synth.make_inputs(synth.custom_workload(2, 1, 16, [500, 500]), seed=1)
    idx = synth.make_sparse_indices(inp, 200, seed=2, pad_frac=0.3)
    bad = (idx < 0) | (idx >= 500)
    frac = float(bad.float().mean())
    assert 0.15 < frac < 0.45
    assert bool(((idx == -1) | (idx == (1 << 30)) | ((idx >= 0) & (idx < 500))).all())


def test_sparse_work_counts_the_used_entries():
    w = synth.custom_workload(3, 2, 8, [10, 200, 64], causal=True)
    inp = synth.make_inputs(w, seed=4)
    idx = synth.make_sparse_indices(inp, 100, seed=5, pad_frac=0.25)
    nbytes, flops = synth.sparse_algorithmic_work(inp, idx)
    used = sum(len(sparse.used_entries(idx[i, j].tolist(), L, 2, j, True))
               for i, L in enumerate(inp.cache_seqlens.tolist()) for j in range(2))
    assert flops == 2 * (576 + 512) * 8 * used
    fixed = 3 * 2 * 8 * (576 * 2 + 512 * 2) + 3 * 8 * 2 * 4 + idx.numel() * 4
    assert nbytes == used * 1152 + fixed


def test_dense_work_with_fp8_row_bytes():
    inp = synth.make_inputs("tiny", seed=0)
    b16, f16 = synth.algorithmic_work(inp)
    b8, f8 = synth.algorithmic_work(inp, 580)
    total = int(inp.cache_seqlens.sum())
    assert f8 == f16 and b16 - b8 == total * (1152 - 580)
    # 167 cached rows, q in, out and lse out, 2 lengths and 1 + 3 block-table entries
    assert b16 == 167 * 1152 + 2 * 16 * 576 * 2 + 2 * 16 * 512 * 2 + 2 * 16 * 4 + 4 * (2 + 4)
    assert f16 == 2 * 1088 * 16 * 167
