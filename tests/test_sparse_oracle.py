"""Pins for the CPU statement of sparse (top-k) decoding (oracle/sparse.py),
without a GPU.

The defining property is checked directly: attending over a list of selected
tokens equals the dense decode (the pinned C oracle) over a sequence made of
exactly those cached rows.  Around it: the full list in order is the dense
decode, the list's order and padding entries do not matter, one token gives its
value row, an empty list gives zero and -inf, and planted mistakes fail.
"""
import importlib.util

import numpy as np
import pytest
import torch

import oracle
from oracle import sparse
from mla_paged_latent_decode_b200 import synth

PAGE = 64


def compacted(inp, rows_per_seq):
    """A cache and block table whose sequence i is exactly rows_per_seq[i]
    (lists of (page, slot) cached rows, in order), with fresh pages."""
    b = inp.batch
    n_pages = [max(1, -(-len(r) // PAGE)) for r in rows_per_seq]
    kc = torch.zeros((sum(n_pages), PAGE, 576), dtype=torch.bfloat16)
    bt = torch.zeros((b, max(n_pages)), dtype=torch.int32)
    cur = 0
    for i, rows in enumerate(rows_per_seq):
        for k, (pg, sl) in enumerate(rows):
            kc[cur + k // PAGE, k % PAGE] = inp.kcache[pg, sl]
        bt[i, :n_pages[i]] = torch.arange(cur, cur + n_pages[i], dtype=torch.int32)
        cur += n_pages[i]
    lens = torch.tensor([len(r) for r in rows_per_seq], dtype=torch.int32)
    return kc, bt, lens


def phys(inp, i, t):
    return int(inp.block_table[i, t // PAGE]), t % PAGE


@pytest.mark.parametrize("s_q,causal", [(1, False), (2, False), (2, True), (3, True)])
def test_full_list_is_the_dense_decode(s_q, causal):
    w = synth.custom_workload(3, s_q, 4, [5, 64, 130], causal=causal)
    inp = synth.make_inputs(w, seed=41)
    L = int(inp.cache_seqlens.max())
    idx = torch.full((3, s_q, L), -1, dtype=torch.int32)
    for i, Li in enumerate(inp.cache_seqlens.tolist()):
        idx[i, :, :Li] = torch.arange(Li, dtype=torch.int32)
    out, lse = sparse.decode(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens, idx,
                             inp.scale, causal)
    ref_out, ref_lse = oracle.decode(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens,
                                     inp.scale, causal)
    np.testing.assert_allclose(out, ref_out, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("seed", range(4))
def test_selection_equals_dense_decode_of_the_selected_rows(seed):
    g = np.random.default_rng(seed)
    w = synth.custom_workload(3, 1, 8, [300, 70, 129])
    inp = synth.make_inputs(w, seed=50 + seed)
    topk = 40
    idx = torch.full((3, 1, topk), -1, dtype=torch.int32)
    chosen = []
    for i, L in enumerate(inp.cache_seqlens.tolist()):
        k = int(g.integers(1, min(L, topk) + 1))
        sel = g.choice(L, size=k, replace=False)
        if seed == 3:  # a repeated token counts once per occurrence
            sel = np.concatenate([sel[:-1], sel[:1]]) if k > 1 else sel
        idx[i, 0, :len(sel)] = torch.from_numpy(sel.astype(np.int32))
        chosen.append([phys(inp, i, int(t)) for t in sel])
    out, lse = sparse.decode(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens, idx,
                             inp.scale, False)
    kc, bt, lens = compacted(inp, chosen)
    ref_out, ref_lse = oracle.decode(inp.q, kc, bt, lens, inp.scale, False)
    np.testing.assert_allclose(out, ref_out, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-14)


def test_order_and_padding_do_not_matter():
    g = np.random.default_rng(7)
    w = synth.custom_workload(2, 2, 4, [200, 90], causal=True)
    inp = synth.make_inputs(w, seed=60)
    idx = torch.from_numpy(g.integers(0, 90, size=(2, 2, 24)).astype(np.int32))
    out, lse = sparse.decode(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens, idx,
                             inp.scale, True)
    perm = torch.from_numpy(g.permutation(24))
    padded = torch.cat([idx[:, :, perm], torch.full((2, 2, 9), -1, dtype=torch.int32),
                        torch.full((2, 2, 3), 100000, dtype=torch.int32)], dim=2)
    out2, lse2 = sparse.decode(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens, padded,
                               inp.scale, True)
    np.testing.assert_allclose(out2, out, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse2, lse, rtol=1e-12, atol=1e-14)


def test_one_token_and_no_token():
    w = synth.custom_workload(2, 1, 4, [100, 100])
    inp = synth.make_inputs(w, seed=61)
    idx = torch.tensor([[[37, -1]], [[-1, -1]]], dtype=torch.int32)
    out, lse = sparse.decode(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens, idx,
                             inp.scale, False)
    pg, sl = phys(inp, 0, 37)
    row = inp.kcache[pg, sl].double().numpy()
    for h in range(4):
        np.testing.assert_array_equal(out[0, 0, h], row[:512])
        s = inp.scale * float(inp.q[0, 0, h].double().numpy() @ row)
        assert abs(lse[0, h, 0] - s) <= 1e-12 * max(1.0, abs(s))
    assert not out[1].any() and np.all(np.isneginf(lse[1]))


def test_causal_limit_per_query_position():
    # s_q = 3, L = 10: query j sees t <= 7 + j; index 9 is used by j = 2 only
    w = synth.custom_workload(1, 3, 2, [10], causal=True)
    inp = synth.make_inputs(w, seed=62)
    idx = torch.tensor([[[9, 8, 3], [9, 8, 3], [9, 8, 3]]], dtype=torch.int32)
    out, lse = sparse.decode(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens, idx,
                             inp.scale, True)
    assert sparse.used_entries([9, 8, 3], 10, 3, 0, True) == [3]
    assert sparse.used_entries([9, 8, 3], 10, 3, 1, True) == [8, 3]
    assert sparse.used_entries([9, 8, 3], 10, 3, 2, True) == [9, 8, 3]
    pg, sl = phys(inp, 0, 3)
    np.testing.assert_array_equal(out[0, 0, 0], inp.kcache[pg, sl].double().numpy()[:512])


MUTATIONS = {
    "causal_off_by_one": ("limit = L - s_q + j + 1 if causal else L",
                          "limit = L - s_q + j if causal else L"),
    "slot_wrong": ("kd[bt[i, t // PAGE], t % PAGE]", "kd[bt[i, t // PAGE], t // PAGE]"),
    "value_dims_wrong": ("@ rows[:, :D_V]", "@ rows[:, D_QK - D_V:]"),
    "scale_dropped": ("logits = scale * (qd[i, j] @ rows.T)", "logits = (qd[i, j] @ rows.T)"),
    "padding_used": ("if 0 <= int(t) < limit", "if int(t) < limit"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_reject_mutation(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(sparse.__file__).read()
    assert src.count(old) == 1, old
    path = tmp_path / f"mut_{name}.py"
    path.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"mut_{name}", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    saved = sparse.decode, sparse.used_entries
    sparse.decode, sparse.used_entries = mod.decode, mod.used_entries
    try:
        failed = False
        try:
            test_full_list_is_the_dense_decode(2, True)
            for seed in range(4):
                test_selection_equals_dense_decode_of_the_selected_rows(seed)
            test_order_and_padding_do_not_matter()
            test_one_token_and_no_token()
        except (AssertionError, IndexError):
            failed = True
        assert failed, f"mutation {name} went undetected"
    finally:
        sparse.decode, sparse.used_entries = saved
