"""Pins for the CPU statement of the paged cache's append / allocate / release
(oracle/paged_cache.py), without a GPU.

The pins do not re-run the oracle's own rule.  They check it against a model
with no paging at all (each sequence a plain Python list of rows), against
closed forms (a sequence of L tokens holds ceil(L / 64) pages; pages are
conserved and never shared), against hand-derived small cases, and against the
decode oracle's brute force on the grown sequences.  Planted mistakes in a copy
of the oracle's source must fail them.
"""
import importlib.util
import math
import os
import sys

import numpy as np
import pytest

from oracle import paged_cache as pc

PAGE = 64
SRC = pc.__file__


def fresh_state(lens, pool, stride, seed, d=8):
    """A cache of `pool` pages with sequences of the given lengths on shuffled
    pages and every other page on the free stack (narrow rows keep it fast)."""
    g = np.random.default_rng(seed)
    kcache = g.integers(-1000, 1000, size=(pool, PAGE, d)).astype(np.int32)
    perm = g.permutation(pool).astype(np.int32)
    bt = np.full((len(lens), stride), -1, dtype=np.int32)
    cur = 0
    logical = []
    for i, L in enumerate(lens):
        n = pc.pages_for(L)
        bt[i, :n] = perm[cur:cur + n]
        cur += n
        logical.append([kcache[bt[i, t // PAGE], t % PAGE].copy() for t in range(L)])
    free = np.zeros(pool, dtype=np.int32)
    free[:pool - cur] = perm[cur:]
    return kcache, bt, np.asarray(lens, dtype=np.int32), free, pool - cur, logical


def check_against_model(mod, state, logical):
    kcache, bt, lens, free, fc = state
    pool = kcache.shape[0]
    used = []
    for i, L in enumerate(lens):
        assert int(L) == len(logical[i])
        got = mod.sequence_rows(kcache, bt, lens, i)
        want = np.stack(logical[i]) if logical[i] else np.zeros((0, kcache.shape[2]))
        np.testing.assert_array_equal(got, want)
        used.extend(int(p) for p in bt[i, :math.ceil(int(L) / PAGE)])
    # pages in use are distinct; in use + free is the whole pool, each once
    assert len(used) == len(set(used))
    assert sorted(used + [int(p) for p in free[:fc]]) == list(range(pool))


def random_walk(mod, seed, steps=60):
    g = np.random.default_rng(seed)
    b, pool, stride, d = 5, 40, 12, 8
    kcache, bt, lens, free, fc, logical = fresh_state(
        [int(v) for v in g.integers(0, 200, size=b)], pool, stride, seed, d)
    for _ in range(steps):
        if g.random() < 0.2:
            mask = (g.random(b) < 0.4).astype(np.int32)
            bt, lens, free, fc, st = mod.release(bt, lens, free, fc, mask)
            assert st == "ok"
            for i in range(b):
                if mask[i]:
                    logical[i] = []
        else:
            s_new = int(g.choice([1, 2, 3, 63, 64, 65]))
            rows = g.integers(-1000, 1000, size=(b, s_new, d)).astype(np.int32)
            before = (kcache, bt, lens, free, fc)
            kcache, bt, lens, free, fc, st = mod.append(kcache, bt, lens, free, fc, rows)
            if st == "ok":
                for i in range(b):
                    logical[i].extend(rows[i, k].copy() for k in range(s_new))
            else:
                # nothing changed
                for x, y in zip(before, (kcache, bt, lens, free, fc)):
                    np.testing.assert_array_equal(x, y)
        check_against_model(mod, (kcache, bt, lens, free, fc), logical)


@pytest.mark.parametrize("seed", range(6))
def test_random_appends_and_releases_match_unpaged_model(seed):
    random_walk(pc, seed)


@pytest.mark.parametrize("L", [0, 1, 62, 63, 64, 65, 127, 128, 129])
@pytest.mark.parametrize("s_new", [1, 2, 64, 65, 130])
def test_pages_grow_in_64_token_increments(L, s_new):
    kcache, bt, lens, free, fc, logical = fresh_state([L], 10, 8, seed=L + s_new)
    rows = np.full((1, s_new, 8), 7, dtype=np.int32)
    kcache2, bt2, lens2, free2, fc2, st = pc.append(kcache, bt, lens, free, fc, rows)
    assert st == "ok"
    # closed form: new pages = ceil((L + s) / 64) - ceil(L / 64)
    new_pages = -(-(L + s_new) // 64) - -(-L // 64)
    assert fc - fc2 == new_pages
    assert int(lens2[0]) == L + s_new
    # the rows before L are untouched, the new ones are all 7
    rows_now = pc.sequence_rows(kcache2, bt2, lens2, 0)
    if L:
        np.testing.assert_array_equal(rows_now[:L], np.stack(logical[0]))
    assert np.all(rows_now[L:] == 7)


def test_hand_derived_pops_and_pushes():
    # pool of 8 pages; seq 0 holds page 3 fully (64 tokens), seq 1 is empty,
    # seq 2 holds 10 tokens on page 1.  Free stack bottom..top = [0, 2, 4, 5, 6, 7].
    kcache = np.zeros((8, PAGE, 1), dtype=np.int32)
    bt = np.array([[3, -1], [-1, -1], [1, -1]], dtype=np.int32)
    lens = np.array([64, 0, 10], dtype=np.int32)
    free = np.array([0, 2, 4, 5, 6, 7, 0, 0], dtype=np.int32)
    rows = np.array([[[11]], [[22]], [[33]]], dtype=np.int32)
    kc, bt2, lens2, free2, fc, st = pc.append(kcache, bt, lens, free, 6, rows)
    # seq 0 crosses into its second page and pops 7; seq 1 needs its first page
    # and pops 6; seq 2 still fits in page 1
    assert st == "ok" and fc == 4
    assert bt2.tolist() == [[3, 7], [6, -1], [1, -1]]
    assert lens2.tolist() == [65, 1, 11]
    assert kc[7, 0, 0] == 11 and kc[6, 0, 0] == 22 and kc[1, 10, 0] == 33
    assert int(np.count_nonzero(kc)) == 3
    # releasing seqs 0 and 2 pushes 3, 7, then 1 on top of [0, 2, 4, 5]
    bt3, lens3, free3, fc3, st = pc.release(bt2, lens2, free2, fc, np.array([1, 0, 1]))
    assert st == "ok" and fc3 == 7
    assert free3[:7].tolist() == [0, 2, 4, 5, 3, 7, 1]
    assert lens3.tolist() == [0, 1, 0]
    # the next page popped is the last one pushed
    kc4, bt4, lens4, _, fc4, st = pc.append(kc, bt3, lens3, free3, fc3,
                                            np.array([[[1]], [[2]], [[3]]], dtype=np.int32))
    assert st == "ok" and fc4 == 5
    assert bt4[0, 0] == 1 and bt4[2, 0] == 7 and bt4[1, 0] == 6


@pytest.mark.parametrize("case", ["too_few_pages", "row_too_short", "negative_length",
                                  "bad_free_page", "bad_last_page"])
def test_failed_append_changes_nothing(case):
    kcache, bt, lens, free, fc, _ = fresh_state([100, 64], 6, 3, seed=3)
    s_new = 1
    if case == "too_few_pages":
        s_new = 64 * 3  # needs 2 + 3 pages, 2 are free
    elif case == "row_too_short":
        s_new = 129      # 100 + 129 tokens need 4 pages, the row holds 3
    elif case == "negative_length":
        lens[1] = -1
    elif case == "bad_free_page":
        free[fc - 1] = 99
    elif case == "bad_last_page":
        bt[0, 1] = 6
    rows = np.ones((2, s_new, 8), dtype=np.int32)
    res = pc.append(kcache, bt, lens, free, fc, rows)
    assert res[-1] != "ok"
    for x, y in zip((kcache, bt, lens, free, fc), res[:-1]):
        np.testing.assert_array_equal(x, y)


def test_release_that_overfills_changes_nothing():
    kcache, bt, lens, free, fc, _ = fresh_state([100, 64], 6, 3, seed=4)
    small = free[:fc + 2].copy()  # room for 2 more pages, releasing both needs 3
    res = pc.release(bt, lens, small, fc, np.array([1, 1]))
    assert res[-1] != "ok"
    np.testing.assert_array_equal(res[1], lens)
    assert res[3] == fc


def test_decode_over_appended_rows_matches_brute_force():
    """A decode step after an append attends over the grown sequences: the
    decode oracle on the appended cache equals dense attention over the rows
    kept by the unpaged model."""
    import torch
    import oracle
    from test_oracle_pins import brute_force
    from mla_paged_latent_decode_b200 import synth

    w = synth.custom_workload(3, 1, 4, [63, 64, 1], pool_pages=8)
    inp = synth.make_inputs(w, seed=5)
    kc = inp.kcache.view(torch.int16).numpy()
    used = {int(p) for i in range(3) for p in inp.block_table[i, :synth.pages_for(
        int(inp.cache_seqlens[i]))]}
    free = np.array([p for p in range(8) if p not in used], dtype=np.int32)
    bt = np.zeros((3, 4), dtype=np.int32)
    bt[:, :inp.block_table.shape[1]] = inp.block_table.numpy()
    new_rows = torch.randn(3, 2, 576, generator=torch.Generator().manual_seed(9)).to(
        torch.bfloat16).view(torch.int16).numpy()
    kc2, bt2, lens2, _, _, st = pc.append(kc, bt, inp.cache_seqlens.numpy(), free, len(free),
                                          new_rows)
    assert st == "ok" and lens2.tolist() == [65, 66, 3]
    grown = synth.DecodeInputs(w, 5, inp.q, torch.from_numpy(kc2).view(torch.bfloat16),
                               torch.from_numpy(bt2), torch.from_numpy(lens2), inp.scale, False)
    out, lse = oracle.decode(grown.q, grown.kcache, grown.block_table, grown.cache_seqlens,
                             grown.scale, False)
    ref_out, ref_lse = brute_force(grown)
    np.testing.assert_allclose(out, ref_out, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-14)
    # and the last token of each sequence is the appended row
    for i in range(3):
        seq = pc.sequence_rows(kc2, bt2, lens2, i)
        np.testing.assert_array_equal(seq[-1], new_rows[i, 1])
        np.testing.assert_array_equal(seq[-2], new_rows[i, 0])


MUTATIONS = {
    "floor_page_count": ("need.append(pages_for(L + s_new) - pages_for(L))",
                         "need.append((L + s_new) // PAGE - L // PAGE)"),
    "row_in_page_wrong": ("kcache[page, t % PAGE, :] = rows[i, k, :]",
                          "kcache[page, k % PAGE, :] = rows[i, k, :]"),
    "pop_from_bottom": ("block_table[i, first_new + r] = free_pages[top]",
                        "block_table[i, first_new + r] = free_pages[int(free_count) - 1 - top]"),
    "length_not_grown": ("seqlens[i] = L + s_new", "seqlens[i] = L"),
    "release_keeps_length": ("            seqlens[i] = 0\n", "            pass\n"),
    "release_skips_last_page": ("for r in range(pages_for(int(seqlens[i]))):",
                                "for r in range(int(seqlens[i]) // PAGE):"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_reject_mutation(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor missing: {old}"
    path = tmp_path / f"mut_{name}.py"
    path.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"mut_{name}", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    with pytest.raises(AssertionError):
        for seed in range(6):
            random_walk(mod, seed)
