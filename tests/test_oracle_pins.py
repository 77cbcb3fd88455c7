"""Pins for the fp64 oracle, from mathematics and brute force (no GPU).

Each check is chosen so that a plausible slip in the oracle (a dropped rope
term, a wrong page index, an off-by-one in the causal limit, the value taken
from the wrong dims, a missing normalisation) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from mla_paged_latent_decode_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def brute_force(inp):
    """Dense reference from torch library routines: gather the rows of each
    sequence into a contiguous K, then softmax(scale * Q K^T) V with V = K[:, :512]."""
    b, s_q, h_q = inp.batch, inp.s_q, inp.h_q
    outs = torch.zeros(b, s_q, h_q, 512, dtype=torch.float64)
    lses = torch.zeros(b, h_q, s_q, dtype=torch.float64)
    kc = inp.kcache.to(torch.float64)
    for i in range(b):
        L = int(inp.cache_seqlens[i])
        npages = (L + 63) // 64
        rows = kc[inp.block_table[i, :npages].long()].reshape(-1, 576)[:L]
        for j in range(s_q):
            vis = L - s_q + j + 1 if inp.causal else L
            vis = max(0, min(vis, L))
            qj = inp.q[i, j].to(torch.float64)
            if vis == 0:
                lses[i, :, j] = -math.inf
                continue
            logits = inp.scale * qj @ rows[:vis].T
            outs[i, j] = torch.softmax(logits, dim=-1) @ rows[:vis, :512]
            lses[i, :, j] = torch.logsumexp(logits, dim=-1)
    return outs.numpy(), lses.numpy()


def run_oracle(inp):
    return oracle.decode(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens, inp.scale,
                         inp.causal)


@pytest.mark.parametrize("h_q", [1, 16])
@pytest.mark.parametrize("s_q", [1, 2])
@pytest.mark.parametrize("causal", [False, True])
def test_matches_brute_force(h_q, s_q, causal):
    w = synth.custom_workload(3, s_q, h_q, [1, 63, 130], causal=causal)
    inp = synth.make_inputs(w, seed=11)
    out, lse = run_oracle(inp)
    ref_out, ref_lse = brute_force(inp)
    np.testing.assert_allclose(out, ref_out, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-14)
    w2 = synth.custom_workload(3, s_q, h_q, [2, 64, 65], causal=causal)
    inp2 = synth.make_inputs(w2, seed=12)
    out, lse = run_oracle(inp2)
    ref_out, ref_lse = brute_force(inp2)
    np.testing.assert_allclose(out, ref_out, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-14)


def test_golden_two_token_sigmoid():
    with open(os.path.join(GOLDEN, "two_token_sigmoid.json")) as f:
        g = json.load(f)
    w = synth.custom_workload(1, 1, 1, [g["seqlen"]], scale=g["scale"])
    inp = synth.make_inputs(w, seed=0)
    inp.q.zero_()
    for c, v in g["q_nonzero"].items():
        inp.q[0, 0, 0, int(c)] = v
    inp.kcache.zero_()
    page = int(inp.block_table[0, 0])
    for t, row in enumerate(g["k_rows_nonzero"]):
        for c, v in row.items():
            inp.kcache[page, t, int(c)] = v
    out, lse = run_oracle(inp)
    expect = np.zeros(512)
    for c, v in g["expected_out_nonzero"].items():
        expect[int(c)] = v
    np.testing.assert_allclose(out[0, 0, 0], expect, rtol=1e-15, atol=1e-16)
    assert abs(lse[0, 0, 0] - g["expected_lse"]) < 1e-15


def test_single_token_returns_its_value_row():
    w = synth.custom_workload(2, 1, 16, [1, 1])
    inp = synth.make_inputs(w, seed=3)
    out, lse = run_oracle(inp)
    for i in range(2):
        row = inp.kcache[int(inp.block_table[i, 0]), 0].to(torch.float64).numpy()
        np.testing.assert_array_equal(out[i, 0], np.broadcast_to(row[:512], (16, 512)))
        logits = inp.scale * (inp.q[i, 0].to(torch.float64).numpy() @ row)
        np.testing.assert_allclose(lse[i, :, 0], logits, rtol=1e-13)


def test_identical_scores_give_mean_of_values():
    # q is zero on the 512 value dims, and every key shares its 64 rope dims, so all
    # logits are equal while the value rows differ: the output is their plain mean.
    L = 150
    w = synth.custom_workload(1, 1, 4, [L])
    inp = synth.make_inputs(w, seed=5)
    inp.q[..., :512] = 0
    shared_rope = inp.kcache[0, 0, 512:].clone()
    inp.kcache[..., 512:] = shared_rope
    out, lse = run_oracle(inp)
    rows = inp.kcache.to(torch.float64)[inp.block_table[0, :3].long()].reshape(-1, 576)[:L]
    mean_v = rows[:, :512].mean(0).numpy()
    for h in range(4):
        np.testing.assert_allclose(out[0, 0, h], mean_v, rtol=1e-11, atol=1e-13)
        s = inp.scale * float(inp.q[0, 0, h, 512:].to(torch.float64) @ shared_rope.to(torch.float64))
        assert abs(lse[0, h, 0] - (s + math.log(L))) < 1e-11


def test_zero_scale_gives_mean_and_log_count():
    w = synth.custom_workload(2, 2, 2, [70, 3], causal=True, scale=0.0)
    inp = synth.make_inputs(w, seed=6)
    out, lse = run_oracle(inp)
    kc = inp.kcache.to(torch.float64)
    for i, L in enumerate([70, 3]):
        rows = kc[inp.block_table[i, :(L + 63) // 64].long()].reshape(-1, 576)[:L]
        for j in range(2):
            vis = L - 2 + j + 1
            np.testing.assert_allclose(out[i, j], np.broadcast_to(rows[:vis, :512].mean(0).numpy(),
                                                                  (2, 512)), rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(lse[i, :, j], math.log(vis), rtol=1e-14)


def test_dominant_key_selects_its_value():
    L = 200
    w = synth.custom_workload(1, 1, 2, [L])
    inp = synth.make_inputs(w, seed=7)
    inp.q.zero_()
    inp.q[0, 0, :, 575] = 1.0
    inp.kcache[..., 575] = 0.0
    t_star = 137
    page = int(inp.block_table[0, t_star // 64])
    inp.kcache[page, t_star % 64, 575] = 1024.0   # logit gap = 1024 * scale ~ 74
    out, lse = run_oracle(inp)
    v = inp.kcache[page, t_star % 64, :512].to(torch.float64).numpy()
    np.testing.assert_allclose(out[0, 0, 0], v, rtol=1e-20, atol=1e-28)
    gap = 1024.0 * inp.scale
    assert abs(lse[0, 0, 0] - (gap + math.log1p((L - 1) * math.exp(-gap)))) < 1e-12


def test_page_permutation_invariance():
    w = synth.custom_workload(3, 2, 8, [130, 64, 200], causal=True)
    inp = synth.make_inputs(w, seed=8)
    out, lse = run_oracle(inp)
    nb = inp.kcache.shape[0]
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(99))
    new_cache = torch.empty_like(inp.kcache)
    new_cache[perm] = inp.kcache          # physical page p moves to perm[p]
    inp.kcache = new_cache
    inp.block_table = perm[inp.block_table.long()].to(torch.int32)
    out2, lse2 = run_oracle(inp)
    np.testing.assert_array_equal(out, out2)
    np.testing.assert_array_equal(lse, lse2)


def test_poisoned_tails_and_pad_pages_do_not_leak():
    w = synth.custom_workload(3, 2, 4, [37, 130, 64], causal=True)
    clean = synth.make_inputs(w, seed=9)
    poisoned = synth.make_inputs(w, seed=9, poison=True)
    assert poisoned.poison_page is not None
    out, lse = run_oracle(clean)
    out2, lse2 = run_oracle(poisoned)
    np.testing.assert_array_equal(out, out2)
    np.testing.assert_array_equal(lse, lse2)


def test_output_is_convex_combination_of_values():
    w = synth.custom_workload(2, 1, 16, [300, 90])
    inp = synth.make_inputs(w, seed=10)
    out, _ = run_oracle(inp)
    kc = inp.kcache.to(torch.float64)
    for i, L in enumerate([300, 90]):
        rows = kc[inp.block_table[i, :(L + 63) // 64].long()].reshape(-1, 576)[:L, :512].numpy()
        lo, hi = rows.min(0), rows.max(0)
        assert np.all(out[i, 0] >= lo - 1e-12) and np.all(out[i, 0] <= hi + 1e-12)


def test_lse_is_logsumexp_of_scaled_logits():
    from scipy.special import logsumexp
    w = synth.custom_workload(2, 2, 3, [100, 65], causal=True)
    inp = synth.make_inputs(w, seed=13)
    _, lse = run_oracle(inp)
    kc = inp.kcache.to(torch.float64).numpy()
    for i, L in enumerate([100, 65]):
        rows = kc[inp.block_table[i, :(L + 63) // 64].numpy()].reshape(-1, 576)[:L]
        for j in range(2):
            vis = L - 2 + j + 1
            logits = inp.scale * (inp.q[i, j].to(torch.float64).numpy() @ rows[:vis].T)
            np.testing.assert_allclose(lse[i, :, j], logsumexp(logits, axis=-1), rtol=1e-13)


def test_causal_single_query_equals_noncausal():
    w = synth.custom_workload(2, 1, 8, [77, 129], causal=False)
    inp = synth.make_inputs(w, seed=14)
    out, lse = run_oracle(inp)
    inp.causal = True
    out2, lse2 = run_oracle(inp)
    np.testing.assert_array_equal(out, out2)
    np.testing.assert_array_equal(lse, lse2)


def test_causal_limit_is_bottom_right():
    # query j of s_q sees t <= L - s_q + j: with s_q = 3 the first query misses the
    # last two tokens.  Make those two keys dominant; only query 2 may see both.
    L, s_q = 10, 3
    w = synth.custom_workload(1, s_q, 1, [L], causal=True)
    inp = synth.make_inputs(w, seed=15)
    inp.q.zero_()
    inp.q[0, :, 0, 575] = 1.0
    page = int(inp.block_table[0, 0])
    inp.kcache[page, :, 575] = 0.0
    inp.kcache[page, L - 1, 575] = 2048.0
    inp.kcache[page, L - 2, 575] = 1024.0
    out, _ = run_oracle(inp)
    kc = inp.kcache[page].to(torch.float64).numpy()
    np.testing.assert_allclose(out[0, 2, 0], kc[L - 1, :512], rtol=1e-20, atol=1e-28)
    np.testing.assert_allclose(out[0, 1, 0], kc[L - 2, :512], rtol=1e-20, atol=1e-28)
    assert np.max(np.abs(out[0, 0, 0] - kc[:L - 2, :512].mean(0))) < 1e-12


def test_empty_visible_set():
    w = synth.custom_workload(3, 2, 2, [0, 1, 5], causal=True)
    inp = synth.make_inputs(w, seed=16)
    out, lse = run_oracle(inp)
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0]))
    # L = 1 < s_q = 2: query 0 sees nothing, query 1 sees token 0
    assert np.all(out[1, 0] == 0) and np.all(np.isneginf(lse[1, :, 0]))
    assert np.all(np.isfinite(lse[1, :, 1]))
    assert np.all(np.isfinite(lse[2]))


@pytest.mark.parametrize("cut", [1, 63, 64, 65, 128, 199])
def test_split_and_combine_reproduces_unsplit(cut):
    L = 200
    w = synth.custom_workload(1, 2, 2, [L], causal=True)
    inp = synth.make_inputs(w, seed=17)
    full_out, full_lse = run_oracle(inp)
    rows = []
    for j in range(2):
        for h in range(2):
            rows += [(0, j, h, 0, cut), (0, j, h, cut, L)]
    po, pl = oracle.decode_rows(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens,
                                inp.scale, inp.causal, rows)
    k = 0
    for j in range(2):
        for h in range(2):
            o, l = oracle.combine(po[k:k + 2], pl[k:k + 2])
            np.testing.assert_allclose(o, full_out[0, j, h], rtol=1e-12, atol=1e-14)
            assert abs(l - full_lse[0, h, j]) < 1e-12
            k += 2


def test_combine_of_empty_ranges():
    o, l = oracle.combine(np.zeros((3, 512)), [-np.inf] * 3)
    assert np.all(o == 0) and l == -np.inf
    o, l = oracle.combine(np.stack([np.ones(512), np.zeros(512)]), [0.5, -np.inf])
    assert np.all(o == 1.0) and l == 0.5


def test_rows_api_matches_full_decode():
    inp = synth.make_inputs("tiny", seed=0)
    out, lse = run_oracle(inp)
    sel = [(1, 0, 5), (0, 0, 15), (1, 0, 0)]
    o, l = oracle.decode_rows(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens, inp.scale,
                              inp.causal, sel)
    for k, (i, j, h) in enumerate(sel):
        np.testing.assert_array_equal(o[k], out[i, j, h])
        assert l[k] == lse[i, h, j]
