"""Pins for the CPU restatement of the split-KV partition rule (no GPU).

The rule is the library's own design (the pages print none), so these checks
fix what any correct partition must satisfy, and brute force over small cases.
"""
import itertools

import pytest

from oracle.scheduler import PAGE, PIECE_COST_CTA, PIECE_COST_PAIR, piece_cost_for, split_plan

COSTS = (PIECE_COST_CTA, PIECE_COST_PAIR)


def items_of(L):
    return max((L + PAGE - 1) // PAGE, 1)


def check_plan(lens, W, P):
    md, ns = split_plan(lens, W, P)
    b = len(lens)
    assert len(md) == W and len(ns) == b + 1 and ns[0] == 0
    # every item of every sequence is covered exactly once, workers in order
    seen = {}
    pieces = {i: [] for i in range(b)}
    order = []
    for w, row in enumerate(md):
        bs, bi, es, ei, bsplit, npieces = row[:6]
        assert row[6] == 0 and row[7] == 0
        if npieces == 0:
            assert row == [0] * 8
            continue
        assert npieces == es - bs + 1 and bs <= es
        for i in range(bs, es + 1):
            lo = bi if i == bs else 0
            hi = ei if i == es else items_of(lens[i])
            assert 0 <= lo < hi <= items_of(lens[i])
            for j in range(lo, hi):
                assert (i, j) not in seen
                seen[(i, j)] = w
                order.append((i, j))
            pieces[i].append((w, lo, hi))
    assert len(seen) == sum(items_of(L) for L in lens)
    assert order == sorted(order)  # contiguous, lexicographic runs
    for i in range(b):
        k = ns[i + 1] - ns[i]
        assert k == len(pieces[i]) and k >= 1
        # split indices: the worker that starts a sequence has split 0, the next 1, ...
        for s, (w, lo, hi) in enumerate(pieces[i]):
            expect = md[w][4] if md[w][0] == i else 0
            assert s == expect
    # balance: no worker owns more than cap items; with sequences kept whole
    # (b <= W and no sequence above cap + 2P units) one sequence per worker
    total = sum(P + items_of(L) for L in lens)
    cap = -(-total // W)
    whole = b <= W and max(P + items_of(L) for L in lens) <= cap + 2 * P
    if whole:
        assert ns == list(range(b + 1))
        for w in range(W):
            assert md[w][:6] == ([w, 0, w, items_of(lens[w]), 0, 1] if w < b else [0] * 6)
    else:
        for w in range(W):
            assert sum(1 for v in seen.values() if v == w) <= cap
    # pieces beyond one per sequence come only from worker boundaries
    assert ns[-1] <= b + W - 1
    return md, ns


def test_cost_follows_the_kernel_the_rows_select():
    # up to 64 query rows run on one CTA per worker, more on CTA pairs
    assert piece_cost_for(1, 16) == piece_cost_for(1, 64) == piece_cost_for(4, 16) == PIECE_COST_CTA
    assert piece_cost_for(1, 65) == piece_cost_for(1, 128) == piece_cost_for(2, 128) == PIECE_COST_PAIR


@pytest.mark.parametrize("P", COSTS)
def test_single_worker_takes_everything(P):
    md, ns = check_plan([37, 130, 0], 1, P)
    assert md[0][:6] == [0, 0, 2, 1, 0, 3]
    assert ns == [0, 1, 2, 3]


@pytest.mark.parametrize("P", COSTS)
def test_one_sequence_per_worker_when_costs_align(P):
    # 4 sequences of 6 pages each, P + 6 units each, 4 workers: one each, no splits
    md, ns = check_plan([6 * 64] * 4, 4, P)
    assert ns == [0, 1, 2, 3, 4]
    assert [r[:6] for r in md] == [[i, 0, i, 6, 0, 1] for i in range(4)]


def test_cost_moves_pages_off_workers_that_start_sequences():
    # 3 sequences of 10 pages, 2 workers.  P = 2: 36 units, cap 18, worker 0
    # takes units 0..17 = sequence 0 (2 + 10) and units 12..17 of sequence 1,
    # i.e. its cost and 4 pages.  P = 7: 51 units, cap 26, worker 0 takes
    # sequence 0 (7 + 10) and units 17..25 of sequence 1, its cost and 2 pages.
    md, ns = check_plan([640] * 3, 2, 2)
    assert md[0][:6] == [0, 0, 1, 4, 0, 2]
    md, ns = check_plan([640] * 3, 2, 7)
    assert md[0][:6] == [0, 0, 1, 2, 0, 2]
    assert md[1][:6] == [1, 2, 2, 10, 1, 2]


def test_uniform_long_sequences_stay_whole():
    # 64 sequences of 64 pages on 74 workers.  P = 7: 71 units each, cap 62,
    # 71 <= 62 + 14, so one worker per sequence and no splits.  P = 2: 66 units,
    # cap 58, 66 > 58 + 4, so the linear rule splits them.
    md, ns = check_plan([4096] * 64, 74, 7)
    assert ns == list(range(65)) and sum(1 for r in md if r[5]) == 64
    md, ns = check_plan([4096] * 64, 74, 2)
    assert ns[-1] > 64


def test_whole_sequence_threshold():
    # two workers, P = 7.  30 + 2 pages: 37 + 9 = 46 units, cap 23, the longest
    # is 37 = cap + 14: whole.  32 + 2 pages: 39 + 9 = 48 units, cap 24, 39 > 38:
    # split by the linear rule.
    md, ns = check_plan([30 * 64, 2 * 64], 2, 7)
    assert ns == [0, 1, 2] and md[0][:6] == [0, 0, 0, 30, 0, 1] and md[1][:6] == [1, 0, 1, 2, 0, 1]
    md, ns = check_plan([32 * 64, 2 * 64], 2, 7)
    assert ns == [0, 2, 3]
    # more sequences than workers: the linear rule (worker 1 takes sequences 1 and 2)
    md, ns = check_plan([64] * 3, 2, 7)
    assert ns == [0, 1, 2, 3] and md[1][:6] == [1, 0, 2, 1, 0, 2]


@pytest.mark.parametrize("P", COSTS)
def test_long_sequence_is_split_across_workers(P):
    md, ns = check_plan([32768] * 15 + [1], 74, P)
    assert ns[-1] > 16                  # the long sequences are cut
    assert ns[16] - ns[15] == 1         # the one-token sequence is whole


@pytest.mark.parametrize("P", COSTS)
def test_more_workers_than_items(P):
    # 1 + 3 pages on 148 workers: cap 1 and the longer sequence costs P + 3 <=
    # 1 + 2P units, so both stay whole
    md, ns = check_plan([37, 130], 148, P)
    assert ns == [0, 1, 2] and sum(1 for r in md if r[5] > 0) == 2
    # 1 + 20 pages: P + 20 > 1 + 2P, so the linear rule gives one worker per page
    md, ns = check_plan([37, 20 * 64], 148, P)
    assert sum(1 for r in md if r[5] > 0) == 21
    assert ns == [0, 1, 21]


@pytest.mark.parametrize("P", COSTS)
@pytest.mark.parametrize("W", [1, 2, 3, 5, 7])
def test_brute_force_small(W, P):
    lengths = [0, 1, 63, 64, 65, 128, 129, 300]
    for b in (1, 2, 3, 4):
        for lens in itertools.product(lengths, repeat=b):
            check_plan(list(lens), W, P)


@pytest.mark.parametrize("P", COSTS)
def test_realistic_shapes(P):
    import torch
    g = torch.Generator().manual_seed(0)
    for W in (37, 74, 148):
        lens = torch.randint(1, 8193, (128,), generator=g).tolist()
        check_plan(lens, W, P)
        check_plan([4096] * 64, W, P)
