"""CPU restatement of the split-KV work partition (TEST INFRASTRUCTURE ONLY).

The pages ask for a decode kernel optimised for serving variable-length
sequences ("OpenSourceWeek Day 1: FlashMLA", opening paragraph; "DeepSeek
merilis open source FlashMLA", release bullets) but print no partition rule.  The rule below is the
one the library documents in its header, restated independently in plain
Python loops so that the GPU's metadata can be compared with it bit for bit:

  n_i     = ceil(L_i / 64) pages of sequence i
  items_i = max(n_i, 1)        (an empty sequence still owns one item: its
                                 output, zeros and lse = -inf, must be written)
  every sequence costs P + items_i units; laid end to end, sequence i starts
  at unit start_i and its item j sits at unit start_i + P + j.
  cap     = ceil(total / W);  the item at unit u belongs to worker u // cap.
  P       = PIECE_COST_CTA (2) when s_q * h_q <= 64 query rows run on one CTA
            per worker, PIECE_COST_PAIR (7) when they run on CTA pairs; the
            header states both as the library's tuned constants.
  Exception: if b <= W and every sequence costs at most cap + 2 P units, the
  sequences stay whole: worker i takes every item of sequence i (i < b).

A worker therefore owns one contiguous run of items, which may begin or end
inside a sequence.  A sequence spread over k workers yields k pieces ("splits")
that are merged afterwards by log-sum-exp.

Per worker the metadata row holds 8 int32:
  [begin_seq, begin_item, end_seq, end_item (exclusive), begin_split, num_pieces, 0, 0]
with num_pieces = 0 (and the rest 0) for a worker that owns nothing.
num_splits[i + 1] - num_splits[i] is the number of pieces of sequence i.
"""
from __future__ import annotations

PAGE = 64
PIECE_COST_CTA = 2
PIECE_COST_PAIR = 7
ROWS_PER_CTA = 64
MD_STRIDE = 8


def piece_cost_for(s_q: int, h_q: int) -> int:
    """The per-sequence cost P the rule uses for s_q * h_q query rows."""
    return PIECE_COST_CTA if s_q * h_q <= ROWS_PER_CTA else PIECE_COST_PAIR


def split_plan(seqlens, num_workers: int, piece_cost: int):
    """Returns (tile_md as a list of num_workers rows of 8 ints, num_splits list of b+1)."""
    lens = [int(v) for v in seqlens]
    W = int(num_workers)
    P = int(piece_cost)
    assert W >= 1 and P >= 0
    items = []
    for L in lens:
        n = (L + PAGE - 1) // PAGE if L > 0 else 0
        items.append(max(n, 1))
    starts = []
    total = 0
    for it in items:
        starts.append(total)
        total += P + it
    cap = max(1, -(-total // W))

    if len(lens) <= W and max(P + it for it in items) <= cap + 2 * P:
        md = [[0] * MD_STRIDE for _ in range(W)]
        for i, it in enumerate(items):
            md[i] = [i, 0, i, it, 0, 1, 0, 0]
        return md, list(range(len(lens) + 1))

    # which worker owns each item, written out item by item
    owner = {}
    for i, it in enumerate(items):
        for j in range(it):
            owner[(i, j)] = (starts[i] + P + j) // cap

    md = [[0] * MD_STRIDE for _ in range(W)]
    pieces_of_seq = [0] * len(lens)
    first_worker_of_seq = [None] * len(lens)
    for i, it in enumerate(items):
        ws = sorted({owner[(i, j)] for j in range(it)})
        pieces_of_seq[i] = len(ws)
        first_worker_of_seq[i] = ws[0]
    for w in range(W):
        mine = [(i, j) for i, it in enumerate(items) for j in range(it) if owner[(i, j)] == w]
        if not mine:
            continue
        (bs, bi), (es, ei) = mine[0], mine[-1]
        n_pieces = len({i for i, _ in mine})
        md[w] = [bs, bi, es, ei + 1, w - first_worker_of_seq[bs], n_pieces, 0, 0]
    num_splits = [0]
    for k in pieces_of_seq:
        num_splits.append(num_splits[-1] + k)
    return md, num_splits


def num_workers_for(num_sms: int, s_q: int, h_q: int) -> int:
    """Upper bound on the workers the decode grid uses: one CTA per SM for up to
    64 query rows, else one pair of CTAs per 128-row block (the library may use
    fewer pairs, as many as the device holds at once)."""
    rows = s_q * h_q
    if rows <= 64:
        return max(1, num_sms)
    blocks = -(-rows // 128)
    return max(1, num_sms // (2 * blocks))
