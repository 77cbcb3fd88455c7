"""Plain CPU statement of the paged latent cache's bookkeeping: appending new
tokens' latent rows and allocating / releasing 64-token pages.

TEST INFRASTRUCTURE ONLY: the tests are its only callers.  It shares no code
with the CUDA path and imports nothing from it.

What it follows:
  - After each decoding step the newest token's cached state is added to the
    cache for later steps ("DeepSeek #OpenSourceWeek Day 1: Launch of FlashMLA",
    "How KV Caching Works?"), and in MLA that state is the one latent row c_t
    per token ("How MLA Optimizes Memory Usage").
  - The cache is paged: 64-token blocks, allocated on demand like OS virtual
    memory, so a sequence grows in 64-token increments, and blocks a sequence
    no longer uses are released ("FlashMLA: Revolutionizing Efficient
    Decoding...", section 4.3.2 "Paged KV Cache").

The pages give no allocation order; the reading taken here (the library uses
the same rule, stated in its header):
  - free pages form a stack free_pages[0:free_count]; allocation pops from the
    top, sequence after sequence in batch order and page after page within a
    sequence;
  - release pushes a released sequence's pages in page order, sequences in
    batch order, and sets its length to 0;
  - an append that cannot be satisfied (too few free pages, a block-table row
    too short, a page id outside the cache, a negative length) changes nothing;
    so does a release that would overfill the free-page array.

Every function works on copies and returns the new state plus a status string
("ok" or the reason nothing changed).
"""
from __future__ import annotations

import numpy as np

PAGE = 64
D_QK = 576


def pages_for(length: int) -> int:
    """Pages a sequence of `length` tokens occupies: ceil(length / 64)."""
    return -(-int(length) // PAGE)


def append(kcache, block_table, seqlens, free_pages, free_count: int, rows):
    """Append rows[i, k] (k < s_new) as tokens L_i + k of every sequence i.

    kcache [nblk, 64, 576] (any dtype; values are moved, never computed on),
    block_table [b, stride] int32, seqlens [b] int32, free_pages [cap] int32,
    free_count int, rows [b, s_new, 576] (same dtype as kcache).
    Returns (kcache, block_table, seqlens, free_pages, free_count, status).
    """
    kcache = np.array(kcache, copy=True)
    block_table = np.array(block_table, dtype=np.int32, copy=True)
    seqlens = np.array(seqlens, dtype=np.int32, copy=True)
    free_pages = np.array(free_pages, dtype=np.int32, copy=True)
    rows = np.asarray(rows)
    b, s_new = rows.shape[0], rows.shape[1]
    nblk, stride = kcache.shape[0], block_table.shape[1]
    unchanged = (kcache, block_table, seqlens, free_pages, int(free_count))

    # 1. how many new pages each sequence needs, checked before anything moves
    need = []
    for i in range(b):
        L = int(seqlens[i])
        if L < 0:
            return unchanged + ("negative length",)
        if pages_for(L + s_new) > stride:
            return unchanged + ("block-table row too short",)
        if L % PAGE != 0:
            last = int(block_table[i, L // PAGE])
            if not 0 <= last < nblk:
                return unchanged + ("page id outside the cache",)
        need.append(pages_for(L + s_new) - pages_for(L))
    if sum(need) > free_count:
        return unchanged + ("too few free pages",)
    for slot in range(int(free_count) - sum(need), int(free_count)):
        if not 0 <= int(free_pages[slot]) < nblk:
            return unchanged + ("page id outside the cache",)

    # 2. pop pages off the free stack into the block-table rows
    top = int(free_count)
    for i in range(b):
        first_new = pages_for(int(seqlens[i]))
        for r in range(need[i]):
            top -= 1
            block_table[i, first_new + r] = free_pages[top]

    # 3. write each new row into its page, then grow the length
    for i in range(b):
        L = int(seqlens[i])
        for k in range(s_new):
            t = L + k
            page = int(block_table[i, t // PAGE])
            kcache[page, t % PAGE, :] = rows[i, k, :]
        seqlens[i] = L + s_new
    return kcache, block_table, seqlens, free_pages, top, "ok"


def release(block_table, seqlens, free_pages, free_count: int, release_mask):
    """Give back every page of the sequences with release_mask[i] != 0.

    Pages are pushed onto the free stack (sequence order, page order within a
    sequence) and those sequences' lengths become 0.  Their block-table rows
    are left as they are: entries past a sequence's length are never read.
    Returns (block_table, seqlens, free_pages, free_count, status).
    """
    block_table = np.array(block_table, dtype=np.int32, copy=True)
    seqlens = np.array(seqlens, dtype=np.int32, copy=True)
    free_pages = np.array(free_pages, dtype=np.int32, copy=True)
    cap = free_pages.shape[0]
    unchanged = (block_table, seqlens, free_pages, int(free_count))
    give = 0
    for i in range(len(seqlens)):
        if release_mask[i]:
            L = int(seqlens[i])
            if L < 0 or pages_for(L) > block_table.shape[1]:
                return unchanged + ("bad length",)
            give += pages_for(L)
    if free_count + give > cap:
        return unchanged + ("free-page array full",)
    top = int(free_count)
    for i in range(len(seqlens)):
        if release_mask[i]:
            for r in range(pages_for(int(seqlens[i]))):
                free_pages[top] = block_table[i, r]
                top += 1
            seqlens[i] = 0
    return block_table, seqlens, free_pages, top, "ok"


def sequence_rows(kcache, block_table, seqlens, i: int):
    """The cached rows of sequence i in token order, read through the block table."""
    L = int(seqlens[i])
    return np.stack([kcache[int(block_table[i, t // PAGE]), t % PAGE] for t in range(L)]) \
        if L > 0 else np.zeros((0,) + tuple(kcache.shape[2:]), dtype=kcache.dtype)
