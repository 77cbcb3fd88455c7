"""Plain CPU statement of sparse (top-k) MLA decoding over the paged latent
cache: each query position attends only to a given list of cached tokens.

TEST INFRASTRUCTURE ONLY: the tests are its only callers.  It shares no code
with the CUDA path and imports nothing from it.

The pages describe dynamic sparse attention as attention restricted to the most
relevant parts of the input instead of the whole sequence, reached by gathering
those tokens ("Boosting DeepSeek V3.2: Faster LLM Inference With FlashMLA",
the paragraph on Dynamic Sparse Attention).  How the tokens are chosen (an
indexer with trained weights) is outside this statement: the selection is an
input.  The reading taken here:
  - indices[i][j] lists, for sequence i and query position j, logical token
    positions t of that sequence; every head of the position uses the same
    list (one cached latent row per token serves all heads);
  - an entry is used when 0 <= t < L_i, and with `causal` also
    t <= L_i - s_q + j (the bottom-right alignment of the dense decode);
    other entries (padding such as -1) are skipped;
  - each used entry contributes one term, so a position listed twice counts
    twice (callers pass distinct positions);
  - over the used entries it is the dense decode's definition: s = scale *
    q . K_t over all 576 dims, out = softmax(s) . V with V_t = K_t[0:512],
    lse = ln sum exp(s); no used entry gives out = 0 and lse = -inf.
"""
from __future__ import annotations

import numpy as np

PAGE = 64
D_QK = 576
D_V = 512


def _f64(t):
    import torch
    if isinstance(t, torch.Tensor):
        return t.detach().cpu().to(torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def _i64(t):
    return np.asarray(t.detach().cpu() if hasattr(t, "detach") else t, dtype=np.int64)


def used_entries(indices_ij, L: int, s_q: int, j: int, causal: bool):
    """The entries of one index list the decode uses, in list order."""
    limit = L - s_q + j + 1 if causal else L
    limit = min(limit, L)
    return [int(t) for t in indices_ij if 0 <= int(t) < limit]


def decode(q, kcache, block_table, cache_seqlens, indices, scale: float, causal: bool):
    """Sparse decode.  q [b, s_q, h_q, 576], kcache [nblk, 64, 576], block_table
    [b, stride], cache_seqlens [b], indices [b, s_q, topk] (int).
    Returns (out [b, s_q, h_q, 512] float64, lse [b, h_q, s_q] float64)."""
    qd, kd = _f64(q), _f64(kcache)
    bt, lens, idx = _i64(block_table), _i64(cache_seqlens), _i64(indices)
    b, s_q, h_q, _ = qd.shape
    out = np.zeros((b, s_q, h_q, D_V))
    lse = np.full((b, h_q, s_q), -np.inf)
    for i in range(b):
        for j in range(s_q):
            toks = used_entries(idx[i, j], int(lens[i]), s_q, j, causal)
            if not toks:
                continue
            rows = np.stack([kd[bt[i, t // PAGE], t % PAGE] for t in toks])   # [n, 576]
            logits = scale * (qd[i, j] @ rows.T)                                 # [h_q, n]
            m = logits.max(axis=1, keepdims=True)
            w = np.exp(logits - m)
            total = w.sum(axis=1, keepdims=True)
            out[i, j] = (w / total) @ rows[:, :D_V]
            lse[i, :, j] = (m + np.log(total))[:, 0]
    return out, lse
