"""Oracle: token-level top-k selection with a forced local window, and the
first-generation block-level selection (comparison path).

Test infrastructure only (see the package docstring).

Readings of the pages (they give the sizes and the rule, not the details):
* the window is the ``window`` most recent tokens including the query's own
  position: [max(0, t - window + 1), t];
* global tokens are drawn only from outside the window: candidates [0, t - window];
* "most relevant" = highest score; equal scores are ordered by lower position;
* output = selected global positions ascending, then the window ascending,
  padded with -1 to ``k + window`` entries.
"""
from __future__ import annotations

import numpy as np


def candidate_count(t: int, window: int) -> int:
    """Number of positions outside the window: |[0, t - window]|."""
    return max(0, t - window + 1)


def window_range(t: int, window: int) -> np.ndarray:
    """The forced local window [max(0, t - window + 1), t]."""
    return np.arange(max(0, t - window + 1), t + 1, dtype=np.int64)


def _finish(sel: np.ndarray, t: int, k: int, window: int):
    out = np.concatenate([np.sort(sel).astype(np.int64), window_range(t, window)])
    count = int(out.size)
    padded = np.full(k + window, -1, dtype=np.int32)
    padded[:count] = out
    return padded, count


def topk_select(scores: np.ndarray, t: int, k: int = 1024, window: int = 128):
    """Token-level selection for one (query, KV group) row.

    scores: float32 array with at least max(0, t-window+1) entries; entry j is
    the score of position j.  Returns (idx [k + window] int32 padded with -1,
    count).  If there are at most k candidates, all of them are taken;
    otherwise candidates are ordered by (score descending, position ascending)
    and the first k are taken.
    """
    nc = candidate_count(t, window)
    cand = np.arange(nc, dtype=np.int64)
    if nc <= k:
        sel = cand
    else:
        s = np.asarray(scores[:nc], dtype=np.float32).astype(np.float64)
        order = np.lexsort((cand, -s))     # last key is primary: -score, then position
        sel = cand[order[:k]]
    return _finish(sel, t, k, window)


def block_select(scores: np.ndarray, t: int, n_blocks: int = 16, block: int = 64,
                 window: int = 128):
    """First-generation block-level selection for one (query, KV group) row.

    Block b covers positions [block*b, block*b + block - 1].  Only candidate
    positions (outside the window) count: a block's score is the maximum
    score of its candidate positions, and a block with none is not eligible.
    The n_blocks eligible blocks with the highest score (ties: lower block
    index) are kept whole - all their candidate positions - and the window is
    added.  Returns (idx [n_blocks*block + window] int32 padded with -1, count).
    """
    nc = candidate_count(t, window)
    nb = (nc + block - 1) // block
    bidx = np.arange(nb, dtype=np.int64)
    if nb <= n_blocks:
        chosen = bidx
    else:
        s = np.asarray(scores[:nc], dtype=np.float32).astype(np.float64)
        bscore = np.array([s[b * block:min((b + 1) * block, nc)].max() for b in range(nb)])
        order = np.lexsort((bidx, -bscore))
        chosen = bidx[order[:n_blocks]]
    toks = [np.arange(b * block, min((b + 1) * block, nc), dtype=np.int64)
            for b in np.sort(chosen)]
    sel = np.concatenate(toks) if toks else np.zeros(0, dtype=np.int64)
    return _finish(sel, t, n_blocks * block, window)
