"""The split of token selection that context-parallel decode relies on,
checked on the oracle (CPU): for random position splits of a sequence across
ranks and scores with many exact ties, taking each rank's top-(k + window)
over all its positions, dropping the window positions and keeping the k best
of the union by (score desc, position asc) gives exactly the unsplit
selection.  A planted case shows the `+ window` is needed."""
import numpy as np
import pytest

import oracle


def merged_selection(scores, t, k, window, lens, local_k=None):
    """The context-parallel selection of one row, written with oracle calls."""
    local_k = k + window if local_k is None else local_k
    pos0 = np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int64)
    cand = []
    for p0, n in zip(pos0, lens):
        idx, cnt = oracle.topk_select(scores[p0:p0 + n], int(n) - 1, local_k, 0)
        cand += [(float(scores[p0 + j]), int(p0 + j)) for j in idx[:cnt]]
    cand = [c for c in cand if c[1] <= t - window]      # the window is added, not selected
    cand.sort(key=lambda c: (-c[0], c[1]))
    sel = np.array(sorted(p for _, p in cand[:k]), dtype=np.int64)
    return np.concatenate([sel, oracle.window_range(t, window)])


def _random_split(rng, N, R):
    R = min(R, N)
    cuts = np.sort(rng.choice(np.arange(1, N), size=R - 1, replace=False)) if R > 1 else []
    return np.diff(np.concatenate([[0], cuts, [N]])).astype(np.int64)


@pytest.mark.parametrize("seed", range(40))
def test_split_selection_equals_unsplit_selection(seed):
    rng = np.random.default_rng(seed)
    N = int(rng.integers(1, 5000))
    k = int(rng.choice([1, 7, 64, 300, 1024]))
    window = int(rng.choice([1, 5, 128]))
    levels = int(rng.choice([2, 16, 1 << 20]))          # few levels: many exact ties
    scores = (rng.integers(0, levels, N) / levels).astype(np.float32)
    lens = _random_split(rng, N, int(rng.integers(1, 9)))
    t = N - 1
    exp_idx, exp_cnt = oracle.topk_select(scores, t, k, window)
    got = merged_selection(scores, t, k, window, lens)
    assert got.size == exp_cnt and list(got) == list(exp_idx[:exp_cnt])


def test_local_top_k_alone_is_not_enough():
    """The rank holding the window ranks its window positions too: with only its
    local top-k, high-scoring window keys crowd out its real candidates."""
    N, k, window = 40, 3, 4
    scores = np.linspace(0.1, 0.5, N).astype(np.float32)
    scores[N - window:] = 1.0                           # the window outscores everything
    t = N - 1
    exp_idx, exp_cnt = oracle.topk_select(scores, t, k, window)
    lens = [N]
    assert list(merged_selection(scores, t, k, window, lens)) == list(exp_idx[:exp_cnt])
    short = merged_selection(scores, t, k, window, lens, local_k=k)
    assert list(short) != list(exp_idx[:exp_cnt])
