"""The softmax-partial merge that context-parallel decode relies on, checked
on the oracle (CPU): per-range full attention (its own max, sum and
normalised output) merged as M = max_r m_r, w_r = l_r exp(m_r - M),
O = sum_r w_r O_r / sum_r w_r, L = sum_r w_r equals full attention over the
whole sequence, and each range's scores computed from its logits with the
merged (M, L) equal the unsplit scores.  A planted mistake (weights without
l_r) must fail the same check."""
import numpy as np
import pytest

import oracle


def _merge(parts, with_l=True):
    m = np.stack([p[1] for p in parts])        # [R, Hq]
    l = np.stack([p[2] for p in parts])
    O = np.stack([p[0] for p in parts])        # [R, Hq, D]
    M = m.max(axis=0)
    w = np.exp(m - M) * (l if with_l else 1.0)
    L = w.sum(axis=0)
    return (w[:, :, None] * O).sum(axis=0) / L[:, None], M, L


@pytest.mark.parametrize("seed", range(12))
def test_merged_partials_equal_full_attention(seed):
    rng = np.random.default_rng(seed)
    Hq, Hkv, D = 8, 2, 16
    N = int(rng.integers(2, 400))
    q = rng.standard_normal((Hq, D)) * 2.0
    k = rng.standard_normal((N, Hkv, D))
    v = rng.standard_normal((N, Hkv, D))
    scale = 1.0 / np.sqrt(D)
    R = int(rng.integers(1, min(N, 6) + 1))
    cuts = np.sort(rng.choice(np.arange(1, N), size=R - 1, replace=False)) if R > 1 else []
    bounds = np.concatenate([[0], cuts, [N]]).astype(int)
    parts = [oracle.full_attention_row(q, k[a:b], v[a:b], b - a - 1, scale)
             for a, b in zip(bounds[:-1], bounds[1:])]
    O, M, L = _merge(parts)
    Oref, mref, lref, Pref = oracle.full_attention_row(q, k, v, N - 1, scale)
    assert np.allclose(O, Oref, rtol=1e-12, atol=1e-12)
    # the logits come from matrix-vector products over different slices: equal
    # up to the last bits of their rounding
    assert np.allclose(M, mref, rtol=1e-13, atol=0) and np.allclose(L, lref, rtol=1e-12)
    # each range's probabilities from its own logits and the merged (M, L)
    P = np.concatenate([np.exp(np.log(p[3]) + p[1][:, None] - M[:, None]) * p[2][:, None] / L[:, None]
                        for p in parts], axis=1)
    assert np.allclose(P, Pref, rtol=1e-10, atol=1e-300)
    # float32 scores: at most one rounding step apart
    assert np.allclose(oracle.selection_scores(P, Hkv), oracle.selection_scores(Pref, Hkv),
                       rtol=2.0 ** -22, atol=0)
    if R > 1:
        Obad, _, _ = _merge(parts, with_l=False)
        assert not np.allclose(Obad, Oref, rtol=1e-6, atol=1e-9)
