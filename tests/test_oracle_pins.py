"""The CPU oracle against closed forms, invariants, brute force and the pages'
stated sizes; and planted mistakes in copies of the oracle, each of which must
be caught by at least one of those checks."""
import os

import numpy as np
import pytest

import oracle
from tests import _pins as P

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hysparse2_constants.txt")

ATTN_CHECKS = [P.check_brute_force_attention, P.check_known_logits, P.check_uniform_and_single,
               P.check_probability_sums, P.check_gqa_mapping, P.check_causality,
               P.check_shift_and_permutation]


@pytest.mark.parametrize("check", ATTN_CHECKS, ids=lambda c: c.__name__)
def test_attention_pins(check):
    assert check(oracle.full_attention_row, oracle.selection_scores) is None


def test_topk_pins():
    assert P.check_topk_brute(oracle.topk_select) is None
    assert P.check_topk_structure(oracle.topk_select) is None


def test_block_pins():
    assert P.check_block_brute(oracle.block_select) is None


def test_sparse_pins():
    assert P.check_sparse_equals_full(oracle.full_attention_row, oracle.sparse_attention_row,
                                      oracle.topk_select, oracle.selection_scores) is None
    assert P.check_sparse_brute(oracle.sparse_attention_row) is None


def _golden():
    vals = {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, value = line.split("|")[0].split()
        vals.setdefault(name, set()).add(int(value))
    return vals


def test_golden_sizes_match_oracle_defaults():
    g = _golden()
    assert all(len(v) == 1 for v in g.values()), "pages disagree on a size"
    k, w, blk = (g["topk_global_tokens"].pop(), g["local_window_tokens"].pop(),
                 g["gen1_block_tokens"].pop())
    t = 10_000
    idx, c = oracle.topk_select(np.random.default_rng(0).random(t + 1).astype(np.float32), t)
    assert idx.size == k + w == 1152 and c == k + w
    assert list(idx[k:c]) == list(range(t - w + 1, t + 1))
    idx, c = oracle.block_select(np.ones(t + 1, np.float32), t)
    assert c == 16 * blk + w and list(idx[:16 * blk]) == list(range(16 * blk))


def test_run_helpers_rows_and_padding():
    rng = np.random.default_rng(12)
    Hq, Hkv, D = 4, 2, 8
    kv_off = np.array([0, 300, 310])
    q_off = np.array([0, 2, 5])
    q = rng.standard_normal((5, Hq, D))
    k = rng.standard_normal((310, Hkv, D))
    v = rng.standard_normal((310, Hkv, D))
    res = oracle.run_full_attention(q, k, v, q_off, kv_off, Hkv, 0.3)
    # query rows of sequence 1 (kv 10, q 3) sit at positions 7, 8, 9
    assert [res[r][4] for r in range(5)] == [298, 299, 7, 8, 9]
    O, m, l, Pr = oracle.full_attention_row(q[3], k[300:310], v[300:310], 8, 0.3)
    assert np.array_equal(res[3][0], O)
    idx = np.full((5, Hkv, 1152), -1, np.int32)
    cnt = np.zeros((5, Hkv), np.int32)
    for r in range(5):
        for g in range(Hkv):
            i, c = oracle.topk_select(res[r][3][g], res[r][4])
            idx[r, g], cnt[r, g] = i, c
    sp = oracle.run_sparse_attention(q, k, v, q_off, kv_off, idx, cnt, 0.3)
    for r in range(5):  # every context here is <= 1152: sparse == full
        assert np.allclose(sp[r], res[r][0], atol=1e-12)


# ----------------------------------------------------------------------------
# planted mistakes: each mutant copy must fail at least one pin
# ----------------------------------------------------------------------------
def _attn_fails(far, ss):
    return any(c(far, ss) is not None for c in ATTN_CHECKS)


def _mut_no_scale(q, k, v, t, scale):
    return oracle.full_attention_row(q, k, v, t, 1.0)


def _mut_sees_future(q, k, v, t, scale):
    return oracle.full_attention_row(q, k, v, min(t + 1, k.shape[0] - 1), scale)


def _mut_drops_current(q, k, v, t, scale):
    O, m, l, Pm = oracle.full_attention_row(q, k, v, t - 1, scale)
    return O, m, l, np.concatenate([Pm, np.zeros((Pm.shape[0], 1))], axis=1)


def _mut_gqa_modulo(q, k, v, t, scale):
    # head h reads KV head h % Hkv instead of h // G
    Hq, Hkv = q.shape[0], k.shape[1]
    G = Hq // Hkv
    order = np.array([h % Hkv for h in range(Hq)])
    qq = np.empty_like(q)
    for g in range(Hkv):  # regroup heads so that group g holds heads with h % Hkv == g
        qq[g * G:(g + 1) * G] = q[order == g]
    O, m, l, Pm = oracle.full_attention_row(qq, k, v, t, scale)
    inv = np.concatenate([np.where(order == g)[0] for g in range(Hkv)])
    O2, P2 = np.empty_like(O), np.empty_like(Pm)
    O2[inv], P2[inv] = O, Pm
    return O2, m, l, P2


def _mut_transposed_qk(q, k, v, t, scale):
    # uses the query's own vector for every key (a transposed operand collapses keys)
    O, m, l, Pm = oracle.full_attention_row(q, k, v, t, scale)
    n = t + 1
    Pu = np.full_like(Pm, 1.0 / max(n, 1))
    G = q.shape[0] // k.shape[1]
    Ou = np.stack([Pu[h] @ v[:n, h // G] for h in range(q.shape[0])]) if n > 0 else O
    return Ou, m, l, Pu


def _mut_scores_mean(Pm, Hkv):
    G = Pm.shape[0] // Hkv
    return (oracle.selection_scores(Pm, Hkv).astype(np.float64) / G).astype(np.float32)


def _mut_scores_one_head(Pm, Hkv):
    G = Pm.shape[0] // Hkv
    return np.stack([Pm[g * G] for g in range(Hkv)]).astype(np.float32)


@pytest.mark.parametrize("mut", [_mut_no_scale, _mut_sees_future, _mut_drops_current,
                                 _mut_gqa_modulo, _mut_transposed_qk],
                         ids=lambda f: f.__name__)
def test_planted_attention_mistakes_are_caught(mut):
    assert _attn_fails(mut, oracle.selection_scores)


@pytest.mark.parametrize("mut", [_mut_scores_mean, _mut_scores_one_head], ids=lambda f: f.__name__)
def test_planted_score_mistakes_are_caught(mut):
    assert _attn_fails(oracle.full_attention_row, mut)


def _mut_tie_high_index(scores, t, k=1024, window=128):
    nc = max(0, t - window + 1)
    cand = np.arange(nc)
    if nc <= k:
        sel = cand
    else:
        s = scores[:nc].astype(np.float64)
        sel = cand[np.lexsort((-cand, -s))[:k]]
    out = np.concatenate([np.sort(sel), np.arange(max(0, t - window + 1), t + 1)])
    pad = np.full(k + window, -1, np.int32)
    pad[:out.size] = out
    return pad, out.size


def _mut_window_off_by_one(scores, t, k=1024, window=128):
    # candidates run up to t - window + 1, overlapping the window by one
    nc = max(0, t - window + 2)
    cand = np.arange(nc)
    if nc <= k:
        sel = cand
    else:
        s = scores[:nc].astype(np.float64)
        sel = cand[np.lexsort((cand, -s))[:k]]
    out = np.concatenate([np.sort(sel), np.arange(max(0, t - window + 1), t + 1)])
    pad = np.full(k + window + 1, -1, np.int32)
    pad[:out.size] = out
    return pad[:k + window], min(out.size, k + window)


def _mut_ascending_scores(scores, t, k=1024, window=128):
    return oracle.topk_select(-np.asarray(scores, np.float32), t, k, window)


@pytest.mark.parametrize("mut", [_mut_tie_high_index, _mut_window_off_by_one, _mut_ascending_scores],
                         ids=lambda f: f.__name__)
def test_planted_topk_mistakes_are_caught(mut):
    assert P.check_topk_brute(mut) is not None or P.check_topk_structure(mut) is not None


def _mut_block_mean(scores, t, n_blocks=16, block=64, window=128):
    nc = max(0, t - window + 1)
    nb = (nc + block - 1) // block
    if nb <= n_blocks:
        chosen = np.arange(nb)
    else:
        bs = np.array([scores[b * block:min((b + 1) * block, nc)].astype(np.float64).mean()
                       for b in range(nb)])
        chosen = np.lexsort((np.arange(nb), -bs))[:n_blocks]
    toks = [np.arange(b * block, min((b + 1) * block, nc)) for b in np.sort(chosen)]
    sel = np.concatenate(toks) if toks else np.zeros(0, np.int64)
    out = np.concatenate([sel, np.arange(max(0, t - window + 1), t + 1)])
    pad = np.full(n_blocks * block + window, -1, np.int32)
    pad[:out.size] = out
    return pad, out.size


def _mut_block_whole_last(scores, t, n_blocks=16, block=64, window=128):
    # keeps the block cut by the window whole (runs into the window)
    idx, c = oracle.block_select(scores, t, n_blocks, block, window)
    nc = max(0, t - window + 1)
    if nc % block and (nc - 1) in idx[:c]:
        extra = np.arange(nc, (nc // block + 1) * block)
        out = np.concatenate([idx[:c], extra])
        pad = np.full(max(out.size, idx.size), -1, np.int32)
        pad[:out.size] = out
        return pad[:idx.size], min(out.size, idx.size)
    return idx, c


@pytest.mark.parametrize("mut", [_mut_block_mean, _mut_block_whole_last], ids=lambda f: f.__name__)
def test_planted_block_mistakes_are_caught(mut):
    assert P.check_block_brute(mut) is not None


def _mut_sparse_ignores_group(q, k, v, sets, scale):
    return oracle.sparse_attention_row(q, k, v, [sets[0]] * len(sets), scale)


def _mut_sparse_drops_last(q, k, v, sets, scale):
    return oracle.sparse_attention_row(q, k, v, [s[:-1] for s in sets], scale)


@pytest.mark.parametrize("mut", [_mut_sparse_ignores_group, _mut_sparse_drops_last],
                         ids=lambda f: f.__name__)
def test_planted_sparse_mistakes_are_caught(mut):
    a = P.check_sparse_equals_full(oracle.full_attention_row, mut, oracle.topk_select,
                                   oracle.selection_scores)
    b = P.check_sparse_brute(mut)
    assert a is not None or b is not None
