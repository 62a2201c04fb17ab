"""CPU checks of the end-to-end parity rules the GPU tests apply to index
sets (tests/gpu_util.py): the oracle's own result passes, a swap at a near-tie
passes, and a swap away from the threshold or a block not kept whole fails."""
import numpy as np
import pytest

import oracle
from tests.gpu_util import check_block_sets, check_index_sets


def _scores(n, seed):
    return np.random.default_rng(seed).random(n).astype(np.float32)


def test_token_rule_accepts_oracle_and_near_tie_only():
    t = 5000
    s = _scores(t + 1, 1)
    nc = t - 128 + 1
    order = np.lexsort((np.arange(nc), -s[:nc].astype(np.float64)))
    kth, nxt = int(order[1023]), int(order[1024])
    s[nxt] = s[kth]  # an exact tie straddling the threshold
    oi, oc = oracle.topk_select(s, t)
    assert check_index_sets(oi, oc, oi, oc, s, t, 1024, 128, "same") == 0
    kept = set(oi[:oc - 128].tolist())
    inside, outside = (kth, nxt) if kth in kept else (nxt, kth)
    assert inside in kept and outside not in kept
    swapped = oi.copy()
    glob = sorted((kept - {inside}) | {outside})
    swapped[:oc - 128] = glob
    assert check_index_sets(swapped, oc, oi, oc, s, t, 1024, 128, "tie") == 2
    far = oi.copy()
    best = int(order[0])
    glob = sorted((kept - {best}) | {outside})
    far[:oc - 128] = glob
    with pytest.raises(AssertionError):
        check_index_sets(far, oc, oi, oc, s, t, 1024, 128, "far")


def _blocks_to_idx(blocks, nc, t, width, block=64, window=128):
    toks = np.concatenate([np.arange(b * block, min((b + 1) * block, nc)) for b in sorted(blocks)])
    w = np.arange(max(0, t - window + 1), t + 1)
    out = np.full(width, -1, np.int32)
    allp = np.concatenate([toks, w])
    out[:allp.size] = allp
    return out, int(allp.size)


def test_block_rule_accepts_oracle_and_near_tie_only():
    t = 9000
    s = _scores(t + 1, 2)
    nc = t - 128 + 1
    nb = (nc + 63) // 64
    bmax = np.array([s[b * 64:min((b + 1) * 64, nc)].max() for b in range(nb)], np.float64)
    order = np.lexsort((np.arange(nb), -bmax))
    b16, b17 = int(order[15]), int(order[16])
    # make block b17's maximum equal block b16's: a tie at the threshold
    j = b17 * 64 + int(np.argmax(s[b17 * 64:min((b17 + 1) * 64, nc)]))
    s[j] = np.float32(bmax[b16])
    oi, oc = oracle.block_select(s, t)
    width = 16 * 64 + 128
    assert check_block_sets(oi, oc, oi, oc, s, t, 16, 64, 128, "same") == 0
    chosen = set((oi[:oc - 128] // 64).tolist())
    alt = (chosen - {b16}) | {b17} if b16 in chosen else (chosen - {b17}) | {b16}
    gi, gc = _blocks_to_idx(alt, nc, t, width)
    assert check_block_sets(gi, gc, oi, oc, s, t, 16, 64, 128, "tie") == 2
    top = int(order[0])
    far = (chosen - {top}) | {int(order[40])}
    gi, gc = _blocks_to_idx(far, nc, t, width)
    with pytest.raises(AssertionError):
        check_block_sets(gi, gc, oi, oc, s, t, 16, 64, 128, "far")
    # a block that is not kept whole
    gi2 = oi.copy()
    gi2[5] = gi2[6]
    with pytest.raises(AssertionError):
        check_block_sets(gi2, oc, oi, oc, s, t, 16, 64, 128, "partial")
