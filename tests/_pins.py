"""Checks that pin the CPU oracle to facts outside itself.

Each ``check_*`` takes the oracle functions as arguments so that the same
check can run against the real oracle (it must pass) and against copies with a
planted mistake (at least one check must fail).  A check returns None when it
holds and a short message when it does not.

The facts used: closed forms of softmax attention (uniform keys, one visible
key, logits chosen as log-weights), invariants (probabilities of each head sum
to one, causality, grouped-query head mapping, shift and permutation
invariance), brute force on tiny inputs in pure Python (exp of the raw logits
without the max shift, fsum), and the rank definition of "the k highest,
lower position first".
"""
from __future__ import annotations

import math

import numpy as np

SCALE128 = float(np.float32(1.0 / math.sqrt(128.0)))


# --------------------------------------------------------------------------
# brute-force references (pure Python, tiny inputs only)
# --------------------------------------------------------------------------
def brute_attention(q_row, k_seq, v_seq, t, scale, keys=None):
    """Softmax attention by the textbook formula, pure Python, no max shift.

    keys: optional list per KV group of the positions to attend (default 0..t).
    Returns (O [Hq][D], P [Hq][list]) as Python floats.
    """
    Hq, D = len(q_row), len(q_row[0])
    Hkv = len(k_seq[0])
    G = Hq // Hkv
    O, P = [], []
    for h in range(Hq):
        g = h // G
        pos = list(range(t + 1)) if keys is None else [int(j) for j in keys[g]]
        w = [math.exp(scale * math.fsum(float(q_row[h][d]) * float(k_seq[j][g][d])
                                        for d in range(D))) for j in pos]
        z = math.fsum(w)
        p = [x / z for x in w]
        P.append(p)
        O.append([math.fsum(p[i] * float(v_seq[j][g][d]) for i, j in enumerate(pos))
                  for d in range(D)])
    return O, P


def brute_topk(scores, t, k, window):
    """Rank definition: candidate j is kept iff fewer than k candidates beat it,
    where i beats j when s_i > s_j, or s_i == s_j and i < j."""
    nc = max(0, t - window + 1)
    s = [float(x) for x in scores[:nc]]
    keep = []
    for j in range(nc):
        beaten = sum(1 for i in range(nc) if s[i] > s[j] or (s[i] == s[j] and i < j))
        if beaten < k:
            keep.append(j)
    return keep + list(range(max(0, t - window + 1), t + 1))


def brute_blocks(scores, t, n_blocks, block, window):
    nc = max(0, t - window + 1)
    s = [float(x) for x in scores[:nc]]
    nb = (nc + block - 1) // block
    bs = [max(s[b * block:min(nc, (b + 1) * block)]) for b in range(nb)]
    keep = []
    for b in range(nb):
        beaten = sum(1 for c in range(nb) if bs[c] > bs[b] or (bs[c] == bs[b] and c < b))
        if beaten < n_blocks:
            keep.extend(range(b * block, min(nc, (b + 1) * block)))
    return keep + list(range(max(0, t - window + 1), t + 1))


def _rng(seed):
    return np.random.default_rng(seed)


# --------------------------------------------------------------------------
# full attention + scores
# --------------------------------------------------------------------------
def check_brute_force_attention(full_attention_row, selection_scores):
    rng = _rng(1)
    for (Hq, Hkv, D, N, t) in [(4, 2, 8, 12, 11), (6, 3, 5, 9, 4), (2, 1, 7, 1, 0)]:
        q = rng.standard_normal((Hq, D))
        k = rng.standard_normal((N, Hkv, D))
        v = rng.standard_normal((N, Hkv, D))
        O, m, l, P = full_attention_row(q, k, v, t, 0.37)
        Ob, Pb = brute_attention(q, k, v, t, 0.37)
        if not np.allclose(O, np.array(Ob), rtol=0, atol=1e-12):
            return "O differs from brute force"
        if not np.allclose(P, np.array(Pb), rtol=0, atol=1e-13):
            return "P differs from brute force"
        G = Hq // Hkv
        s = selection_scores(P, Hkv)
        sb = np.array([[math.fsum(Pb[h][j] for h in range(g * G, (g + 1) * G))
                        for j in range(t + 1)] for g in range(Hkv)], dtype=np.float32)
        if not np.allclose(s, sb, rtol=2e-7, atol=0):
            return "scores differ from brute force"
    return None


def check_known_logits(full_attention_row, selection_scores):
    """Logits set to ln(j+1): P_j = (j+1) / sum(i+1) = 2(j+1)/((t+1)(t+2))."""
    D, t, Hq, Hkv = 128, 9, 4, 2
    q = np.zeros((Hq, D))
    q[:, 0] = 1.0 / SCALE128
    k = np.zeros((t + 1, Hkv, D))
    for j in range(t + 1):
        k[j, :, 0] = math.log(j + 1)
    rng = _rng(2)
    v = rng.standard_normal((t + 1, Hkv, D))
    O, m, l, P = full_attention_row(q, k, v, t, SCALE128)
    p = np.array([2.0 * (j + 1) / ((t + 1) * (t + 2)) for j in range(t + 1)])
    for h in range(Hq):
        if not np.allclose(P[h], p, rtol=1e-12, atol=0):
            return "P != closed form"
        g = h // (Hq // Hkv)
        if not np.allclose(O[h], p @ v[:, g, :], rtol=0, atol=1e-12):
            return "O != closed form"
    s = selection_scores(P, Hkv)
    if not np.allclose(s, np.float32(2) * p.astype(np.float32)[None, :], rtol=1e-6, atol=0):
        return "scores of identical heads != G * P"
    return None


def check_uniform_and_single(full_attention_row, selection_scores):
    rng = _rng(3)
    Hq, Hkv, D, N = 8, 2, 16, 40
    q = rng.standard_normal((Hq, D))
    k = np.repeat(rng.standard_normal((1, Hkv, D)), N, axis=0)  # all keys equal
    v = rng.standard_normal((N, Hkv, D))
    for t in (0, 1, 17, N - 1):
        O, m, l, P = full_attention_row(q, k, v, t, 0.25)
        for h in range(Hq):
            g = h // (Hq // Hkv)
            if not np.allclose(O[h], v[:t + 1, g].mean(axis=0), atol=1e-12):
                return "uniform keys: O != mean(V)"
            if t == 0 and not np.array_equal(O[h], v[0, g]):
                return "one visible key: O != v_0"
        s = selection_scores(P, Hkv)
        if not np.allclose(s, (Hq // Hkv) / (t + 1), rtol=1e-6):
            return "uniform keys: scores != G/(t+1)"
    return None


def check_probability_sums(full_attention_row, selection_scores):
    rng = _rng(4)
    Hq, Hkv, D, N = 8, 2, 32, 3000
    q = rng.standard_normal((Hq, D))
    k = rng.standard_normal((N, Hkv, D))
    v = rng.standard_normal((N, Hkv, D))
    O, m, l, P = full_attention_row(q, k, v, N - 1, 0.2)
    if not np.allclose(P.sum(axis=1), 1.0, rtol=1e-12):
        return "a head's probabilities do not sum to 1"
    s = selection_scores(P, Hkv).astype(np.float64)
    if not np.allclose(s.sum(axis=1), Hq // Hkv, rtol=1e-6):
        return "a group's scores do not sum to G"
    return None


def check_gqa_mapping(full_attention_row, selection_scores):
    """Heads 0..G-1 read KV head 0 only: poison KV head 1 and compare with a
    one-KV-head run of the same heads."""
    rng = _rng(5)
    Hq, Hkv, D, N = 4, 2, 8, 10
    q = rng.standard_normal((Hq, D))
    k = rng.standard_normal((N, Hkv, D))
    v = rng.standard_normal((N, Hkv, D))
    kp, vp = k.copy(), v.copy()
    kp[:, 1] = np.nan
    vp[:, 1] = np.nan
    O, m, l, P = full_attention_row(q, kp, vp, N - 1, 0.3)
    O1, _, _, _ = full_attention_row(q[:2], k[:, :1], v[:, :1], N - 1, 0.3)
    if not np.all(np.isfinite(O[:2])) or not np.allclose(O[:2], O1, atol=1e-14):
        return "heads of group 0 read another KV head"
    O2, _, _, _ = full_attention_row(q[2:], k[:, 1:], v[:, 1:], N - 1, 0.3)
    O, _, _, _ = full_attention_row(q, k, v, N - 1, 0.3)
    if not np.allclose(O[2:], O2, atol=1e-14):
        return "heads of group 1 do not read KV head 1"
    return None


def check_causality(full_attention_row, selection_scores):
    rng = _rng(6)
    Hq, Hkv, D, N = 2, 1, 8, 20
    q = rng.standard_normal((Hq, D))
    k = rng.standard_normal((N, Hkv, D))
    v = rng.standard_normal((N, Hkv, D))
    t = 12
    O, _, _, P = full_attention_row(q, k, v, t, 0.3)
    if P.shape[1] != t + 1:
        return "row does not see exactly keys 0..t"
    k2, v2 = k.copy(), v.copy()
    k2[t + 1:] = rng.standard_normal(k2[t + 1:].shape)
    v2[t + 1:] = 100.0
    O2, _, _, _ = full_attention_row(q, k2, v2, t, 0.3)
    if not np.array_equal(O, O2):
        return "keys after t change the output"
    v3 = v.copy()
    v3[t] += 1.0
    O3, _, _, _ = full_attention_row(q, k, v3, t, 0.3)
    if np.allclose(O, O3):
        return "the key at t is not seen"
    return None


def check_shift_and_permutation(full_attention_row, selection_scores):
    rng = _rng(7)
    Hq, Hkv, D, N = 4, 1, 8, 30
    q = rng.standard_normal((Hq, D))
    k = rng.standard_normal((N, Hkv, D))
    v = rng.standard_normal((N, Hkv, D))
    O, _, _, P = full_attention_row(q, k, v, N - 1, 0.5)
    u = rng.standard_normal(D) * 3.0
    Os, _, _, Ps = full_attention_row(q, k + u[None, None, :], v, N - 1, 0.5)
    if not np.allclose(O, Os, atol=1e-12) or not np.allclose(P, Ps, atol=1e-12):
        return "adding one vector to every key changes the output"
    perm = rng.permutation(N)
    Op, _, _, Pp = full_attention_row(q, k[perm], v[perm], N - 1, 0.5)
    if not np.allclose(O, Op, atol=1e-12) or not np.allclose(P[:, perm], Pp, atol=1e-14):
        return "permuting the keys is not an equivariance"
    return None


# --------------------------------------------------------------------------
# selection
# --------------------------------------------------------------------------
def check_topk_brute(topk_select):
    rng = _rng(8)
    for trial in range(60):
        k = int(rng.integers(1, 9))
        w = int(rng.integers(1, 6))
        t = int(rng.integers(0, 40))
        # few distinct values -> many ties across the threshold
        s = rng.integers(0, 4, size=t + 1).astype(np.float32)
        idx, c = topk_select(s, t, k, w)
        ref = brute_topk(s, t, k, w)
        if c != len(ref) or list(idx[:c]) != ref or np.any(idx[c:] != -1) or idx.size != k + w:
            return f"top-k differs from the rank definition (t={t}, k={k}, w={w})"
    return None


def check_topk_structure(topk_select):
    k, w = 1024, 128
    for t in (0, 1, 126, 127, 128, 129, 1150, 1151, 1152, 1153, 1279, 4095):
        s = np.ones(t + 1, np.float32)
        idx, c = topk_select(s, t, k, w)
        win = list(range(max(0, t - w + 1), t + 1))
        if c != min(t + 1, k + w):
            return f"count wrong at t={t}"
        if list(idx[c - len(win):c]) != win:
            return f"window missing at t={t}"
        if np.any(np.diff(idx[:c]) <= 0):
            return f"not ascending at t={t}"
        if t + 1 <= k + w and list(idx[:c]) != list(range(t + 1)):
            return f"short context does not keep everything at t={t}"
        if t + 1 > k + w and list(idx[:k]) != list(range(k)):
            return "equal scores do not keep the lowest positions"
    t = 3000
    s = np.arange(t + 1, dtype=np.float32)  # strictly increasing
    idx, c = topk_select(s, t, k, w)
    if list(idx[:k]) != list(range(t - w + 1 - k, t - w + 1)):
        return "increasing scores do not keep the last candidates"
    s = np.zeros(t + 1, np.float32)
    s[5] = -0.0
    s[7] = 1.0
    idx, c = topk_select(s, t, k, w)
    if list(idx[:k]) != list(range(k)):
        return "-0.0 and +0.0 are not one value"
    return None


def check_block_brute(block_select):
    rng = _rng(9)
    for trial in range(60):
        nbk = int(rng.integers(1, 5))
        blk = int(rng.integers(1, 6))
        w = int(rng.integers(1, 6))
        t = int(rng.integers(0, 50))
        s = rng.integers(0, 4, size=t + 1).astype(np.float32)
        idx, c = block_select(s, t, nbk, blk, w)
        ref = brute_blocks(s, t, nbk, blk, w)
        if c != len(ref) or list(idx[:c]) != ref or np.any(idx[c:] != -1):
            return f"block select differs from the rank definition (t={t})"
    t = 5000
    idx, c = block_select(np.ones(t + 1, np.float32), t, 16, 64, 128)
    if list(idx[:1024]) != list(range(1024)) or c != 1152:
        return "equal scores do not keep blocks 0..15"
    s = np.zeros(t + 1, np.float32)
    s[t - 128] = 5.0  # last candidate: its block is cut by the window
    idx, c = block_select(s, t, 16, 64, 128)
    b = (t - 128) // 64
    if (t - 128) not in idx[:c] or (t - 127) in idx[:c - 128] or c != 15 * 64 + (t - 128 - 64 * b + 1) + 128:
        return "partial block at the window edge handled wrongly"
    return None


# --------------------------------------------------------------------------
# sparse attention
# --------------------------------------------------------------------------
def check_sparse_equals_full(full_attention_row, sparse_attention_row, topk_select, selection_scores):
    rng = _rng(10)
    Hq, Hkv, D = 4, 2, 16
    for N in (1, 50, 1152):
        q = rng.standard_normal((Hq, D))
        ql = rng.standard_normal((Hq, D))
        k = rng.standard_normal((N, Hkv, D))
        v = rng.standard_normal((N, Hkv, D))
        t = N - 1
        O, _, _, P = full_attention_row(q, k, v, t, 0.3)
        s = selection_scores(P, Hkv)
        sets = []
        for g in range(Hkv):
            idx, c = topk_select(s[g], t, 1024, 128)
            sets.append(idx[:c])
        Os = sparse_attention_row(q, k, v, sets, 0.3)
        if not np.allclose(Os, O, atol=1e-12):
            return f"sparse != full with the whole context selected (N={N})"
        Ofl, _, _, _ = full_attention_row(ql, k, v, t, 0.3)
        if not np.allclose(sparse_attention_row(ql, k, v, sets, 0.3), Ofl, atol=1e-12):
            return "sparse != full for a reuse-layer query"
    return None


def check_sparse_brute(sparse_attention_row):
    rng = _rng(11)
    Hq, Hkv, D, N = 4, 2, 6, 30
    q = rng.standard_normal((Hq, D))
    k = rng.standard_normal((N, Hkv, D))
    v = rng.standard_normal((N, Hkv, D))
    sets = [np.array([0, 3, 4, 17, 29]), np.array([2, 8])]
    O = sparse_attention_row(q, k, v, sets, 0.4)
    Ob, _ = brute_attention(q, k, v, N - 1, 0.4, keys=sets)
    if not np.allclose(O, np.array(Ob), atol=1e-12):
        return "sparse differs from brute force on a subset"
    return None
