"""Oracle: full attention with selection scores, and sparse attention (float64).

Test infrastructure only (see the package docstring).

Notation: a query row sits at absolute position ``t`` of its sequence and sees
keys 0..t (causal).  Query head ``h`` reads KV head ``g = h // G`` with
``G = Hq / Hkv`` (grouped-query attention).  ``scale`` multiplies q.k.
"""
from __future__ import annotations

import numpy as np


def full_attention_row(q_row: np.ndarray, k_seq: np.ndarray, v_seq: np.ndarray,
                       t: int, scale: float):
    """Full causal attention of one query token.

    q_row [Hq, D], k_seq / v_seq [N, Hkv, D] (float64), t = query position.
    Returns (O [Hq, D], m [Hq], l [Hq], P [Hq, t+1]) where, for each head h,
    x_j = scale * q_h . k_{g,j}, m = max_j x_j, l = sum_j exp(x_j - m),
    P_j = exp(x_j - m) / l and O = sum_j P_j v_{g,j}.
    A row with no visible key (t < 0) gives O = 0 and an empty P.
    """
    Hq, D = q_row.shape
    Hkv = k_seq.shape[1]
    G = Hq // Hkv
    n = t + 1
    if n <= 0:
        return (np.zeros((Hq, D)), np.full(Hq, -np.inf), np.zeros(Hq), np.zeros((Hq, 0)))
    O = np.empty((Hq, D))
    m = np.empty(Hq)
    l = np.empty(Hq)
    P = np.empty((Hq, n))
    for g in range(Hkv):
        Kg = k_seq[:n, g, :]          # [n, D]
        Vg = v_seq[:n, g, :]
        for h in range(g * G, (g + 1) * G):
            x = scale * (Kg @ q_row[h])          # [n]
            m[h] = x.max()
            e = np.exp(x - m[h])
            l[h] = e.sum()
            P[h] = e / l[h]
            O[h] = P[h] @ Vg
    return O, m, l, P


def selection_scores(P: np.ndarray, Hkv: int) -> np.ndarray:
    """Per-KV-group key scores s_g[j] = sum over the group's heads of P[h, j].

    P [Hq, n] from ``full_attention_row``.  The sum is taken in float64 and
    the result is stored as float32, the precision selection works on.
    Returns [Hkv, n] float32.
    """
    Hq, n = P.shape
    G = Hq // Hkv
    s = np.empty((Hkv, n))
    for g in range(Hkv):
        s[g] = P[g * G:(g + 1) * G].sum(axis=0)
    return s.astype(np.float32)


def sparse_attention_row(q_row: np.ndarray, k_seq: np.ndarray, v_seq: np.ndarray,
                         idx_per_group, scale: float) -> np.ndarray:
    """One sparse-attention layer for one query token.

    idx_per_group[g] lists the selected key positions of KV group g (the
    window included).  Each head of group g attends, with its own query, to
    exactly those rows of the shared cache:
    O_h = sum_{j in I_g} softmax_{I_g}(scale * q_h . k_j) v_j.
    An empty index set gives O_h = 0.
    """
    Hq, D = q_row.shape
    Hkv = k_seq.shape[1]
    G = Hq // Hkv
    O = np.zeros((Hq, D))
    for g in range(Hkv):
        I = np.asarray(idx_per_group[g], dtype=np.int64)
        if I.size == 0:
            continue
        Kg = k_seq[I, g, :]
        Vg = v_seq[I, g, :]
        for h in range(g * G, (g + 1) * G):
            x = scale * (Kg @ q_row[h])
            e = np.exp(x - x.max())
            O[h] = (e / e.sum()) @ Vg
    return O


def _seq_of_rows(q_offsets: np.ndarray) -> np.ndarray:
    return np.repeat(np.arange(len(q_offsets) - 1), np.diff(q_offsets))


def run_full_attention(q, k, v, q_offsets, kv_offsets, Hkv: int, scale: float, rows=None):
    """Full attention + scores for the listed query rows (all rows by default).

    q [sum Tq, Hq, D], k / v [sum kv, Hkv, D] (float64), offsets int64 [B+1].
    Query row r of sequence b with kv length N and q length Tq sits at
    t = N - Tq + (r - q_offsets[b]).
    Returns a dict row -> (O [Hq, D], m, l, scores [Hkv, t+1] float32, t).
    """
    q_offsets = np.asarray(q_offsets)
    kv_offsets = np.asarray(kv_offsets)
    seq = _seq_of_rows(q_offsets)
    rows = range(q.shape[0]) if rows is None else rows
    out = {}
    for r in rows:
        b = int(seq[r])
        N = int(kv_offsets[b + 1] - kv_offsets[b])
        Tq = int(q_offsets[b + 1] - q_offsets[b])
        t = N - Tq + (r - int(q_offsets[b]))
        ks = k[kv_offsets[b]:kv_offsets[b + 1]]
        vs = v[kv_offsets[b]:kv_offsets[b + 1]]
        O, m, l, P = full_attention_row(q[r], ks, vs, t, scale)
        out[r] = (O, m, l, selection_scores(P, Hkv), t)
    return out


def run_sparse_attention(q_l, k, v, q_offsets, kv_offsets, idx, count, scale: float, rows=None):
    """Sparse attention of one reuse layer for the listed query rows.

    idx [sum Tq, Hkv, S] int32 (padded with -1), count [sum Tq, Hkv].
    Returns a dict row -> O [Hq, D].
    """
    q_offsets = np.asarray(q_offsets)
    kv_offsets = np.asarray(kv_offsets)
    seq = _seq_of_rows(q_offsets)
    rows = range(q_l.shape[0]) if rows is None else rows
    Hkv = k.shape[1]
    out = {}
    for r in rows:
        b = int(seq[r])
        ks = k[kv_offsets[b]:kv_offsets[b + 1]]
        vs = v[kv_offsets[b]:kv_offsets[b + 1]]
        sets = [idx[r, g, :int(count[r, g])] for g in range(Hkv)]
        out[r] = sparse_attention_row(q_l[r], ks, vs, sets, scale)
    return out
