"""Oracle: the KV cache update of a decode or chunk step (test infrastructure).

Test infrastructure only (see the package docstring).

A Hybrid Block's full-attention layer owns the KV cache that its sparse layers
reuse; each Full Attention layer of the Cross-Decoder builds its own cache
("Xiaomi Unveils HySparse2 for Faster Long-Context AI", section "Two-Level KV
Sharing": KV Bridging and KV Reuse).  A step adds its new tokens' K/V rows to
that cache.  The position convention is the path's: query row i of a sequence
with cache length N and Tq new tokens sits at t = N - Tq + i, sees positions
0..t, and its own key is cache position t.
"""
from __future__ import annotations

import numpy as np


def kv_append(K: np.ndarray, V: np.ndarray, K_new: np.ndarray, V_new: np.ndarray,
              q_offsets, kv_offsets):
    """The cache after the step's new rows are written at their own positions.

    K, V [total_kv, Hkv, D]; K_new, V_new [total_q, Hkv, D]; offsets are the
    per-sequence prefix sums (B + 1 entries).  Returns new arrays (the inputs
    are not modified): for every sequence b and query row i of it,
    row kv_offsets[b] + (N_b - Tq_b + i) takes K_new / V_new row q_offsets[b] + i.
    """
    K = np.array(K, copy=True)
    V = np.array(V, copy=True)
    qo = np.asarray(q_offsets, dtype=np.int64)
    ko = np.asarray(kv_offsets, dtype=np.int64)
    for b in range(len(ko) - 1):
        n_kv = int(ko[b + 1] - ko[b])
        n_q = int(qo[b + 1] - qo[b])
        for i in range(n_q):
            t = n_kv - n_q + i
            K[ko[b] + t] = K_new[qo[b] + i]
            V[ko[b] + t] = V_new[qo[b] + i]
    return K, V
