"""Oracle: KV Bridging, the cache of a Cross-Decoder full-attention layer from
Self-Decoder hidden states (test infrastructure).

Test infrastructure only (see the package docstring).

"Xiaomi Unveils HySparse2 for Faster Long-Context AI", section "Two-Level KV
Sharing" (KV Bridging): each Full Attention layer of the Cross-Decoder builds
its KV cache from the hidden states of the corresponding Full Attention layer
of the Self-Decoder.  Read as the usual key and value projections of those
hidden states: K = H W_K, V = H W_V.  The pages give neither the hidden size
nor the weights.
"""
from __future__ import annotations

import numpy as np


def kv_bridge(H: np.ndarray, Wk_t: np.ndarray, Wv_t: np.ndarray, Hkv: int, D: int):
    """K and V [N, Hkv, D] (float64) from hidden states H [N, hidden] and the
    transposed projections Wk_t, Wv_t [Hkv*D, hidden]:
    K[n, g, d] = sum_i H[n, i] * Wk_t[g*D + d, i] (V likewise)."""
    H = np.asarray(H, dtype=np.float64)
    N = H.shape[0]
    K = (H @ np.asarray(Wk_t, dtype=np.float64).T).reshape(N, Hkv, D)
    V = (H @ np.asarray(Wv_t, dtype=np.float64).T).reshape(N, Hkv, D)
    return K, V
