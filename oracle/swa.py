"""Oracle: sliding-window attention, the local layer of the Hybrid SWA baseline
(test infrastructure).

Test infrastructure only (see the package docstring).

"Xiaomi Releases HySparse2, Targeting Long-Horizon Reasoning for Agents",
section "From Hybrid SWA to HySparse2, Xiaomi Continues to Refine the Attention
Structure": the MiMo-V2 models combined a few full-attention layers with
sliding-window layers that attend only to a local neighbourhood.  The pages do
not give the window; it is a parameter here (declared 128 where a value is
needed, the size of HySparse2's forced local window).
"""
from __future__ import annotations

import numpy as np


def swa_attention_row(q_row: np.ndarray, k_seq: np.ndarray, v_seq: np.ndarray, t: int,
                      window: int, scale: float) -> np.ndarray:
    """Causal sliding-window attention of one query token at position t.

    q_row [Hq, D], k_seq / v_seq [N, Hkv, D] (float64).  Each head h of KV
    group g attends to the keys at positions max(0, t - window + 1) .. t:
    O_h = sum_j softmax_j(scale * q_h . k_{g,j}) v_{g,j} over that range.
    No visible key (t < 0 or window < 1) gives O = 0.
    """
    Hq, D = q_row.shape
    Hkv = k_seq.shape[1]
    G = Hq // Hkv
    O = np.zeros((Hq, D))
    lo, hi = max(0, t - window + 1), t + 1
    if hi <= lo:
        return O
    for g in range(Hkv):
        Kg = k_seq[lo:hi, g, :]
        Vg = v_seq[lo:hi, g, :]
        for h in range(g * G, (g + 1) * G):
            x = scale * (Kg @ q_row[h])
            e = np.exp(x - x.max())
            O[h] = (e / e.sum()) @ Vg
    return O
