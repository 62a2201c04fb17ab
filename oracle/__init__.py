"""CPU oracle for the HySparse2 hybrid-block attention path (test infrastructure).

This package is test infrastructure, not part of the product.  Only the tests,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
or run it.  The CUDA library never calls it and shares no code with it.

It is the plain definition of each step, in float64 with numpy, one query row
at a time, with no blocking, fusion or reordering beyond what the definitions
state.  Sources (page title, then section):

* ``full_attention_row``   - causal softmax attention of one query token over the
  whole shared KV cache: the Full Attention layer of a Hybrid Block.
  "Xiaomi Releases HySparse2, Targeting Long-Horizon Reasoning for Agents",
  section "From Hybrid SWA to HySparse2, Xiaomi Continues to Refine the
  Attention Structure"; "Xiaomi Unveils HySparse2 for Faster Long-Context AI",
  section "Two-Level KV Sharing" (KV Reuse).
* ``selection_scores``     - per-(query, KV group) key importance.  The pages say
  only that the full-attention layer also "determines which tokens are
  important" (same sections).  Declared reading: the sum over the group's
  query heads of that layer's attention probabilities.
* ``topk_select``          - token-level selection of the 1024 highest-scoring
  tokens outside the 128 most recent ones, which are always kept.
  "Xiaomi Unveils HySparse2 for Faster Long-Context AI", section "Token-Level
  Selection and Unified Local Access"; "Xiaomi discloses MiMo-V3 plans to adopt
  HySparse2 architecture", section "Article".
* ``block_select``         - the first-generation (HySparse) block-level
  selection, kept as a comparison path: 64-token groups retained whole.
  "Xiaomi discloses MiMo-V3 plans to adopt HySparse2 architecture", section
  "Article".
* ``sparse_attention_row`` - one sparse-attention layer reusing the cache and the
  index set: softmax attention restricted to the selected rows.  "Xiaomi
  Unveils HySparse2 for Faster Long-Context AI", sections "Two-Level KV
  Sharing" (KV Reuse) and "Token-Level Selection and Unified Local Access".
* ``kv_append``            - a step's new K/V rows written into the cache at the
  tokens' own positions, the cache each Full Attention layer of the
  Cross-Decoder owns.  "Xiaomi Unveils HySparse2 for Faster Long-Context AI",
  section "Two-Level KV Sharing" (KV Bridging, KV Reuse).

* ``swa_attention_row``    - sliding-window attention, the local layer of the
  Hybrid SWA baseline the pages compare against.  "Xiaomi Releases HySparse2,
  Targeting Long-Horizon Reasoning for Agents", section "From Hybrid SWA to
  HySparse2, Xiaomi Continues to Refine the Attention Structure".

* ``kv_bridge``            - KV Bridging: a Cross-Decoder layer's K and V from the
  Self-Decoder's hidden states, K = H W_K, V = H W_V.  "Xiaomi Unveils
  HySparse2 for Faster Long-Context AI", section "Two-Level KV Sharing".

Every function is pinned by ``tests/test_oracle_pins.py`` (``kv_append`` by
``tests/test_kv_append_pins.py``, ``swa_attention_row`` by
``tests/test_swa_pins.py``, ``kv_bridge`` by ``tests/test_bridge_pins.py``)
against closed forms, invariants and brute force on tiny inputs.
"""
from .attention import (full_attention_row, selection_scores, sparse_attention_row,
                        run_full_attention, run_sparse_attention)
from .selection import topk_select, block_select, candidate_count, window_range
from .cache import kv_append
from .swa import swa_attention_row
from .bridge import kv_bridge

__all__ = [
    "full_attention_row", "selection_scores", "sparse_attention_row",
    "run_full_attention", "run_sparse_attention",
    "topk_select", "block_select", "candidate_count", "window_range",
    "kv_append", "swa_attention_row", "kv_bridge",
]
