"""One Hybrid Block step through the hs2 C ABI: the full-attention layer with
its selection scores, token-level top-k selection, and L sparse-attention
layers that reuse the same KV cache and index set (KV Reuse).

Source: "Xiaomi Unveils HySparse2 for Faster Long-Context AI", section
"Two-Level KV Sharing" (a Hybrid Block is one Full Attention layer followed by
Sparse Attention layers that reuse its KV cache and selection) and section
"Token-Level Selection and Unified Local Access" (1024 global + 128 local).

This module owns device buffers (torch allocations) and calls the C ABI in
order on one stream; it does no arithmetic of its own.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from . import hs2


@dataclass
class StepOutputs:
    O: torch.Tensor            # [total_q, Hq, D] full-attention output
    scores: torch.Tensor       # [total_q * Hkv, stride] float32
    idx: torch.Tensor          # [total_q * Hkv, k + window] int32
    count: torch.Tensor        # [total_q * Hkv] int32
    O_layers: list             # L x [total_q, Hq, D] sparse-layer outputs


class HybridBlockStep:
    """Buffers and launch sequence of one hybrid-block step for a fixed batch shape.

    q_lens / kv_lens: per-sequence query and cache lengths (host ints).
    dtype: torch.bfloat16 or torch.float32 (Q, K, V and outputs).
    select: "token" (HySparse2) or "block" (first-generation comparison path).
    """

    def __init__(self, Hq: int, Hkv: int, D: int, dtype, q_lens, kv_lens, n_layers: int,
                 k: int = 1024, window: int = 128, select: str = "token",
                 n_blocks: int = 16, block: int = 64, scale: float | None = None,
                 device: str | torch.device = "cuda"):
        self.device = torch.device(device)
        q_lens = np.asarray(q_lens, dtype=np.int64)
        kv_lens = np.asarray(kv_lens, dtype=np.int64)
        self.B = len(kv_lens)
        self.Hq, self.Hkv, self.D, self.dtype = Hq, Hkv, D, dtype
        self.k, self.window, self.n_layers = k, window, n_layers
        self.select, self.n_blocks, self.block = select, n_blocks, block
        self.total_q = int(q_lens.sum())
        self.total_kv = int(kv_lens.sum())
        self.max_q = int(q_lens.max())
        self.max_kv = int(kv_lens.max())
        self.rows = self.total_q * Hkv
        self.scale = float(np.float32(1.0 / np.sqrt(D))) if scale is None else float(scale)
        qo = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int64)
        ko = np.concatenate([[0], np.cumsum(kv_lens)]).astype(np.int64)
        self.q_offsets = torch.from_numpy(qo).to(self.device)
        self.kv_offsets = torch.from_numpy(ko).to(self.device)
        self.problem = hs2.make_problem(self.B, Hq, Hkv, D, dtype, self.q_offsets,
                                        self.kv_offsets, self.total_q, self.total_kv,
                                        self.max_q, self.max_kv, self.scale)
        self.stride = max(1, (self.max_kv + 3) // 4 * 4)
        self.idx_stride = (k + window) if select == "token" else (n_blocks * block + window)
        dev = self.device
        self.O = torch.empty(self.total_q, Hq, D, dtype=dtype, device=dev)
        self.scores = torch.empty(self.rows, self.stride, dtype=torch.float32, device=dev)
        self.idx = torch.empty(self.rows, self.idx_stride, dtype=torch.int32, device=dev)
        self.count = torch.empty(self.rows, dtype=torch.int32, device=dev)
        self.O_layers = [torch.empty(self.total_q, Hq, D, dtype=dtype, device=dev)
                         for _ in range(n_layers)]
        p = self.problem
        sizes = [hs2.hs2_full_attn_workspace_size(p),
                 hs2.hs2_sparse_attn_workspace_size(p, self.idx_stride)]
        if select == "token":
            sizes.append(hs2.hs2_topk_workspace_size(p, k, window))
        else:
            sizes.append(hs2.hs2_block_select_workspace_size(p, n_blocks, block, window))
        # the calls run one after another on one stream: one workspace serves all
        self.ws_bytes = max(sizes)
        self.workspace = torch.empty(max(1, self.ws_bytes), dtype=torch.uint8, device=dev)

    def full_attention(self, Q, K, V, stream=None) -> None:
        hs2.hs2_full_attn_scores(self.problem, Q, K, V, self.O, self.scores, self.stride,
                                 self.workspace, stream)

    def select_tokens(self, stream=None) -> None:
        if self.select == "token":
            hs2.hs2_topk_select(self.problem, self.scores, self.stride, self.k, self.window,
                                self.idx, self.count, self.workspace, stream)
        else:
            hs2.hs2_block_select(self.problem, self.scores, self.stride, self.n_blocks,
                                 self.block, self.window, self.idx, self.count,
                                 self.workspace, stream)

    def sparse_layer(self, l: int, Q_l, K, V, stream=None) -> None:
        hs2.hs2_sparse_attn(self.problem, Q_l, K, V, self.idx, self.count, self.idx_stride,
                            self.O_layers[l], self.workspace, stream)

    def run(self, Q, K, V, Q_layers, stream=None) -> StepOutputs:
        """Launches the whole step on ``stream`` (no synchronisation)."""
        self.full_attention(Q, K, V, stream)
        self.select_tokens(stream)
        for l in range(self.n_layers):
            self.sparse_layer(l, Q_layers[l], K, V, stream)
        return StepOutputs(self.O, self.scores, self.idx, self.count, self.O_layers)

    def launches_per_step(self) -> int:
        """Kernels one ``run`` launches."""
        full = hs2.hs2_full_attn_launches(self.problem)
        sel = 1 if self.select == "token" else 3
        return full + sel + self.n_layers
