"""A decode step through several Hybrid Blocks, captured in one CUDA graph.

Source: "Xiaomi Unveils HySparse2 for Faster Long-Context AI", section
"Two-Level KV Sharing": the Cross-Decoder is built from Hybrid Blocks (one Full
Attention layer followed by Sparse Attention layers), and each of its Full
Attention layers owns a KV cache (KV Bridging) that the block's sparse layers
reuse with the block's token selection (KV Reuse).

Per block, in order on one stream: hs2_kv_append (the step's new K/V rows into
that block's cache), then the block's full attention with scores, selection and
sparse layers (``HybridBlockStep.run``).  The blocks are independent here: in a
model, block i+1's queries come from block i's output through layers this path
does not include, so each block takes its own queries as inputs.

``capture()`` records the whole step once in a CUDA graph (after one eager run,
which also prepares the library for the device); ``replay()`` launches it.
The shapes are fixed by the graph: a step with longer caches needs a new
``MultiBlockDecodeStep`` (or a new capture).  This module owns buffers and
launch order only; every step runs in the library's kernels.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import hs2
from .block import HybridBlockStep


@dataclass
class BlockInputs:
    K: torch.Tensor        # [total_kv, Hkv, D] the block's cache (updated in place)
    V: torch.Tensor
    K_new: torch.Tensor    # [total_q, Hkv, D] the step's new rows
    V_new: torch.Tensor
    Q: torch.Tensor        # [total_q, Hq, D] full-attention queries
    Q_layers: list         # L x [total_q, Hq, D] sparse-layer queries


class MultiBlockDecodeStep:
    """``n_blocks`` Hybrid Blocks of the same shape, each with its own cache."""

    def __init__(self, n_blocks: int, *block_args, **block_kwargs):
        self.blocks = [HybridBlockStep(*block_args, **block_kwargs) for _ in range(n_blocks)]
        self.graph = None
        self.inputs = None

    def run(self, inputs: list, stream=None):
        """Launches the step eagerly on ``stream`` (no synchronisation)."""
        outs = []
        for blk, x in zip(self.blocks, inputs):
            hs2.hs2_kv_append(blk.problem, x.K_new, x.V_new, x.K, x.V, stream)
            outs.append(blk.run(x.Q, x.K, x.V, x.Q_layers, stream))
        return outs

    def capture(self, inputs: list):
        """Records ``run(inputs)`` in a CUDA graph; the input tensors are bound to it."""
        self.inputs = inputs
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self.run(inputs)  # first call on the device happens outside the capture
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            outs = self.run(inputs)
        return outs

    def replay(self):
        self.graph.replay()

    def launches_per_step(self) -> int:
        return sum(1 + blk.launches_per_step() for blk in self.blocks)
