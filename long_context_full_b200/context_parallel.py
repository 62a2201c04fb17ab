"""Context-parallel decode step of a Hybrid Block: the KV cache of every
sequence is split by position across ranks (one process per GPU), and the
ranks exchange only small partials.

Rank r holds the contiguous global positions [pos0[b], pos0[b] + n[r][b]) of
sequence b (the ranges of a sequence are ordered by rank and cover it).  One
step, as in the unsplit Hybrid Block (full attention with selection scores,
token top-k plus the window, the sparse reuse layers):

1. ``hs2_cp_attn_partial`` on the rank's rows; all-gather the (m, 1/l, O)
   partials; ``hs2_cp_merge`` gives every rank the full-attention output and
   each head's global softmax max and sum;
2. ``hs2_cp_scores``: selection scores of the rank's own keys;
3. ``hs2_cp_topk_local``: the rank's top-(k + window) as (score, global
   position) pairs; all-gather; ``hs2_cp_topk_merge``: the global index set,
   the same on every rank;
4. each sparse layer: ``hs2_cp_sparse_partial`` over the selected rows the
   rank holds; all-gather; ``hs2_cp_merge``.

Every step runs in the library's kernels; this module owns the buffers and
the order of the calls.  The exchange is a callable ``all_gather(t)`` returning
the ranks' tensors stacked in rank order: ``nccl_all_gather`` over
``torch.distributed`` (NCCL between GPUs), or, with several ranks driven from
one process, ``LocalRanks`` (each rank's kernels run in turn and the stack is
a copy, so no kernel waits for another).

Sources: the Full Attention and Sparse Attention layers of a Hybrid Block and
the token selection ("Xiaomi Releases HySparse2, Targeting Long-Horizon
Reasoning for Agents", section "From Hybrid SWA to HySparse2, ..."; "Xiaomi
Unveils HySparse2 for Faster Long-Context AI", sections "Two-Level KV Sharing"
and "Token-Level Selection and Unified Local Access").  The pages describe one
device; the split is this library's.
"""
from __future__ import annotations

import numpy as np
import torch

from . import hs2


def shard_offsets(shard_lens) -> np.ndarray:
    """pos0[r][b]: first global position of rank r's range of sequence b."""
    n = np.asarray(shard_lens, dtype=np.int64)
    return np.concatenate([np.zeros((1, n.shape[1]), np.int64), np.cumsum(n, axis=0)[:-1]], axis=0)


class ContextParallelDecodeStep:
    """Buffers and calls of one rank.

    shard_lens [world][B]: every rank's number of positions of every sequence
    (each >= 1; a sequence's ranges in rank order make up the sequence).
    dtype: torch.bfloat16 or torch.float32.
    """

    def __init__(self, rank: int, world: int, Hq: int, Hkv: int, D: int, dtype, shard_lens,
                 n_layers: int, k: int = 1024, window: int = 128, scale: float | None = None,
                 device: str | torch.device = "cuda"):
        n = np.asarray(shard_lens, dtype=np.int64)
        if n.ndim != 2 or n.shape[0] != world or (n < 1).any():
            raise ValueError("shard_lens must be [world][B] with every entry >= 1")
        self.rank, self.world = rank, world
        self.B = n.shape[1]
        self.Hq, self.Hkv, self.D, self.dtype = Hq, Hkv, D, dtype
        self.k, self.window, self.n_layers = k, window, n_layers
        self.scale = float(np.float32(1.0 / np.sqrt(D))) if scale is None else float(scale)
        dev = self.device = torch.device(device)
        B = self.B
        local = n[rank]
        glob = n.sum(axis=0)
        qo = np.arange(B + 1, dtype=np.int64)
        lko = np.concatenate([[0], np.cumsum(local)]).astype(np.int64)
        gko = np.concatenate([[0], np.cumsum(glob)]).astype(np.int64)
        self.q_offsets = torch.from_numpy(qo).to(dev)
        self.kv_offsets = torch.from_numpy(lko).to(dev)
        self.kv_offsets_global = torch.from_numpy(gko).to(dev)
        self.pos0 = torch.from_numpy(shard_offsets(n)[rank].copy()).to(dev)
        self.local_lens, self.global_lens = local, glob
        self.problem = hs2.make_problem(B, Hq, Hkv, D, dtype, self.q_offsets, self.kv_offsets, B,
                                        int(local.sum()), 1, int(local.max()), self.scale)
        self.problem_global = hs2.make_problem(B, Hq, Hkv, D, dtype, self.q_offsets,
                                               self.kv_offsets_global, B, int(glob.sum()), 1,
                                               int(glob.max()), self.scale)
        self.rows = B * Hkv
        self.kk = k + window
        self.stride = max(1, (int(local.max()) + 3) // 4 * 4)
        f32, i32 = torch.float32, torch.int32
        self.O_part = torch.empty(B, Hq, D, dtype=f32, device=dev)
        self.ml_part = torch.empty(B, Hq, 2, dtype=f32, device=dev)
        self.O = torch.empty(B, Hq, D, dtype=dtype, device=dev)
        self.ml = torch.empty(B, Hq, 2, dtype=f32, device=dev)
        self.scores = torch.empty(self.rows, self.stride, dtype=f32, device=dev)
        self.idx_tmp = torch.empty(self.rows, self.kk, dtype=i32, device=dev)
        self.count_tmp = torch.empty(self.rows, dtype=i32, device=dev)
        self.pair_score = torch.empty(self.rows, self.kk, dtype=f32, device=dev)
        self.pair_pos = torch.empty(self.rows, self.kk, dtype=i32, device=dev)
        self.idx = torch.empty(self.rows, self.kk, dtype=i32, device=dev)
        self.count = torch.empty(self.rows, dtype=i32, device=dev)
        self.O_layers = [torch.empty(B, Hq, D, dtype=dtype, device=dev) for _ in range(n_layers)]
        self.workspace = torch.empty(max(1, hs2.hs2_full_attn_workspace_size(self.problem)),
                                     dtype=torch.uint8, device=dev)

    # ---- the phases (each launches kernels on ``stream``; no synchronisation)
    def attention_partial(self, Q, K, V, stream=None) -> None:
        hs2.hs2_cp_attn_partial(self.problem, Q, K, V, self.O_part, self.ml_part, self.workspace,
                                stream)

    def attention_merge(self, O_parts, ml_parts, stream=None) -> None:
        hs2.hs2_cp_merge(self.B * self.Hq, self.world, O_parts, ml_parts, self.dtype, self.O,
                         self.ml, stream)

    def local_selection(self, stream=None) -> None:
        hs2.hs2_cp_scores(self.problem, self.ml, self.scores, self.stride, self.workspace, stream)
        hs2.hs2_cp_topk_local(self.problem, self.scores, self.stride, self.k, self.window, self.pos0,
                              self.idx_tmp, self.count_tmp, self.pair_score, self.pair_pos, stream)

    def selection_merge(self, pair_scores, pair_pos, stream=None) -> None:
        hs2.hs2_cp_topk_merge(self.problem_global, self.world, self.k, self.window, pair_scores,
                              pair_pos, self.idx, self.count, stream)

    def sparse_partial(self, Q_l, K, V, stream=None) -> None:
        hs2.hs2_cp_sparse_partial(self.problem, Q_l, K, V, self.idx, self.count, self.kk, self.pos0,
                                  self.O_part, self.ml_part, stream)

    def sparse_merge(self, l: int, O_parts, ml_parts, stream=None) -> None:
        hs2.hs2_cp_merge(self.B * self.Hq, self.world, O_parts, ml_parts, self.dtype,
                         self.O_layers[l], None, stream)

    def run(self, Q, K, V, Q_layers, all_gather, stream=None):
        """One step on this rank; ``all_gather(t)`` stacks the ranks' ``t``.
        Everything, the exchange included, is ordered on ``stream`` (default:
        the current stream)."""
        with torch.cuda.stream(stream):
            self.attention_partial(Q, K, V)
            self.attention_merge(all_gather(self.O_part), all_gather(self.ml_part))
            self.local_selection()
            self.selection_merge(all_gather(self.pair_score), all_gather(self.pair_pos))
            for l in range(self.n_layers):
                self.sparse_partial(Q_layers[l], K, V)
                self.sparse_merge(l, all_gather(self.O_part), all_gather(self.ml_part))
        return self.O, self.scores, self.idx, self.count, self.O_layers


def nccl_all_gather(group=None):
    """all_gather(t) over torch.distributed: the ranks' tensors stacked in rank order."""
    import torch.distributed as dist

    def gather(t: torch.Tensor) -> torch.Tensor:
        world = dist.get_world_size(group)
        parts = [torch.empty_like(t) for _ in range(world)]
        dist.all_gather(parts, t.contiguous(), group=group)
        return torch.stack(parts)
    return gather


class LocalRanks:
    """Several ranks driven from one process on one device: each phase runs for
    every rank in turn, and the exchange stacks the ranks' buffers."""

    def __init__(self, steps):
        self.steps = list(steps)

    def run(self, Q, Ks, Vs, Q_layers, stream=None):
        """One step of every rank, ordered on ``stream`` (default: the current stream)."""
        S = self.steps
        with torch.cuda.stream(stream):
            for r, st in enumerate(S):
                st.attention_partial(Q, Ks[r], Vs[r])
            O_parts = torch.stack([st.O_part for st in S])
            ml_parts = torch.stack([st.ml_part for st in S])
            for st in S:
                st.attention_merge(O_parts, ml_parts)
            for st in S:
                st.local_selection()
            ps = torch.stack([st.pair_score for st in S])
            pp = torch.stack([st.pair_pos for st in S])
            for st in S:
                st.selection_merge(ps, pp)
            for l in range(S[0].n_layers):
                for r, st in enumerate(S):
                    st.sparse_partial(Q_layers[l], Ks[r], Vs[r])
                O_parts = torch.stack([st.O_part for st in S])
                ml_parts = torch.stack([st.ml_part for st in S])
                for st in S:
                    st.sparse_merge(l, O_parts, ml_parts)
