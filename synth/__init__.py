"""Seeded synthetic inputs for the hybrid-block attention path.

This module is shared by the tests, the benchmark and the CPU oracle's callers.
It only draws numbers and lays them out; it computes nothing of the attention
method itself (no dot products, softmax, scores or selection).

Generator: numpy's Philox4x32-10 counter-based bit generator (Salmon et al.,
"Parallel random numbers: as easy as 1, 2, 3", SC'11) keyed per stream, with
numpy's standard-normal transform on top.  Every tensor is cut into streams of
``BLOCK_TOKENS`` tokens per sequence, each with its own key
``[seed, tensor_id << 40 | seq << 20 | block]``, so a process that owns a
subset of the sequences (one rank of a data-parallel run) regenerates exactly
the same bits for them, and blocks can be drawn in parallel threads.

Values are drawn as float32 and then stored either as float32 or as bfloat16
(round to nearest even).  Both the CUDA path and the oracle read those stored
bits; the oracle decodes them exactly into float64.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

BLOCK_TOKENS = 8192

# tensor ids of the generator streams
TID_Q = 1
TID_K = 2
TID_V = 3
TID_NEEDLE_NOISE = 4
TID_NEEDLE_POS = 5
TID_LENGTHS = 6
TID_QL_BASE = 100  # reuse layer l draws its query from TID_QL_BASE + l


def _gen(seed: int, tid: int, seq: int, block: int) -> np.random.Generator:
    key = np.array([seed & 0xFFFFFFFFFFFFFFFF, (tid << 40) | (seq << 20) | block],
                   dtype=np.uint64)
    return np.random.Generator(np.random.Philox(key=key))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bits to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def stored_to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 view of stored values ("bf16" = uint16 bits, "f32" = float32)."""
    if dtype == "bf16":
        return bf16_bits_to_f32(a).astype(np.float64)
    return np.asarray(a, dtype=np.float32).astype(np.float64)


def _store(x32: np.ndarray, dtype: str) -> np.ndarray:
    return f32_to_bf16_bits(x32) if dtype == "bf16" else x32.astype(np.float32)


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def normal_tokens(seed: int, tid: int, seq: int, n_tokens: int, row_shape: tuple,
                  dtype: str, out: np.ndarray | None = None) -> np.ndarray:
    """N(0,1) tensor [n_tokens, *row_shape] of one sequence, stored as ``dtype``.

    Token block c of the sequence comes from its own stream, so the result does
    not depend on how many threads draw it.
    """
    row = int(np.prod(row_shape))
    sdt = np.uint16 if dtype == "bf16" else np.float32
    if out is None:
        out = np.empty((n_tokens,) + tuple(row_shape), dtype=sdt)
    flat = out.reshape(n_tokens, row)
    nblk = (n_tokens + BLOCK_TOKENS - 1) // BLOCK_TOKENS

    def one(c: int) -> None:
        a = c * BLOCK_TOKENS
        e = min(n_tokens, a + BLOCK_TOKENS)
        x = _gen(seed, tid, seq, c).standard_normal((e - a) * row, dtype=np.float32)
        flat[a:e] = _store(x, dtype).reshape(e - a, row)

    if nblk <= 1:
        for c in range(nblk):
            one(c)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(one, range(nblk)))
    return out


def ragged_lengths(seed: int, batch: int, lo: int, hi: int) -> np.ndarray:
    """Sequence lengths log-uniform in [lo, hi]: round(exp(U(ln lo, ln hi)))."""
    u = _gen(seed, TID_LENGTHS, 0, 0).random(batch)
    n = np.rint(np.exp(math.log(lo) + u * (math.log(hi) - math.log(lo)))).astype(np.int64)
    return np.clip(n, lo, hi)


@dataclass
class Workload:
    """One synthetic instance of the hybrid-block decode / chunk problem.

    Layout (token-major, packed over sequences):
      q   [sum q_len, Hq, D]     k, v [sum kv_len, Hkv, D]
      q_layers[l] [sum q_len, Hq, D] for reuse layer l
    Arrays hold stored values: uint16 bfloat16 bits or float32.
    """
    name: str
    seed: int
    dtype: str
    Hq: int
    Hkv: int
    D: int
    q_lens: np.ndarray
    kv_lens: np.ndarray
    n_layers: int
    topk: int = 1024
    window: int = 128
    block: int = 64
    n_blocks: int = 16
    q: np.ndarray | None = None
    k: np.ndarray | None = None
    v: np.ndarray | None = None
    q_layers: list = field(default_factory=list)
    needle_pos: np.ndarray | None = None  # [B, n_needles] positions within each sequence

    @property
    def B(self) -> int:
        return int(len(self.kv_lens))

    @property
    def q_offsets(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.q_lens)]).astype(np.int64)

    @property
    def kv_offsets(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.kv_lens)]).astype(np.int64)

    @property
    def scale(self) -> float:
        return float(np.float32(1.0 / math.sqrt(self.D)))

    def query_positions(self) -> np.ndarray:
        """Absolute position t of every query row (query i of a sequence with
        kv_len N and q_len Tq sits at N - Tq + i)."""
        t = []
        for b in range(self.B):
            n, tq = int(self.kv_lens[b]), int(self.q_lens[b])
            t.extend(range(n - tq, n))
        return np.asarray(t, dtype=np.int64)

    def query_seq(self) -> np.ndarray:
        return np.repeat(np.arange(self.B), self.q_lens).astype(np.int64)


def make_workload(name: str, seed: int, dtype: str, Hq: int, Hkv: int, D: int,
                  kv_lens, q_lens, n_layers: int, seq_ids=None,
                  n_needles: int = 0, needle_amp: float = 4.0, needle_std: float = 0.1,
                  window: int = 128, topk: int = 1024) -> Workload:
    """Draw Q, K, V and the reuse-layer queries of a workload.

    ``seq_ids`` gives each local sequence its global index (data-parallel
    shards draw their own sequences with the global stream keys).
    """
    kv_lens = np.asarray(kv_lens, dtype=np.int64)
    q_lens = np.asarray(q_lens, dtype=np.int64)
    B = len(kv_lens)
    seq_ids = np.arange(B) if seq_ids is None else np.asarray(seq_ids)
    sdt = np.uint16 if dtype == "bf16" else np.float32
    w = Workload(name, seed, dtype, Hq, Hkv, D, q_lens, kv_lens, n_layers,
                 topk=topk, window=window)
    tq, tk = int(q_lens.sum()), int(kv_lens.sum())
    w.q = np.empty((tq, Hq, D), dtype=sdt)
    w.k = np.empty((tk, Hkv, D), dtype=sdt)
    w.v = np.empty((tk, Hkv, D), dtype=sdt)
    w.q_layers = [np.empty((tq, Hq, D), dtype=sdt) for _ in range(n_layers)]
    qo, ko = w.q_offsets, w.kv_offsets
    for b in range(B):
        s = int(seq_ids[b])
        normal_tokens(seed, TID_Q, s, int(q_lens[b]), (Hq, D), dtype, w.q[qo[b]:qo[b + 1]])
        normal_tokens(seed, TID_K, s, int(kv_lens[b]), (Hkv, D), dtype, w.k[ko[b]:ko[b + 1]])
        normal_tokens(seed, TID_V, s, int(kv_lens[b]), (Hkv, D), dtype, w.v[ko[b]:ko[b + 1]])
        for l in range(n_layers):
            normal_tokens(seed, TID_QL_BASE + l, s, int(q_lens[b]), (Hq, D), dtype,
                          w.q_layers[l][qo[b]:qo[b + 1]])
    if n_needles:
        plant_needles(w, n_needles, needle_amp, needle_std, seq_ids)
    return w


def plant_needles(w: Workload, n_needles: int, amp: float, std: float, seq_ids) -> None:
    """Overwrite ``n_needles`` key rows per sequence with 'needle' keys.

    Reading of the retrieval workload: for KV head g the needle key is
    amp * q/|q| + N(0, std^2) per element, where q is the sequence's last
    (decode) query of head g*G, the first query head of the group.  The
    positions are drawn uniformly without replacement from [0, N-129] (outside
    the 128-token window) and are shared by all KV heads of the sequence.
    """
    G = w.Hq // w.Hkv
    qo, ko = w.q_offsets, w.kv_offsets
    pos_all = []
    for b in range(w.B):
        s = int(seq_ids[b])
        n = int(w.kv_lens[b])
        hi = n - w.window  # positions 0 .. n-129
        g = _gen(w.seed, TID_NEEDLE_POS, s, 0)
        pos = np.sort(g.choice(hi, size=n_needles, replace=False)).astype(np.int64)
        pos_all.append(pos)
        qrow = stored_to_f64(w.q[qo[b + 1] - 1], w.dtype)  # [Hq, D], decode query
        noise = _gen(w.seed, TID_NEEDLE_NOISE, s, 0).standard_normal(
            (n_needles, w.Hkv, w.D))
        for gi in range(w.Hkv):
            qv = qrow[gi * G]
            unit = qv / np.linalg.norm(qv)
            rows = amp * unit[None, :] + std * noise[:, gi, :]
            stored = _store(rows.astype(np.float32), w.dtype)
            w.k[ko[b] + pos, gi, :] = stored
    w.needle_pos = np.stack(pos_all)


# The five workloads (seed = 1234 + workload number).
def tiny(n_layers: int = 3) -> Workload:
    """B=1, one decode query, context 4096, Hq=4 / Hkv=1, D=128, float32."""
    return make_workload("tiny_4k_f32", 1235, "f32", 4, 1, 128, [4096], [1], n_layers)


def decode_128k(batch: int = 8, first_seq: int = 0, context: int = 131072) -> Workload:
    """Decode batch of 8 sequences x 131072 keys, Hq=32 / Hkv=4, D=128, bf16, 4 reuse layers."""
    ids = np.arange(first_seq, first_seq + batch)
    return make_workload("decode_b8_128k_bf16", 1236, "bf16", 32, 4, 128,
                         [context] * batch, [1] * batch, 4, seq_ids=ids)


def needle_1m(context: int = 1048576, n_needles: int = 64, amp: float = 4.0) -> Workload:
    """One decode query over 1,048,576 keys with 64 planted needle keys, bf16, 4 reuse layers."""
    return make_workload("needle_b1_1m_bf16", 1237, "bf16", 32, 4, 128, [context], [1], 4,
                         n_needles=n_needles, needle_amp=amp)


def chunk_256k(cached: int = 262144, new: int = 2048, n_layers: int = 4) -> Workload:
    """Agent-turn chunk: 2048 new query tokens on a 262,144-token cache, causal, bf16."""
    return make_workload("chunk_262k_plus_2k_bf16", 1238, "bf16", 32, 4, 128,
                         [cached + new], [new], n_layers)


def ragged_16(batch: int = 16, lo: int = 8192, hi: int = 524288) -> Workload:
    """16 decode sequences, lengths log-uniform in [8192, 524288], bf16, 4 reuse layers."""
    lens = ragged_lengths(1239, batch, lo, hi)
    return make_workload("ragged_b16_8k_512k_bf16", 1239, "bf16", 32, 4, 128,
                         lens, [1] * batch, 4)
