"""Helpers of the GPU parity tests: run the CUDA path on a synthetic workload
and compare it with the CPU oracle on the same stored input values."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth
from long_context_full_b200 import hs2
from long_context_full_b200.block import HybridBlockStep

# Tolerances.  bf16 and fp32 outputs: the stated bounds (fp32 made row-relative,
# because element-wise relative error is unbounded near zero).  Scores: from the
# fp32 arithmetic - logits are fp32 sums of 128 exact bf16 products (~1e-7),
# exponentials within 2 ulp, row sums split into independent partials, at most
# G rounded terms per score - about 2e-6, with a 10x margin.  Index sets: the
# stated near-tie rule.
BF16_O_ABS = 2e-2        # bf16 I/O, fp32 accumulation: max |dO| per element
F32_O_REL = 1e-5         # fp32 build: max |dO| / max |O_ref| per (query, head) row
SCORE_REL = 2e-5         # selection scores: |ds| <= SCORE_REL * s_ref (+ tiny absolute floor)
TIE_REL = 1e-6           # index sets may differ only at near-ties of relative gap < 1e-6


def torch_dtype(dtype: str):
    return torch.bfloat16 if dtype == "bf16" else torch.float32


def to_device(a: np.ndarray, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def to_f64(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        bits = t.detach().cpu().view(torch.int16).numpy().view(np.uint16)
        return synth.bf16_bits_to_f32(bits).astype(np.float64)
    return t.detach().cpu().numpy().astype(np.float64)


class CudaPathRun:
    """The CUDA path on one workload: full attention + scores, selection, sparse layers."""

    def __init__(self, w: synth.Workload, select: str = "token"):
        self.w = w
        self.step = HybridBlockStep(w.Hq, w.Hkv, w.D, torch_dtype(w.dtype), w.q_lens, w.kv_lens,
                                    w.n_layers, k=w.topk, window=w.window, select=select,
                                    n_blocks=w.n_blocks, block=w.block)
        self.Q = to_device(w.q, w.dtype)
        self.K = to_device(w.k, w.dtype)
        self.V = to_device(w.v, w.dtype)
        self.QL = [to_device(x, w.dtype) for x in w.q_layers]

    def run(self):
        out = self.step.run(self.Q, self.K, self.V, self.QL)
        torch.cuda.synchronize()
        err = hs2.hs2_get_last_device_error()
        assert err == hs2.HS2_OK, hs2.status_string(err)
        return out


class OracleRows:
    """Oracle results per query row, converting each sequence's cache once."""

    def __init__(self, w: synth.Workload):
        self.w = w
        self.ko = w.kv_offsets
        self.qo = w.q_offsets
        self.seq = w.query_seq()
        self.tpos = w.query_positions()
        self._kv = {}

    def kv(self, b: int):
        if b not in self._kv:
            self._kv.clear()
            w = self.w
            self._kv[b] = (synth.stored_to_f64(w.k[self.ko[b]:self.ko[b + 1]], w.dtype),
                           synth.stored_to_f64(w.v[self.ko[b]:self.ko[b + 1]], w.dtype))
        return self._kv[b]

    def full(self, r: int):
        """(O [Hq, D], scores [Hkv, t+1] float32, t) of query row r."""
        b = int(self.seq[r])
        k, v = self.kv(b)
        t = int(self.tpos[r])
        q = synth.stored_to_f64(self.w.q[r], self.w.dtype)
        O, m, l, P = oracle.full_attention_row(q, k, v, t, self.w.scale)
        return O, oracle.selection_scores(P, self.w.Hkv), t

    def sparse(self, r: int, layer: int, sets):
        b = int(self.seq[r])
        k, v = self.kv(b)
        q = synth.stored_to_f64(self.w.q_layers[layer][r], self.w.dtype)
        return oracle.sparse_attention_row(q, k, v, sets, self.w.scale)


def check_O(got: np.ndarray, ref: np.ndarray, dtype: str, what: str) -> float:
    """got/ref [Hq, D]; returns the error measure and asserts the tolerance."""
    if dtype == "bf16":
        err = float(np.abs(got - ref).max())
        assert err <= BF16_O_ABS, f"{what}: max |dO| {err:.3g} > {BF16_O_ABS}"
        return err
    den = np.maximum(np.abs(ref).max(axis=1), 1e-30)
    err = float((np.abs(got - ref).max(axis=1) / den).max())
    assert err <= F32_O_REL, f"{what}: max row-relative |dO| {err:.3g} > {F32_O_REL}"
    return err


def check_scores(got: np.ndarray, ref: np.ndarray, what: str) -> float:
    """got/ref: scores of the visible positions of one row."""
    got = got.astype(np.float64)
    ref = ref.astype(np.float64)
    tol = SCORE_REL * np.abs(ref) + 1e-30
    rel = np.abs(got - ref) / np.maximum(np.abs(ref), 1e-30)
    bad = np.abs(got - ref) > tol
    assert not bad.any(), f"{what}: {int(bad.sum())} scores off, worst rel {rel.max():.3g}"
    return float(rel.max()) if rel.size else 0.0


def check_index_sets(gidx, gcnt, oidx, ocnt, oscores, t, k, window, what):
    """End-to-end rule: the window part is identical and every position in the
    symmetric difference of the global parts has an oracle score within
    TIE_REL * s* of s*, the oracle's k-th highest candidate score."""
    assert gcnt == ocnt, f"{what}: count {gcnt} != {ocnt}"
    wlen = min(t + 1, window)
    assert list(gidx[gcnt - wlen:gcnt]) == list(oidx[ocnt - wlen:ocnt]), f"{what}: window differs"
    assert np.all(gidx[gcnt:] == -1), f"{what}: padding"
    g = set(gidx[:gcnt - wlen].tolist())
    o = set(oidx[:ocnt - wlen].tolist())
    diff = g ^ o
    if not diff:
        return 0
    nc = max(0, t - window + 1)
    s = np.asarray(oscores[:nc], np.float64)
    sstar = np.sort(s)[::-1][k - 1]
    for j in diff:
        assert abs(s[j] - sstar) <= TIE_REL * sstar, \
            f"{what}: position {j} (score {s[j]:.9g}) differs away from the threshold {sstar:.9g}"
    return len(diff)


def check_block_sets(gidx, gcnt, oidx, ocnt, oscores, t, n_blocks, block, window, what):
    """End-to-end rule of the block path (the token rule lifted to blocks): the
    window part is identical; the global part is a union of whole candidate
    blocks (their positions below t - window + 1), ascending; and every block in
    the symmetric difference of the GPU's and the oracle's block sets has an
    oracle block score within TIE_REL * b* of b*, the n_blocks-th highest
    eligible block score.  Counts then agree unless a near-tie swapped the
    partial block at the window's edge for a whole one."""
    wlen = min(t + 1, window)
    assert list(gidx[gcnt - wlen:gcnt]) == list(oidx[ocnt - wlen:ocnt]), f"{what}: window differs"
    assert np.all(gidx[gcnt:] == -1), f"{what}: padding"
    nc = max(0, t - window + 1)
    glob = np.asarray(gidx[:gcnt - wlen], np.int64)
    assert np.all(np.diff(glob) > 0) and (glob.size == 0 or (glob[0] >= 0 and glob[-1] < nc)), \
        f"{what}: global part not ascending candidates"
    gb = sorted(set((glob // block).tolist()))
    whole = np.concatenate([np.arange(b * block, min((b + 1) * block, nc)) for b in gb]) \
        if gb else np.zeros(0, np.int64)
    assert np.array_equal(glob, whole), f"{what}: blocks not kept whole"
    ob = sorted(set((np.asarray(oidx[:ocnt - wlen], np.int64) // block).tolist()))
    assert len(gb) == len(ob), f"{what}: {len(gb)} blocks != {len(ob)}"
    diff = set(gb) ^ set(ob)
    if not diff:
        assert gcnt == ocnt, f"{what}: count {gcnt} != {ocnt}"
        return 0
    s = np.asarray(oscores[:nc], np.float64)
    nb = (nc + block - 1) // block
    bscore = np.array([s[b * block:min((b + 1) * block, nc)].max() for b in range(nb)])
    bstar = np.sort(bscore)[::-1][n_blocks - 1]
    for b in diff:
        assert abs(bscore[b] - bstar) <= TIE_REL * bstar, \
            f"{what}: block {b} (score {bscore[b]:.9g}) differs away from the threshold {bstar:.9g}"
    return len(diff)


def gpu_select_on(scores_rows: np.ndarray, ts, k=1024, window=128, block_mode=False,
                  n_blocks=16, block=64, stride=None):
    """Runs the GPU selection on given float32 score rows (one query row per
    sequence, Hkv = 1).  ts: position t of each row; stride: row stride of the
    score buffer (default: the row length rounded up to 4).  Returns (idx, count)."""
    R = len(ts)
    kv_lens = np.asarray(ts, np.int64) + 1
    if stride is None:
        stride = max(1, (scores_rows.shape[1] + 3) // 4 * 4)
    S = np.zeros((R, stride), np.float32)
    S[:, :scores_rows.shape[1]] = scores_rows
    qo = torch.arange(R + 1, dtype=torch.int64).cuda()
    ko = torch.from_numpy(np.concatenate([[0], np.cumsum(kv_lens)]).astype(np.int64)).cuda()
    p = hs2.make_problem(R, 1, 1, 128, hs2.HS2_BF16, qo, ko, R, int(kv_lens.sum()), 1,
                         int(kv_lens.max()), 0.1)
    st = torch.from_numpy(S).cuda()
    width = (n_blocks * block + window) if block_mode else (k + window)
    idx = torch.full((R, width), 7777, dtype=torch.int32).cuda()
    cnt = torch.full((R,), 7777, dtype=torch.int32).cuda()
    if block_mode:
        ws = torch.empty(hs2.hs2_block_select_workspace_size(p, n_blocks, block, window),
                         dtype=torch.uint8).cuda()
        hs2.hs2_block_select(p, st, stride, n_blocks, block, window, idx, cnt, ws)
    else:
        ws = torch.empty(hs2.hs2_topk_workspace_size(p, k, window), dtype=torch.uint8).cuda()
        hs2.hs2_topk_select(p, st, stride, k, window, idx, cnt, ws)
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
    return idx.cpu().numpy(), cnt.cpu().numpy()
