"""Context-parallel decode across processes on CPU: ``ContextParallelDecodeStep.run``
with its exchange over torch.distributed (gloo, 2 and 3 ranks), every library
call replaced by a float64 stand-in that does what the C ABI documents for it
(include/hs2.h, "Context parallelism for decode") on the rank's own rows, built
from oracle calls.  Every rank must end with the unsplit oracle's full-attention
output, index sets and sparse-layer outputs.  What this covers is the host
side: the order of the calls and exchanges, the shapes the ranks stack, and
that every rank gets the same merged result; the kernels behind the calls are
covered by the GPU tests."""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import synth

B, HQ, HKV, D, LAYERS, K, WINDOW = 2, 8, 2, 128, 2, 256, 32
LENS = [3000, 1700]


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _split(world):
    """shard_lens [world][B]: uneven ranges, the last rank's range of sequence 1
    shorter than the window, so the window spans two ranks."""
    out = []
    for n in LENS:
        cuts = np.linspace(0, n, world + 1).astype(int)
        cuts[-1] = n
        if world > 1:
            cuts[-2] = n - WINDOW // 2  # a last range shorter than the window
        out.append(np.diff(cuts))
    return np.stack(out, axis=1)


class _Stub:
    """float64 stand-ins for the hs2 context-parallel calls of one rank."""

    def __init__(self, w, rank, lens):
        self.w, self.rank, self.lens = w, rank, lens
        self.pos0 = np.concatenate([np.zeros((1, B), np.int64), np.cumsum(lens, axis=0)[:-1]])[rank]
        self.logits = {}  # (b, h) -> the rank's logits, as the kernels keep them in the workspace

    def kv(self, b):
        ko = self.w.kv_offsets
        s = ko[b] + self.pos0[b]
        n = int(self.lens[self.rank][b])
        return (synth.stored_to_f64(self.w.k[s:s + n], "f32"), synth.stored_to_f64(self.w.v[s:s + n], "f32"))

    # hs2_cp_attn_partial: attention over the rank's keys, O normalised by its own sum
    def attn_partial(self, p, Q, K, V, O_part, ml_part, ws, stream=None):
        for b in range(B):
            k, v = self.kv(b)
            q = Q[b].double().numpy()
            O, m, l, P = oracle.full_attention_row(q, k, v, k.shape[0] - 1, self.w.scale)
            O_part[b] = torch.from_numpy(O)
            ml_part[b, :, 0] = torch.from_numpy(m)
            ml_part[b, :, 1] = torch.from_numpy(1.0 / l)
            for h in range(HQ):  # x = m + log(P * l)
                self.logits[(b, h)] = m[h] + np.log(P[h] * l[h])

    # hs2_cp_merge: M = max m_r, w_r = l_r e^(m_r - M), O = sum w_r O_r / sum w_r
    @staticmethod
    def merge(rows, R, O_parts, ml_parts, dtype, O, ml, stream=None):
        Op = O_parts.double().numpy().reshape(R, rows, D)
        mp_ = ml_parts.double().numpy().reshape(R, rows, 2)
        m, il = mp_[..., 0], mp_[..., 1]
        lr = np.where(il > 0, 1.0 / np.where(il > 0, il, 1.0), 0.0)
        M = m.max(axis=0)
        wr = lr * np.exp(np.where(lr > 0, m - M, -np.inf))
        L = wr.sum(axis=0)
        out = (wr[..., None] * Op).sum(axis=0) / L[:, None]
        O.view(rows, D).copy_(torch.from_numpy(out).to(O.dtype))
        if ml is not None:
            ml.view(rows, 2)[:, 0] = torch.from_numpy(M)
            ml.view(rows, 2)[:, 1] = torch.from_numpy(1.0 / L)

    # hs2_cp_scores: scores of the rank's keys with the global (M, 1/L)
    def scores(self, p, ml, scores, stride, ws, stream=None):
        G = HQ // HKV
        mln = ml.double().numpy()
        for b in range(B):
            n = int(self.lens[self.rank][b])
            for g in range(HKV):
                s = sum(np.exp(self.logits[(b, h)] - mln[b, h, 0]) * mln[b, h, 1]
                        for h in range(g * G, (g + 1) * G))
                scores[b * HKV + g, :n] = torch.from_numpy(s.astype(np.float32))

    # hs2_cp_topk_local: the rank's top-(k + window) over all its positions
    def topk_local(self, p, scores, stride, k, window, pos0, idx_tmp, count_tmp, ps, pp, stream=None):
        kk = k + window
        for b in range(B):
            n = int(self.lens[self.rank][b])
            for g in range(HKV):
                r = b * HKV + g
                s = scores[r, :n].numpy().astype(np.float64)
                order = np.lexsort((np.arange(n), -s))[:kk]
                ps[r] = 0.0
                pp[r] = -1
                ps[r, :order.size] = torch.from_numpy(s[order].astype(np.float32))
                pp[r, :order.size] = torch.from_numpy((order + self.pos0[b]).astype(np.int32))

    # hs2_cp_topk_merge: positions <= t - window compete; k best, ascending; then the window
    @staticmethod
    def topk_merge(p, R, k, window, pair_scores, pair_pos, idx, count, stream=None):
        for b in range(B):
            t = sum(LENS[b:b + 1]) - 1
            for g in range(HKV):
                r = b * HKV + g
                pos = pair_pos[:, r].reshape(-1).numpy()
                sc = pair_scores[:, r].reshape(-1).numpy()
                keep = (pos >= 0) & (pos <= t - window)
                full = np.full(t + 1, -np.inf, np.float32)
                full[pos[keep]] = sc[keep]
                oi, oc = oracle.topk_select(full, t, k, window)
                idx[r] = torch.from_numpy(oi)
                count[r] = oc

    # hs2_cp_sparse_partial: attention over the listed positions the rank holds
    def sparse_partial(self, p, Q_l, K, V, idx, count, kk, pos0, O_part, ml_part, stream=None):
        G = HQ // HKV
        for b in range(B):
            k, v = self.kv(b)
            n = k.shape[0]
            q = Q_l[b].double().numpy()
            for g in range(HKV):
                r = b * HKV + g
                lst = idx[r, :int(count[r])].numpy().astype(np.int64) - self.pos0[b]
                lst = lst[(lst >= 0) & (lst < n)]
                for h in range(g * G, (g + 1) * G):
                    if lst.size == 0:
                        O_part[b, h] = 0.0
                        ml_part[b, h, 0] = -np.inf
                        ml_part[b, h, 1] = 0.0
                        continue
                    x = self.w.scale * (k[lst, g] @ q[h])
                    m = x.max()
                    e = np.exp(x - m)
                    O_part[b, h] = torch.from_numpy(e @ v[lst, g] / e.sum())
                    ml_part[b, h, 0] = m
                    ml_part[b, h, 1] = 1.0 / e.sum()


def _rank(rank, world, port, q):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        from long_context_full_b200 import context_parallel as cp
        w = synth.make_workload("cp", 77, "f32", HQ, HKV, D, LENS, [1] * B, LAYERS, topk=K,
                                window=WINDOW)
        lens = _split(world)
        stub = _Stub(w, rank, lens)
        # the library's calls, replaced for this CPU process
        cp.hs2.make_problem = lambda *a, **k: None
        cp.hs2.hs2_full_attn_workspace_size = lambda p: 1
        cp.hs2.hs2_cp_attn_partial = stub.attn_partial
        cp.hs2.hs2_cp_merge = _Stub.merge
        cp.hs2.hs2_cp_scores = stub.scores
        cp.hs2.hs2_cp_topk_local = stub.topk_local
        cp.hs2.hs2_cp_topk_merge = _Stub.topk_merge
        cp.hs2.hs2_cp_sparse_partial = stub.sparse_partial
        step = cp.ContextParallelDecodeStep(rank, world, HQ, HKV, D, torch.float32, lens, LAYERS,
                                            k=K, window=WINDOW, scale=w.scale, device="cpu")
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
        ko = w.kv_offsets
        pos0 = stub.pos0
        K_loc = torch.cat([t(w.k[ko[b] + pos0[b]:ko[b] + pos0[b] + lens[rank][b]]) for b in range(B)])
        V_loc = torch.cat([t(w.v[ko[b] + pos0[b]:ko[b] + pos0[b] + lens[rank][b]]) for b in range(B)])
        O, scores, idx, count, OL = step.run(t(w.q), K_loc, V_loc, [t(x) for x in w.q_layers],
                                             cp.nccl_all_gather())
        q.put((rank, O.numpy().copy(), idx.numpy().copy(), count.numpy().copy(),
               [x.numpy().copy() for x in OL]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_step_across_processes(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    qq = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, qq)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, *got = qq.get(timeout=300)
        res[r] = got
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    # the unsplit oracle
    w = synth.make_workload("cp", 77, "f32", HQ, HKV, D, LENS, [1] * B, LAYERS, topk=K, window=WINDOW)
    ko = w.kv_offsets
    for b in range(B):
        k = synth.stored_to_f64(w.k[ko[b]:ko[b + 1]], "f32")
        v = synth.stored_to_f64(w.v[ko[b]:ko[b + 1]], "f32")
        tpos = LENS[b] - 1
        Oref, _, _, P = oracle.full_attention_row(synth.stored_to_f64(w.q[b], "f32"), k, v, tpos,
                                                  w.scale)
        s = oracle.selection_scores(P, HKV)
        sets = []
        for g in range(HKV):
            oi, oc = oracle.topk_select(s[g], tpos, K, WINDOW)
            sets.append(oi[:oc])
            for r in range(world):
                O, idx, cnt, OL = res[r]
                assert int(cnt[b * HKV + g]) == oc
                assert np.array_equal(idx[b * HKV + g], oi), (r, b, g)
        for r in range(world):
            O, idx, cnt, OL = res[r]
            assert np.abs(O[b] - Oref).max() <= 1e-5 * np.abs(Oref).max()
            for l in range(LAYERS):
                ref = oracle.sparse_attention_row(synth.stored_to_f64(w.q_layers[l][b], "f32"), k, v,
                                                  sets, w.scale)
                assert np.abs(OL[l][b] - ref).max() <= 1e-5 * np.abs(ref).max()
    # every rank holds the same merged result
    for r in range(1, world):
        for a_, b_ in zip(res[0][:3], res[r][:3]):
            assert np.array_equal(a_, b_)
