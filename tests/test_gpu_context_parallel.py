"""Context-parallel decode (the cache of every sequence split by position
across ranks), with the ranks driven in turn on one GPU: the merged
full-attention output, each rank's scores, the merged index set and the sparse
layers against the oracle on the unsplit sequences; every rank ends with the
same output and index set."""
import numpy as np
import pytest
import torch

import oracle
import synth
from long_context_full_b200 import hs2
from long_context_full_b200.context_parallel import (ContextParallelDecodeStep, LocalRanks,
                                                     shard_offsets)
from tests.gpu_util import (OracleRows, check_index_sets, check_O, check_scores, to_device, to_f64,
                            torch_dtype)

pytestmark = pytest.mark.gpu

SPLITS = {
    "2_ranks_even": [[3000, 1250], [3000, 1250]],
    # the last range of sequence 1 (60 keys) is shorter than the window: the
    # window spans two ranks
    "3_ranks_uneven": [[2000, 1200], [1500, 1240], [2500, 60]],
}


def _rank_rows(w, lens):
    pos0 = shard_offsets(lens)
    out = []
    for r in range(len(lens)):
        rows = [np.arange(w.kv_offsets[b] + pos0[r][b], w.kv_offsets[b] + pos0[r][b] + lens[r][b])
                for b in range(w.B)]
        out.append(np.concatenate(rows))
    return out


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("split", list(SPLITS))
def test_context_parallel_decode_matches_oracle(dtype, split):
    lens = SPLITS[split]
    world = len(lens)
    kv = list(np.sum(lens, axis=0))
    w = synth.make_workload("cp", 61, dtype, 16, 2, 128, kv, [1, 1], 2)
    tdt = torch_dtype(dtype)
    steps = [ContextParallelDecodeStep(r, world, w.Hq, w.Hkv, w.D, tdt, lens, w.n_layers,
                                       k=w.topk, window=w.window, scale=w.scale)
             for r in range(world)]
    rows = _rank_rows(w, lens)
    Ks = [to_device(w.k[rr], dtype) for rr in rows]
    Vs = [to_device(w.v[rr], dtype) for rr in rows]
    Q = to_device(w.q, dtype)
    QL = [to_device(x, dtype) for x in w.q_layers]
    LocalRanks(steps).run(Q, Ks, Vs, QL)
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK

    s0 = steps[0]
    for st in steps[1:]:  # the merges give every rank the same results
        assert torch.equal(st.O, s0.O) and torch.equal(st.idx, s0.idx)
        assert torch.equal(st.count, s0.count)
        for l in range(w.n_layers):
            assert torch.equal(st.O_layers[l], s0.O_layers[l])

    ora = OracleRows(w)
    O = to_f64(s0.O)
    OL = [to_f64(x) for x in s0.O_layers]
    idx, cnt = s0.idx.cpu().numpy(), s0.count.cpu().numpy()
    S = [st.scores.cpu().numpy() for st in steps]
    for q in range(w.B):
        Oref, sref, t = ora.full(q)
        check_O(O[q], Oref, dtype, f"{split} O row {q}")
        for g in range(w.Hkv):
            R = q * w.Hkv + g
            s_full = np.concatenate([S[r][R, :lens[r][q]] for r in range(world)])
            assert s_full.size == t + 1
            check_scores(s_full, sref[g], f"{split} scores row {q} g {g}")
            oi, oc = oracle.topk_select(sref[g], t, w.topk, w.window)
            check_index_sets(idx[R], int(cnt[R]), oi, oc, sref[g], t, w.topk, w.window,
                             f"{split} indices row {q} g {g}")
        sets = [idx[q * w.Hkv + g, :cnt[q * w.Hkv + g]] for g in range(w.Hkv)]
        for l in range(w.n_layers):
            check_O(OL[l][q], ora.sparse(q, l, sets), dtype, f"{split} layer {l} row {q}")


def test_context_parallel_selection_equals_unsplit_selection():
    """On the same scores the merged selection is the unsplit selection, bit
    for bit: the scores of the unsplit run are cut into ranges, each range
    goes through the local selection, and the merge must equal
    hs2_topk_select on the whole rows."""
    rng = np.random.default_rng(8)
    lens = [[4000, 900], [3500, 2000], [500, 100]]
    world = len(lens)
    kv = np.sum(lens, axis=0)
    B, Hkv = 2, 1
    # scores with many exact ties (quantised) so the position rule decides
    full = [np.round(rng.random(n) * 64).astype(np.float32) / 64 for n in kv]
    steps = [ContextParallelDecodeStep(r, world, 8, Hkv, 128, torch.bfloat16, lens, 1)
             for r in range(world)]
    pos0 = shard_offsets(lens)
    for r, st in enumerate(steps):
        S = np.zeros((B * Hkv, st.stride), np.float32)
        for b in range(B):
            S[b, :lens[r][b]] = full[b][pos0[r][b]:pos0[r][b] + lens[r][b]]
        st.scores.copy_(torch.from_numpy(S))
        hs2.hs2_cp_topk_local(st.problem, st.scores, st.stride, st.k, st.window, st.pos0,
                              st.idx_tmp, st.count_tmp, st.pair_score, st.pair_pos)
    ps = torch.stack([st.pair_score for st in steps])
    pp = torch.stack([st.pair_pos for st in steps])
    st = steps[0]
    st.selection_merge(ps, pp)
    # the unsplit selection
    stride = int(kv.max() + 3) // 4 * 4
    S = np.zeros((B, stride), np.float32)
    for b in range(B):
        S[b, :kv[b]] = full[b]
    Sd = torch.from_numpy(S).cuda()
    idx = torch.empty(B, st.kk, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, dtype=torch.int32, device="cuda")
    hs2.hs2_topk_select(st.problem_global, Sd, stride, st.k, st.window, idx, cnt, None)
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
    assert torch.equal(cnt, st.count) and torch.equal(idx, st.idx)
    for b in range(B):
        oi, oc = oracle.topk_select(full[b], int(kv[b]) - 1, 1024, 128)
        assert int(cnt[b]) == oc and list(idx[b, :oc].cpu().numpy()) == list(oi[:oc])
