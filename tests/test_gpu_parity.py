"""CUDA path vs the CPU oracle on the same seeded inputs (small and mid sizes:
several tiles, ragged tails, edge lengths, ties, grouped-query variants)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from long_context_full_b200 import hs2
from tests.gpu_util import (CudaPathRun, OracleRows, check_O, check_block_sets, check_index_sets,
                            check_scores, gpu_select_on, to_f64)

pytestmark = pytest.mark.gpu


def full_check(w, select="token", rows=None, layers=True):
    """Runs the CUDA path and checks O, scores, selection and sparse layers for
    the listed query rows (all by default).  Returns a summary dict."""
    run = CudaPathRun(w, select)
    out = run.run()
    ora = OracleRows(w)
    O = out.O
    S = out.scores.cpu().numpy()
    idx = out.idx.cpu().numpy()
    cnt = out.count.cpu().numpy()
    OL = [to_f64(x) for x in out.O_layers] if layers else None
    Og = to_f64(O)
    rows = range(w.q.shape[0]) if rows is None else rows
    summ = dict(o_err=0.0, score_rel=0.0, flips=0, sparse_err=0.0)
    for r in rows:
        Oref, sref, t = ora.full(r)
        summ["o_err"] = max(summ["o_err"], check_O(Og[r], Oref, w.dtype, f"O row {r}"))
        for g in range(w.Hkv):
            R = r * w.Hkv + g
            summ["score_rel"] = max(summ["score_rel"],
                                    check_scores(S[R, :t + 1], sref[g], f"scores row {r} g {g}"))
            # selection on the oracle's own scores is bit-exact
            if select == "token":
                oi, oc = oracle.topk_select(sref[g], t, w.topk, w.window)
            else:
                oi, oc = oracle.block_select(sref[g], t, w.n_blocks, w.block, w.window)
            if select == "token":
                summ["flips"] += check_index_sets(idx[R], int(cnt[R]), oi, oc, sref[g], t, w.topk,
                                                  w.window, f"indices row {r} g {g}")
            else:
                summ["flips"] += check_block_sets(idx[R], int(cnt[R]), oi, oc, sref[g], t,
                                                  w.n_blocks, w.block, w.window,
                                                  f"blocks row {r} g {g}")
        if layers:
            sets = [idx[r * w.Hkv + g, :cnt[r * w.Hkv + g]] for g in range(w.Hkv)]
            for l in range(w.n_layers):
                ref = ora.sparse(r, l, sets)
                summ["sparse_err"] = max(summ["sparse_err"],
                                         check_O(OL[l][r], ref, w.dtype, f"layer {l} row {r}"))
    return summ, out


def test_tiny_f32_workload():
    """Batch 1, one decode query over 4096 keys, Hq=4 / Hkv=1, fp32, 3 reuse layers."""
    w = synth.tiny()
    summ, out = full_check(w)
    assert summ["flips"] == 0
    assert int(out.count[0]) == 1152


def test_sparse_equals_full_when_budget_covers_context():
    """t + 1 <= 1024 + 128: the index set is the whole context, so a sparse layer
    given the full-attention layer's query reproduces the full output."""
    for dtype in ("f32", "bf16"):
        w = synth.make_workload("short", 11, dtype, 8, 2, 128, [1152, 700, 1], [1, 1, 1], 1)
        w.q_layers[0][:] = w.q  # same queries as the full-attention layer
        run = CudaPathRun(w)
        out = run.run()
        cnt = out.count.cpu().numpy()
        assert list(cnt) == [1152, 1152, 700, 700, 1, 1]
        a, b = to_f64(out.O), to_f64(out.O_layers[0])
        tol = 2e-2 if dtype == "bf16" else 1e-5
        assert np.abs(a - b).max() <= tol * (1 if dtype == "bf16" else np.abs(a).max())


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_ragged_decode_edge_lengths(dtype):
    lens = [1, 2, 127, 128, 129, 1151, 1152, 1153, 1280, 4096, 9000]
    w = synth.make_workload("edges", 21, dtype, 16, 2, 128, lens, [1] * len(lens), 2)
    summ, out = full_check(w)
    cnt = out.count.cpu().numpy().reshape(-1, 2)[:, 0]
    assert list(cnt) == [min(n, 1152) for n in lens]


@pytest.mark.parametrize("dtype,Hq,Hkv", [("bf16", 4, 4), ("bf16", 8, 4), ("bf16", 8, 2),
                                          ("bf16", 32, 4), ("f32", 4, 1), ("f32", 16, 2),
                                          ("f32", 16, 1), ("f32", 6, 2)])
def test_gqa_variants(dtype, Hq, Hkv):
    w = synth.make_workload("gqa", 31, dtype, Hq, Hkv, 128, [3000, 1500], [1, 1], 1)
    full_check(w)


def test_decode_many_tiles_bf16():
    """Two sequences long enough for every CTA of the split to see several
    tiles and a ragged tail, batch boundary inside a CTA range."""
    w = synth.make_workload("mid", 41, "bf16", 32, 4, 128, [70001, 33333], [1, 1], 2)
    summ, _ = full_check(w)
    assert summ["score_rel"] < 2e-5


def _select_rows():
    rng = np.random.default_rng(5)
    n = 20000
    rows = [
        np.ones(n, np.float32),                                      # all equal
        np.arange(n, dtype=np.float32),                              # strictly increasing
        rng.integers(0, 3, n).astype(np.float32),                    # heavy ties at threshold
        rng.random(n).astype(np.float32),                            # distinct
        np.where(rng.random(n) < 0.5, np.float32(0.0), np.float32(-0.0)),  # +0 / -0
        (rng.random(n) * 2 - 1).astype(np.float32),                 # negatives
    ]
    x = rng.random(n).astype(np.float32)
    x[rng.choice(n, 3000, replace=False)] = np.float32(0.75)         # a big block of equal values
    rows.append(x)
    return np.stack(rows)


def test_select_bit_exact_on_fixed_scores():
    S = _select_rows()
    ts = [19999, 19999, 15000, 19999, 19999, 12345, 19999]
    idx, cnt = gpu_select_on(S, ts)
    for r, t in enumerate(ts):
        oi, oc = oracle.topk_select(S[r], t)
        assert int(cnt[r]) == oc
        assert np.array_equal(idx[r], oi), f"row {r}"


@pytest.mark.parametrize("t", [0, 1, 126, 127, 128, 129, 1151, 1152, 1153, 4223, 4224, 4225, 8319, 70000])
def test_select_edge_positions(t):
    rng = np.random.default_rng(t)
    s = rng.integers(0, 50, t + 1).astype(np.float32)
    idx, cnt = gpu_select_on(s[None, :], [t])
    oi, oc = oracle.topk_select(s, t)
    assert int(cnt[0]) == oc and np.array_equal(idx[0], oi)


def test_select_many_rows():
    """Many rows (clusters run in several waves); a row's result does not
    depend on the rows launched with it."""
    rng = np.random.default_rng(17)
    R, n = 1400, 3000
    S = rng.integers(0, 40, (R, n)).astype(np.float32)
    ts = list(rng.integers(1100, n, R))
    idx, cnt = gpu_select_on(S, ts)
    for r in range(0, R, 7):
        oi, oc = oracle.topk_select(S[r], ts[r])
        assert int(cnt[r]) == oc and np.array_equal(idx[r], oi), r
    # the same rows in a small batch give the same result
    sub = list(range(0, 60))
    i2, c2 = gpu_select_on(S[sub], [ts[r] for r in sub])
    assert np.array_equal(i2, idx[sub]) and np.array_equal(c2, cnt[sub])


def test_select_long_rows_wide_slices():
    """Long rows with a large tie block straddling the threshold."""
    rng = np.random.default_rng(23)
    R, n = 40, 100000
    S = rng.random((R, n)).astype(np.float32)
    S[:, ::7] = np.float32(0.999)  # a tie block straddling the threshold
    ts = [n - 1 - 37 * r for r in range(R)]
    idx, cnt = gpu_select_on(S, ts)
    for r in range(R):
        oi, oc = oracle.topk_select(S[r], ts[r])
        assert int(cnt[r]) == oc and np.array_equal(idx[r], oi), r


def test_select_rows_longer_than_shared_memory():
    """Rows whose per-CTA slices do not fit in shared memory (re-read from
    global memory on every pass)."""
    rng = np.random.default_rng(29)
    n = 600000
    S = rng.standard_normal((2, n)).astype(np.float32)
    S[1, rng.choice(n, 5000, replace=False)] = np.float32(2.5)
    ts = [n - 1, n - 1000]
    idx, cnt = gpu_select_on(S, ts)
    for r in range(2):
        oi, oc = oracle.topk_select(S[r], ts[r])
        assert int(cnt[r]) == oc and np.array_equal(idx[r], oi), r


def test_select_many_long_rows():
    """Enough rows to fill the GPU with one CTA per row, rows longer than a
    CTA's candidate buffer: the sampled threshold, then the exact select."""
    rng = np.random.default_rng(31)
    R, n = 320, 30000
    S = rng.standard_normal((R, n)).astype(np.float32)
    S[: R // 2, -5000:] += np.float32(2.0)  # top keys crowded at the end for half the rows
    ts = [n - 1 - 11 * r for r in range(R)]
    idx, cnt = gpu_select_on(S, ts)
    for r in range(0, R, 5):
        oi, oc = oracle.topk_select(S[r], ts[r])
        assert int(cnt[r]) == oc and np.array_equal(idx[r], oi), r


@pytest.mark.parametrize("R,n", [(300, 20000), (2, 50000), (2, 600000)])
def test_select_all_equal_falls_back_to_exact(R, n):
    """Every key ties: more keys reach the sampled threshold than a CTA holds,
    so the exact selection over global memory runs (one CTA per row, and a
    16-CTA cluster per row)."""
    S = np.full((R, n), np.float32(0.5))
    ts = [n - 1 - 3 * r for r in range(R)]
    idx, cnt = gpu_select_on(S, ts)
    for r in range(0, R, max(1, R // 20)):
        oi, oc = oracle.topk_select(S[r], ts[r])
        assert int(cnt[r]) == oc and np.array_equal(idx[r], oi), r


def test_select_cluster_finish_cases():
    """Decode-sized rows on 8-CTA clusters, through the finish that ranks the
    threshold prefix's keys on every CTA and through its fallback: the top
    keys all in one CTA's slice; ties at the threshold under and over the
    number of prefix keys a CTA takes (256); distinct keys that share the
    threshold's 22-bit prefix; ties and near-ties spread over the slices."""
    rng = np.random.default_rng(43)
    n = 131072
    rows = []
    x = rng.random(n).astype(np.float32)
    x[100:100 + 1500] += np.float32(1.0)                      # the top keys in slice 0
    rows.append(x)
    for nt in (200, 300):                                      # 1000 clear winners + nt ties
        x = rng.random(n).astype(np.float32)
        pos = rng.choice(n - 200, 1000 + nt, replace=False)
        x[pos[:1000]] = np.float32(2.0)
        x[pos[1000:]] = np.float32(1.5)
        rows.append(x)
    x = rng.random(n).astype(np.float32)                       # 100 keys sharing a 22-bit prefix
    pos = rng.choice(n - 200, 1100, replace=False)
    x[pos[:1000]] = np.float32(2.0)
    bits = np.float32(1.5).view(np.uint32) + rng.permutation(100).astype(np.uint32)
    x[pos[1000:]] = bits.view(np.float32)
    rows.append(x)
    x = rng.integers(0, 2000, n).astype(np.float32)            # ties spread over every slice
    rows.append(x)
    S = np.stack(rows)
    ts = [n - 1] * len(rows)
    idx, cnt = gpu_select_on(S, ts)
    for r in range(len(rows)):
        oi, oc = oracle.topk_select(S[r], ts[r])
        assert int(cnt[r]) == oc and np.array_equal(idx[r], oi), r


def test_select_large_k_exact_kernel():
    """k above the sampled kernel's limit runs the exact cluster kernel."""
    rng = np.random.default_rng(37)
    n = 50000
    S = rng.integers(0, 500, (3, n)).astype(np.float32)
    ts = [n - 1, 30000, 2500]
    idx, cnt = gpu_select_on(S, ts, k=3000)
    for r in range(3):
        oi, oc = oracle.topk_select(S[r], ts[r], 3000, 128)
        assert int(cnt[r]) == oc and np.array_equal(idx[r], oi), r


@pytest.mark.parametrize("stride_extra", [1, 2, 3, 37])
def test_select_unaligned_stride(stride_extra):
    """Score rows whose stride is not a multiple of 4 floats (the C ABI allows
    any stride >= the longest sequence)."""
    rng = np.random.default_rng(stride_extra)
    n = 9000
    S = rng.integers(0, 30, (3, n)).astype(np.float32)
    ts = [n - 1, n - 500, 4000]
    idx, cnt = gpu_select_on(S, ts, stride=n + stride_extra)
    for r in range(3):
        oi, oc = oracle.topk_select(S[r], ts[r])
        assert int(cnt[r]) == oc and np.array_equal(idx[r], oi), r


def test_block_select_bit_exact():
    S = _select_rows()
    ts = [19999, 19999, 15000, 19999, 19999, 12345, 19999]
    idx, cnt = gpu_select_on(S, ts, block_mode=True)
    for r, t in enumerate(ts):
        oi, oc = oracle.block_select(S[r], t)
        assert int(cnt[r]) == oc
        assert np.array_equal(idx[r], oi), f"row {r}"
    for t in (0, 5, 127, 128, 191, 192, 1151, 1152, 1153, 1200, 5000):
        s = np.random.default_rng(t).random(t + 1).astype(np.float32)
        i, c = gpu_select_on(s[None, :], [t], block_mode=True)
        oi, oc = oracle.block_select(s, t)
        assert int(c[0]) == oc and np.array_equal(i[0], oi), t


def test_block_select_path_end_to_end():
    w = synth.make_workload("blk", 51, "bf16", 16, 2, 128, [5000, 2000, 300], [1, 1, 1], 1)
    full_check(w, select="block")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_chunk_causal(dtype):
    """Several new query tokens per sequence on top of a cached context."""
    w = synth.make_workload("chunk", 61, dtype, 16, 2, 128, [3000, 1500, 300], [200, 37, 300], 1)
    full_check(w)


def test_chunk_key_split_bf16():
    """A chunk whose query tiles alone would leave most SMs idle: the visible
    keys of each tile are split over several CTAs (statistics per range, then
    scores and O shares per range, then the O sum), with a second, short
    sequence whose ranges are a few key tiles each."""
    w = synth.make_workload("chunks", 63, "bf16", 32, 4, 128, [20000, 3000], [64, 40], 1)
    p = hs2.make_problem(w.B, w.Hq, w.Hkv, w.D, hs2.HS2_BF16, torch.from_numpy(w.q_offsets).cuda(),
                         torch.from_numpy(w.kv_offsets).cuda(), int(w.q_lens.sum()),
                         int(w.kv_lens.sum()), int(w.q_lens.max()), int(w.kv_lens.max()), w.scale)
    assert hs2.hs2_full_attn_launches(p) == 3  # the split form runs on this shape
    full_check(w)


def test_chunk_gqa_bf16():
    for Hq, Hkv in ((4, 4), (8, 4), (8, 2), (32, 4)):
        w = synth.make_workload("chunkg", 62, "bf16", Hq, Hkv, 128, [2500], [150], 1)
        full_check(w)


def test_repeatable():
    w = synth.make_workload("rep", 71, "bf16", 32, 4, 128, [50000, 20000], [1, 1], 1)
    run = CudaPathRun(w)
    a = run.run()
    i1, s1, o1 = a.idx.clone(), a.scores.clone(), a.O_layers[0].clone()
    b = run.run()
    assert torch.equal(i1, b.idx) and torch.equal(s1, b.scores) and torch.equal(o1, b.O_layers[0])


def test_device_input_errors_are_reported():
    w = synth.make_workload("err", 81, "bf16", 8, 1, 128, [500], [1], 1)
    run = CudaPathRun(w)
    run.run()
    bad = run.step.idx.clone()
    bad[0, 3] = 600  # beyond the query position
    hs2.hs2_sparse_attn(run.step.problem, run.QL[0], run.K, run.V, bad, run.step.count,
                        run.step.idx_stride, run.step.O_layers[0], run.step.workspace)
    assert hs2.hs2_get_last_device_error() == hs2.HS2_ERR_DEVICE_INPUT
    assert torch.isfinite(run.step.O_layers[0].float()).all()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK  # cleared


def test_host_checks_launch_nothing():
    w = synth.make_workload("chk", 91, "bf16", 8, 1, 128, [500], [1], 1)
    run = CudaPathRun(w, select="block")
    before = run.step.idx.clone()
    with pytest.raises(hs2.HS2Error) as e:
        hs2.hs2_block_select(run.step.problem, run.step.scores, run.step.stride, 16, 64, 128,
                             run.step.idx, run.step.count, None)
    assert e.value.status == hs2.HS2_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.equal(before, run.step.idx)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("q_lens", [[1, 0, 1, 0, 1, 0], [0, 5, 0, 1, 40, 0]],
                         ids=["decode", "chunk"])
def test_sequences_without_queries(dtype, q_lens):
    """A batch mixing sequences with no query token (Tq_b = 0) with decode and
    chunk sequences: every kernel skips the empty ones by their offsets, and the
    others match the oracle through the whole path (scores, token and block
    selection, the no-allocation block selection, sparse layers)."""
    kv = [3000, 1800, 1300, 2500, 1500, 700]
    w = synth.make_workload("noq", 97, dtype, 16, 2, 128, kv, q_lens, 2)
    summ, out = full_check(w)
    assert summ["flips"] == 0
    summ, out = full_check(w, select="block")
    # the no-allocation block selection gives the same result on the same scores
    run = CudaPathRun(w, select="block")
    o = run.run()
    idx2 = torch.full_like(o.idx, 7777)
    cnt2 = torch.full_like(o.count, 7777)
    hs2.hs2_block_select_noalloc(run.step.problem, o.scores, run.step.stride, w.n_blocks, w.block,
                                 w.window, idx2, cnt2)
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
    assert torch.equal(idx2, o.idx) and torch.equal(cnt2, o.count)


def test_step_without_query_rows():
    """total_q = 0: every call returns HS2_OK and writes nothing - buffers
    handed in anyway keep their canary bytes."""
    B, Hq, Hkv, D = 3, 16, 2, 128
    kv_lens = [500, 300, 1200]
    qo = torch.zeros(B + 1, dtype=torch.int64, device="cuda")
    ko = torch.tensor(np.concatenate([[0], np.cumsum(kv_lens)]), dtype=torch.int64, device="cuda")
    tkv = int(sum(kv_lens))
    for dt, code in ((torch.bfloat16, hs2.HS2_BF16), (torch.float32, hs2.HS2_F32)):
        for max_q in (0, 1, 4):
            p = hs2.make_problem(B, Hq, Hkv, D, code, qo, ko, 0, tkv, max_q, max(kv_lens), 0.088)
            K = torch.randn(tkv, Hkv, D, device="cuda").to(dt)
            V = torch.randn(tkv, Hkv, D, device="cuda").to(dt)
            Kc, Vc = K.clone(), V.clone()
            Q = torch.randn(4, Hq, D, device="cuda").to(dt)
            O = torch.full((4, Hq, D), 7.0, device="cuda").to(dt)
            S = torch.full((8, 1216), 5.0, device="cuda")
            idx = torch.full((8, 1152), 7777, dtype=torch.int32, device="cuda")
            cnt = torch.full((8,), 7777, dtype=torch.int32, device="cuda")
            ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
            canaries = [t.clone() for t in (O, S, idx, cnt)]
            hs2.hs2_full_attn_scores(p, Q, K, V, O, S, 1216, ws)
            hs2.hs2_topk_select(p, S, 1216, 1024, 128, idx, cnt, ws)
            hs2.hs2_block_select(p, S, 1216, 16, 64, 128, idx, cnt, ws)
            hs2.hs2_block_select_noalloc(p, S, 1216, 16, 64, 128, idx, cnt)
            hs2.hs2_sparse_attn(p, Q, K, V, idx, cnt, 1152, O, ws)
            hs2.hs2_swa_attn(p, Q, K, V, 128, O)
            hs2.hs2_kv_append(p, Q[:, :Hkv], Q[:, :Hkv], K, V)
            torch.cuda.synchronize()
            assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
            for a, b in zip((O, S, idx, cnt), canaries):
                assert torch.equal(a, b)
            assert torch.equal(K, Kc) and torch.equal(V, Vc)
