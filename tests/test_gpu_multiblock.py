"""KV append and the multi-block decode step (several Hybrid Blocks in one
CUDA graph) through the C ABI, against the oracle."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import synth
from long_context_full_b200 import hs2
from long_context_full_b200.multiblock import BlockInputs, MultiBlockDecodeStep
from tests.gpu_util import OracleRows, check_O, check_index_sets, check_scores, to_device, to_f64

pytestmark = pytest.mark.gpu


def _new_rows(rng, n, Hkv, D, dtype):
    x = rng.standard_normal((n, Hkv, D)).astype(np.float32)
    return synth.f32_to_bf16_bits(x) if dtype == "bf16" else x


def _bits(t: torch.Tensor, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)
    return t.detach().cpu().numpy()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_kv_append_matches_oracle(dtype):
    """Decode sequences (one new token) and a chunk (several), ragged caches;
    every written row and every untouched row compared bit for bit."""
    rng = np.random.default_rng(11)
    w = synth.make_workload("app", 301, dtype, 8, 2, 128, [700, 1, 3000, 129], [1, 1, 37, 5], 0)
    Kn = _new_rows(rng, int(w.q_lens.sum()), w.Hkv, w.D, dtype)
    Vn = _new_rows(rng, int(w.q_lens.sum()), w.Hkv, w.D, dtype)
    qo = torch.from_numpy(w.q_offsets).cuda()
    ko = torch.from_numpy(w.kv_offsets).cuda()
    p = hs2.make_problem(w.B, w.Hq, w.Hkv, w.D, hs2.HS2_BF16 if dtype == "bf16" else hs2.HS2_F32,
                         qo, ko, int(w.q_lens.sum()), int(w.kv_lens.sum()), int(w.q_lens.max()),
                         int(w.kv_lens.max()), w.scale)
    K, V = to_device(w.k, dtype), to_device(w.v, dtype)
    hs2.hs2_kv_append(p, to_device(Kn, dtype), to_device(Vn, dtype), K, V)
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
    Kr, Vr = oracle.kv_append(w.k, w.v, Kn, Vn, w.q_offsets, w.kv_offsets)
    assert np.array_equal(_bits(K, dtype), Kr) and np.array_equal(_bits(V, dtype), Vr)


def test_kv_append_empty_step_launches_nothing():
    w = synth.make_workload("app0", 302, "bf16", 8, 2, 128, [50, 60], [0, 0], 0)
    qo = torch.from_numpy(w.q_offsets).cuda()
    ko = torch.from_numpy(w.kv_offsets).cuda()
    p = hs2.make_problem(w.B, 8, 2, 128, hs2.HS2_BF16, qo, ko, 0, 110, 0, 60, w.scale)
    K, V = to_device(w.k, "bf16"), to_device(w.v, "bf16")
    before = K.clone()
    hs2.hs2_kv_append(p, None, None, K, V)
    torch.cuda.synchronize()
    assert torch.equal(K, before)


def _block_case(seed, rng):
    w = synth.make_workload(f"mb{seed}", seed, "bf16", 16, 2, 128, [3000, 1500, 700], [1, 1, 1], 2)
    Kn = _new_rows(rng, w.B, w.Hkv, w.D, "bf16")
    Vn = _new_rows(rng, w.B, w.Hkv, w.D, "bf16")
    return w, Kn, Vn


def test_multiblock_graph_matches_eager_and_oracle():
    """Three blocks with their own caches: the graph replay gives exactly the
    eager results, and sampled rows of each block match the oracle run on the
    appended cache."""
    rng = np.random.default_rng(13)
    cases = [_block_case(310 + i, rng) for i in range(3)]
    w0 = cases[0][0]
    args = (w0.Hq, w0.Hkv, w0.D, torch.bfloat16, w0.q_lens, w0.kv_lens, w0.n_layers)

    def inputs():
        return [BlockInputs(to_device(w.k, "bf16"), to_device(w.v, "bf16"), to_device(Kn, "bf16"),
                            to_device(Vn, "bf16"), to_device(w.q, "bf16"),
                            [to_device(x, "bf16") for x in w.q_layers]) for w, Kn, Vn in cases]

    eager = MultiBlockDecodeStep(3, *args)
    outs_e = eager.run(inputs())
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
    snap = [(o.O.clone(), o.scores.clone(), o.idx.clone(), o.count.clone(),
             [x.clone() for x in o.O_layers]) for o in outs_e]

    graphed = MultiBlockDecodeStep(3, *args)
    ins = inputs()
    outs_g = graphed.capture(ins)
    for o in outs_g:  # clear what the warm-up run wrote
        o.O.zero_(); o.scores.zero_(); o.idx.zero_(); o.count.zero_()
        for x in o.O_layers:
            x.zero_()
    graphed.replay()
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
    # per block: append, full attention (pass + finish), select, 2 sparse layers
    assert graphed.launches_per_step() == 3 * (1 + 2 + 1 + 2)
    # score entries past a row's position are undefined: compare 0..t only
    tpos = torch.from_numpy(np.repeat(w0.query_positions(), w0.Hkv)).cuda()
    defined = torch.arange(snap[0][1].shape[1], device="cuda")[None, :] <= tpos[:, None]
    for (O, S, I, C, OL), o in zip(snap, outs_g):
        assert torch.equal(O, o.O) and torch.equal(S[defined], o.scores[defined])
        assert torch.equal(I, o.idx) and torch.equal(C, o.count)
        assert all(torch.equal(a, b) for a, b in zip(OL, o.O_layers))

    for (w, Kn, Vn), o in zip(cases, outs_g):
        k2, v2 = oracle.kv_append(w.k, w.v, Kn, Vn, w.q_offsets, w.kv_offsets)
        wa = dataclasses.replace(w, k=k2, v=v2)
        ora = OracleRows(wa)
        Og, OL = to_f64(o.O), [to_f64(x) for x in o.O_layers]
        for r in (0, w.B - 1):
            Oref, sref, t = ora.full(r)
            check_O(Og[r], Oref, "bf16", f"O row {r}")
            sets = []
            for g in range(w.Hkv):
                R = r * w.Hkv + g
                check_scores(o.scores[R, :t + 1].cpu().numpy(), sref[g], f"scores {r}/{g}")
                idx = o.idx[R].cpu().numpy()
                cnt = int(o.count[R])
                oi, oc = oracle.topk_select(sref[g], t, w.topk, w.window)
                check_index_sets(idx, cnt, oi, oc, sref[g], t, w.topk, w.window, f"idx {r}/{g}")
                sets.append(idx[:cnt])
            for l in range(w.n_layers):
                check_O(OL[l][r], ora.sparse(r, l, sets), "bf16", f"layer {l} row {r}")
