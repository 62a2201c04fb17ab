"""Sparse layers on index lists the selection does not produce: lists longer
than one staged piece of a CTA's share (so the gather runs several rounds on
the same barriers), unsorted lists, and invalid entries in the middle of a
list.  Compared with the oracle row by row."""
import numpy as np
import pytest
import torch

import synth
from long_context_full_b200 import hs2
from tests.gpu_util import OracleRows, check_O, to_device, to_f64

pytestmark = pytest.mark.gpu


def _run(w, idx, count):
    qo = torch.from_numpy(w.q_offsets).cuda()
    ko = torch.from_numpy(w.kv_offsets).cuda()
    p = hs2.make_problem(w.B, w.Hq, w.Hkv, w.D, hs2.HS2_BF16 if w.dtype == "bf16" else hs2.HS2_F32,
                         qo, ko, int(w.q_lens.sum()), int(w.kv_lens.sum()), int(w.q_lens.max()),
                         int(w.kv_lens.max()), w.scale)
    stride = idx.shape[1]
    ws = torch.empty(max(1, hs2.hs2_sparse_attn_workspace_size(p, stride)), dtype=torch.uint8).cuda()
    O = torch.empty(int(w.q_lens.sum()), w.Hq, w.D, dtype=torch.bfloat16 if w.dtype == "bf16" else torch.float32).cuda()
    hs2.hs2_sparse_attn(p, to_device(w.q_layers[0], w.dtype), to_device(w.k, w.dtype),
                        to_device(w.v, w.dtype), torch.from_numpy(idx).cuda(),
                        torch.from_numpy(count).cuda(), stride, O, ws)
    return O


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("n_sel", [3000, 1281, 17])
def test_long_and_unsorted_lists(dtype, n_sel):
    w = synth.make_workload("splist", 51, dtype, 16, 2, 128, [6000, 3500], [1, 1], 1)
    rng = np.random.default_rng(n_sel)
    tpos = w.query_positions()
    rows = len(tpos) * w.Hkv
    stride = 3072
    idx = np.full((rows, stride), -1, np.int32)
    count = np.zeros(rows, np.int32)
    sets = {}
    for r in range(rows):
        t = int(tpos[r // w.Hkv])
        n = min(n_sel, t + 1)
        sel = rng.choice(t + 1, size=n, replace=False).astype(np.int32)  # unsorted
        idx[r, :n] = sel
        count[r] = n
        sets[r] = sel
    O = _run(w, idx, count)
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
    ora = OracleRows(w)
    got = to_f64(O)
    for q in range(len(tpos)):
        ref = ora.sparse(q, 0, [sets[q * w.Hkv + g] for g in range(w.Hkv)])
        check_O(got[q], ref, dtype, f"sparse list {n_sel} row {q}")


def test_invalid_entries_are_skipped_and_reported():
    """Entries outside 0..t in the middle of a long list: reported, and the
    row equals attention over its valid entries."""
    w = synth.make_workload("spbad", 52, "bf16", 16, 2, 128, [5000], [1], 1)
    t = int(w.query_positions()[0])
    rng = np.random.default_rng(3)
    stride = 2048
    idx = np.full((w.Hkv, stride), -1, np.int32)
    count = np.full(w.Hkv, 2000, np.int32)
    sets = []
    for g in range(w.Hkv):
        sel = rng.choice(t + 1, size=2000, replace=False).astype(np.int32)
        bad = rng.choice(2000, size=37, replace=False)
        sel[bad[:20]] = t + 1 + rng.integers(0, 1000, size=20)   # past the query position
        sel[bad[20:]] = -rng.integers(1, 1000, size=17)            # negative
        idx[g, :2000] = sel
        sets.append(np.sort(sel[(sel >= 0) & (sel <= t)]))
    O = _run(w, idx, count)
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_ERR_DEVICE_INPUT
    ref = OracleRows(w).sparse(0, 0, sets)
    check_O(to_f64(O)[0], ref, "bf16", "sparse list with invalid entries")
