"""Sliding-window attention (the Hybrid SWA baseline's local layer) through the
C ABI, against the oracle, and bit for bit against the sparse layer given the
same window positions as an index list."""
import numpy as np
import pytest
import torch

import oracle
import synth
from long_context_full_b200 import hs2
from tests.gpu_util import check_O, to_device, to_f64

pytestmark = pytest.mark.gpu


def _problem(w):
    qo = torch.from_numpy(w.q_offsets).cuda()
    ko = torch.from_numpy(w.kv_offsets).cuda()
    p = hs2.make_problem(w.B, w.Hq, w.Hkv, w.D, hs2.HS2_BF16 if w.dtype == "bf16" else hs2.HS2_F32,
                         qo, ko, int(w.q_lens.sum()), int(w.kv_lens.sum()), int(w.q_lens.max()),
                         int(w.kv_lens.max()), w.scale)
    return p, (qo, ko)


@pytest.mark.parametrize("dtype,window", [("bf16", 128), ("bf16", 1000), ("f32", 128), ("bf16", 1)])
def test_swa_matches_oracle(dtype, window):
    """Decode rows of ragged lengths (some shorter than the window) and a chunk
    of causal queries."""
    w = synth.make_workload("swa", 401, dtype, 16, 2, 128, [3000, 1, 90, 700, 5000], [1, 1, 1, 1, 40], 0)
    p, keep = _problem(w)
    Q, K, V = to_device(w.q, dtype), to_device(w.k, dtype), to_device(w.v, dtype)
    O = torch.empty_like(Q)
    hs2.hs2_swa_attn(p, Q, K, V, window, O)
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
    Og = to_f64(O)
    seq, tpos = w.query_seq(), w.query_positions()
    ko = w.kv_offsets
    for r in list(range(4)) + [4, 20, 43]:
        b, t = int(seq[r]), int(tpos[r])
        k = synth.stored_to_f64(w.k[ko[b]:ko[b + 1]], dtype)
        v = synth.stored_to_f64(w.v[ko[b]:ko[b + 1]], dtype)
        q = synth.stored_to_f64(w.q[r], dtype)
        check_O(Og[r], oracle.swa_attention_row(q, k, v, t, window, w.scale), dtype, f"row {r}")


def test_swa_equals_sparse_layer_on_window_indices():
    w = synth.make_workload("swa2", 402, "bf16", 32, 4, 128, [20000, 333], [1, 1], 0)
    p, keep = _problem(w)
    Q, K, V = to_device(w.q, "bf16"), to_device(w.k, "bf16"), to_device(w.v, "bf16")
    W = 128
    O1, O2 = torch.empty_like(Q), torch.empty_like(Q)
    hs2.hs2_swa_attn(p, Q, K, V, W, O1)
    tpos = np.repeat(w.query_positions(), w.Hkv)
    idx = np.full((len(tpos), W), -1, dtype=np.int32)
    cnt = np.zeros(len(tpos), dtype=np.int32)
    for r, t in enumerate(tpos):
        pos = oracle.window_range(int(t), W)
        idx[r, :len(pos)] = pos
        cnt[r] = len(pos)
    hs2.hs2_sparse_attn(p, Q, K, V, torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda(), W, O2, None)
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
    assert torch.equal(O1, O2)


def test_swa_host_checks():
    w = synth.make_workload("swa3", 403, "bf16", 8, 1, 128, [100], [1], 0)
    p, keep = _problem(w)
    Q, K, V = to_device(w.q, "bf16"), to_device(w.k, "bf16"), to_device(w.v, "bf16")
    O = torch.zeros_like(Q)
    with pytest.raises(hs2.HS2Error) as e:
        hs2.hs2_swa_attn(p, Q, K, V, 0, O)
    assert e.value.status == hs2.HS2_ERR_INVALID_ARG
    assert int(O.abs().sum()) == 0
