"""hs2_block_select_noalloc: block selection for callers that cannot give the
library device memory (an engine or plugin interface that owns all device
allocations and passes no workspace, or code that must not call cudaMalloc
because it can synchronise the device).  The call takes its scratch from a
fixed array inside the library.  Its results must equal those of
hs2_block_select with a caller workspace, call after call, although every
call reuses the same scratch.  This file is collected last on purpose."""
import numpy as np
import pytest
import torch

from long_context_full_b200 import hs2

pytestmark = pytest.mark.gpu


def _problem(ts, stride):
    R = len(ts)
    kv_lens = np.asarray(ts, np.int64) + 1
    qo = torch.arange(R + 1, dtype=torch.int64).cuda()
    ko = torch.from_numpy(np.concatenate([[0], np.cumsum(kv_lens)]).astype(np.int64)).cuda()
    p = hs2.make_problem(R, 1, 1, 128, hs2.HS2_BF16, qo, ko, R, int(kv_lens.sum()), 1,
                         int(kv_lens.max()), 0.1)
    return p, (qo, ko)


def _select_both(scores: np.ndarray, ts, n_blocks=16, block=64, window=128):
    stride = scores.shape[1]
    p, keep = _problem(ts, stride)
    s = torch.from_numpy(scores).cuda()
    width = n_blocks * block + window
    R = len(ts)
    idx_ws = torch.full((R, width), -7, dtype=torch.int32).cuda()
    cnt_ws = torch.full((R,), -7, dtype=torch.int32).cuda()
    ws = torch.empty(hs2.hs2_block_select_workspace_size(p, n_blocks, block, window),
                     dtype=torch.uint8).cuda()
    hs2.hs2_block_select(p, s, stride, n_blocks, block, window, idx_ws, cnt_ws, ws)
    idx_na = torch.full((R, width), -9, dtype=torch.int32).cuda()
    cnt_na = torch.full((R,), -9, dtype=torch.int32).cuda()
    hs2.hs2_block_select_noalloc(p, s, stride, n_blocks, block, window, idx_na, cnt_na)
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
    return (idx_ws.cpu().numpy(), cnt_ws.cpu().numpy()), (idx_na.cpu().numpy(), cnt_na.cpu().numpy())


def test_noalloc_matches_workspace_call_twice_in_a_row():
    rng = np.random.default_rng(7)
    # first call: random scores with ties, several rows of different lengths
    a = rng.integers(0, 20, (5, 30000)).astype(np.float32)
    ts_a = [29999, 20000, 5000, 1200, 190]
    (iw, cw), (ina, cna) = _select_both(a, ts_a)
    assert np.array_equal(cw, cna) and np.array_equal(iw, ina)
    assert (cw > 0).all()
    # second call, other shapes and values: the scratch left by the first call
    # must not leak into the result
    b = rng.standard_normal((3, 50001)).astype(np.float32)
    ts_b = [50000, 44444, 3000]
    (iw, cw), (ina, cna) = _select_both(b, ts_b)
    assert np.array_equal(cw, cna) and np.array_equal(iw, ina)


def test_noalloc_rejects_problems_larger_than_its_scratch():
    # rows x blocks of block maxima beyond the fixed 16 MiB
    ts = [4_000_000] * 70
    p, keep = _problem(ts, 4_000_001)
    need = hs2.hs2_block_select_workspace_size(p, 16, 64, 128)
    assert need > hs2.NOALLOC_SCRATCH_BYTES
    idx = torch.empty((1,), dtype=torch.int32).cuda()
    with pytest.raises(hs2.HS2Error) as e:
        # the score pointer is never touched: the size check comes first
        hs2.hs2_block_select_noalloc(p, idx, 4_000_001, 16, 64, 128, idx, idx)
    assert e.value.status == hs2.HS2_ERR_WORKSPACE
