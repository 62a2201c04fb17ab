"""Bounds and placement checks of the whole hybrid-block path.

Every output and the workspace are carved out of one arena pre-filled with a
canary byte, each region fenced by canary guards.  After full attention,
token selection and one sparse layer:

* every guard byte is intact (no write outside an output or the workspace);
* score entries past each row's query position keep the canary (the kernels
  write positions 0..t of a row and nothing else), including when the score
  row stride is not a multiple of four floats;
* the index padding past ``count`` is -1 and no canary is left in any
  output;
* all values are bit-identical to the same step run in ordinary buffers
  (whose results the parity tests compare with the oracle), and a few rows are
  checked against the oracle here as well.
"""
import numpy as np
import pytest
import torch

import synth
from long_context_full_b200 import hs2
from tests.gpu_util import CudaPathRun, OracleRows, check_O, check_scores, to_f64

pytestmark = pytest.mark.gpu

GUARD = 4096
CANARY = 0xA5


class Arena:
    """Named regions inside one canary-filled device buffer, fenced by guards."""

    def __init__(self, regions):
        self.offs, pos = {}, GUARD
        for name, nbytes in regions:
            self.offs[name] = (pos, nbytes)
            pos += (nbytes + 255) // 256 * 256 + GUARD
        self.buf = torch.full((pos,), CANARY, dtype=torch.uint8, device="cuda")

    def view(self, name, dtype, shape):
        o, n = self.offs[name]
        if n == 0:
            return None
        return self.buf[o:o + n].view(dtype).view(shape)

    def host_bytes(self, name):
        o, n = self.offs[name]
        return self.buf[o:o + n].cpu().numpy()

    def guards_intact(self) -> bool:
        host = self.buf.cpu().numpy()
        keep = np.ones(host.size, dtype=bool)
        for o, n in self.offs.values():
            keep[o:o + n] = False
        return bool((host[keep] == CANARY).all())


CASES = {
    # decode, three ragged caches (one shorter than the window + k)
    "decode_bf16": ("bf16", 16, 2, [5000, 1300, 129], [1, 1, 1]),
    # chunks on a cache: several query tiles, ragged last tile
    "chunk_bf16": ("bf16", 16, 2, [3000, 700], [200, 37]),
    "chunk_f32": ("f32", 8, 2, [1500], [64]),
}


@pytest.mark.parametrize("pad", [0, 13], ids=["stride4", "stride_odd"])
@pytest.mark.parametrize("case", list(CASES))
def test_outputs_stay_in_bounds(case, pad):
    dtype, Hq, Hkv, kv_lens, q_lens = CASES[case]
    w = synth.make_workload("can_" + case, 97, dtype, Hq, Hkv, 128, kv_lens, q_lens, 1)
    ref = CudaPathRun(w)
    out = ref.run()
    step = ref.step
    p = step.problem
    esz = 2 if dtype == "bf16" else 4
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    stride = step.stride + pad
    rows, tq = step.rows, step.total_q
    ws = max(hs2.hs2_full_attn_workspace_size(p),
             hs2.hs2_topk_workspace_size(p, step.k, step.window),
             hs2.hs2_sparse_attn_workspace_size(p, step.idx_stride))
    a = Arena([("O", tq * Hq * 128 * esz), ("scores", rows * stride * 4),
               ("idx", rows * step.idx_stride * 4), ("count", rows * 4),
               ("OL", tq * Hq * 128 * esz), ("ws", ws)])
    O = a.view("O", tdt, (tq, Hq, 128))
    S = a.view("scores", torch.float32, (rows, stride))
    idx = a.view("idx", torch.int32, (rows, step.idx_stride))
    cnt = a.view("count", torch.int32, (rows,))
    OL = a.view("OL", tdt, (tq, Hq, 128))
    W = a.view("ws", torch.uint8, (ws,))

    hs2.hs2_full_attn_scores(p, ref.Q, ref.K, ref.V, O, S, stride, W)
    hs2.hs2_topk_select(p, S, stride, step.k, step.window, idx, cnt, W)
    hs2.hs2_sparse_attn(p, ref.QL[0], ref.K, ref.V, idx, cnt, step.idx_stride, OL, W)
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK

    assert a.guards_intact()
    tpos = np.repeat(w.query_positions(), Hkv)
    sb = a.host_bytes("scores").reshape(rows, stride * 4)
    for r in range(rows):
        assert (sb[r, (tpos[r] + 1) * 4:] == CANARY).all(), f"score row {r} written past t"
    for name in ("O", "OL", "count"):
        assert not (a.host_bytes(name).reshape(-1, 4) == CANARY).all(axis=1).any(), name

    # the same values as the step in ordinary buffers
    assert torch.equal(O, out.O) and torch.equal(OL, out.O_layers[0])
    assert torch.equal(cnt, out.count) and torch.equal(idx, out.idx)
    s_host, r_host = S.cpu().numpy(), out.scores.cpu().numpy()
    for r in range(rows):
        assert np.array_equal(s_host[r, :tpos[r] + 1].view(np.uint32),
                              r_host[r, :tpos[r] + 1].view(np.uint32)), r
    i_host, c_host = idx.cpu().numpy(), cnt.cpu().numpy()
    for r in range(rows):
        assert (i_host[r, c_host[r]:] == -1).all()

    # and a few rows against the oracle
    orc = OracleRows(w)
    O64 = to_f64(O)
    for q in sorted({0, tq // 2, tq - 1}):
        Or, sc, t = orc.full(q)
        check_O(O64[q], Or, dtype, f"{case} O row {q}")
        for g in range(Hkv):
            check_scores(s_host[q * Hkv + g, :t + 1].astype(np.float64), sc[g],
                         f"{case} scores row {q}/{g}")
