"""Device offsets that disagree with the host totals (a caller bug the host
cannot see) are reported as HS2_ERR_DEVICE_INPUT by the kernels' own checks;
every access stays inside the buffers the host sizes describe, the sequences
with valid offsets keep their exact results, and the next clean call is
error-free."""
import numpy as np
import pytest
import torch

import synth
from long_context_full_b200 import hs2
from tests.gpu_util import CudaPathRun

pytestmark = pytest.mark.gpu


def _outputs(out):
    return {"O": out.O.clone(), "scores": out.scores.clone(), "idx": out.idx.clone(),
            "count": out.count.clone(), "O1": out.O_layers[0].clone()}


def _same_scores(a, b, tpos):
    """Score entries 0..t of every row (the only ones the call defines)."""
    return all(torch.equal(a[r, :t + 1], b[r, :t + 1]) for r, t in enumerate(tpos))


@pytest.mark.parametrize("bad", [[0, 2000, 3600], [0, -5, 3000]],
                         ids=["last_sequence_past_total", "negative_start"])
def test_inconsistent_kv_offsets_are_reported(bad):
    w = synth.make_workload("devin", 41, "bf16", 8, 2, 128, [2000, 1000], [1, 1], 1)
    tpos = np.repeat(w.query_positions(), w.Hkv)
    run = CudaPathRun(w)
    clean = _outputs(run.run())
    good = run.step.kv_offsets.clone()

    run.step.kv_offsets.copy_(torch.tensor(bad, dtype=torch.int64))
    out = _outputs(run.step.run(run.Q, run.K, run.V, run.QL))
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_ERR_DEVICE_INPUT
    if bad[1] == 2000:  # sequence 0's offsets are intact: its results are exact
        G = w.Hkv
        assert torch.equal(out["O"][0], clean["O"][0]) and torch.equal(out["O1"][0], clean["O1"][0])
        assert torch.equal(out["idx"][:G], clean["idx"][:G])
        assert torch.equal(out["count"][:G], clean["count"][:G])
        assert _same_scores(out["scores"][:G], clean["scores"][:G], tpos[:G])

    run.step.kv_offsets.copy_(good)
    again = _outputs(run.run())  # CudaPathRun.run asserts HS2_OK
    for name in ("O", "idx", "count", "O1"):
        assert torch.equal(again[name], clean[name]), name
    assert _same_scores(again["scores"], clean["scores"], tpos)
