"""Failure detection on the GPU without a fault: a bounded device wait that
nothing ends runs out, records HS2_ERR_TIMEOUT in the device error word, the
host reads and clears it, and the context keeps working."""
import numpy as np
import pytest
import torch

import oracle
import synth
from long_context_full_b200 import hs2
from tests.gpu_util import to_device

pytestmark = pytest.mark.gpu

# clock64() counts SM cycles; B200 SMs run at most 1965 MHz, so a wait of
# ``limit`` cycles lasts at least limit / 2.0e9 seconds.
MAX_SM_HZ = 2.0e9


def _small_append_matches_oracle():
    w = synth.make_workload("wt", 303, "bf16", 8, 2, 128, [300, 40], [1, 3], 0)
    rng = np.random.default_rng(5)
    n = int(w.q_lens.sum())
    Kn = synth.f32_to_bf16_bits(rng.standard_normal((n, 2, 128)).astype(np.float32))
    Vn = synth.f32_to_bf16_bits(rng.standard_normal((n, 2, 128)).astype(np.float32))
    qo = torch.from_numpy(w.q_offsets).cuda()
    ko = torch.from_numpy(w.kv_offsets).cuda()
    p = hs2.make_problem(w.B, 8, 2, 128, hs2.HS2_BF16, qo, ko, n, int(w.kv_lens.sum()),
                         int(w.q_lens.max()), int(w.kv_lens.max()), w.scale)
    K, V = to_device(w.k, "bf16"), to_device(w.v, "bf16")
    hs2.hs2_kv_append(p, to_device(Kn, "bf16"), to_device(Vn, "bf16"), K, V)
    status = hs2.hs2_get_last_device_error()
    Kr, Vr = oracle.kv_append(w.k, w.v, Kn, Vn, w.q_offsets, w.kv_offsets)
    bits = lambda t: t.cpu().view(torch.int16).numpy().view(np.uint16)
    return status, np.array_equal(bits(K), Kr) and np.array_equal(bits(V), Vr)


@pytest.mark.parametrize("mode", [0, 1], ids=["mbarrier", "flag"])
def test_wait_runs_out_and_is_reported(mode):
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK      # start from a clear word
    limit = 20_000_000
    s = torch.cuda.current_stream()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s)
    hs2.hs2_wait_selftest(mode, limit)
    t1.record(s)
    assert hs2.hs2_get_last_device_error() == hs2.HS2_ERR_TIMEOUT
    # the wait really spun for its limit before giving up
    assert t0.elapsed_time(t1) >= 0.9 * 1e3 * limit / MAX_SM_HZ
    # reading the word cleared it
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
    # the context is still usable: a real kernel runs and matches the oracle
    status, same = _small_append_matches_oracle()
    assert status == hs2.HS2_OK and same


def test_first_error_is_kept_until_read():
    """Two waits that run out, then a clean kernel: the word holds the timeout
    until the host reads it, and nothing after that reports an error."""
    hs2.hs2_get_last_device_error()
    hs2.hs2_wait_selftest(0, 1_000_000)
    hs2.hs2_wait_selftest(1, 1_000_000)
    status, same = _small_append_matches_oracle()
    assert status == hs2.HS2_ERR_TIMEOUT and same
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK


def test_zero_limit_gives_up_at_once():
    """A zero limit gives up after the first failed check."""
    hs2.hs2_get_last_device_error()
    hs2.hs2_wait_selftest(0, 0)
    assert hs2.hs2_get_last_device_error() == hs2.HS2_ERR_TIMEOUT
