"""KV Bridging GEMM (tcgen05) through the C ABI against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
from long_context_full_b200 import hs2
from tests.gpu_util import to_device, to_f64

pytestmark = pytest.mark.gpu


def _bits(x):
    return synth.f32_to_bf16_bits(np.ascontiguousarray(x, dtype=np.float32))


@pytest.mark.parametrize("rows,hidden,Hkv", [(3000, 512, 4), (129, 64, 1), (700, 192, 2)])
def test_bridge_matches_oracle(rows, hidden, Hkv):
    """Ragged last tile (rows not a multiple of 128), one and several K stages,
    both column tilings (Hkv*D = 512, 256: tiles of 256; 128: tiles of 128).
    Output is bf16-rounded fp32 accumulation: |GPU - exact| <= 2^-8 |exact| + 1e-4."""
    rng = np.random.default_rng(rows + hidden)
    D = 128
    H = _bits(rng.standard_normal((rows, hidden)))
    Wk = _bits(rng.standard_normal((Hkv * D, hidden)) / np.sqrt(hidden))
    Wv = _bits(rng.standard_normal((Hkv * D, hidden)) / np.sqrt(hidden))
    ko = torch.tensor([0, rows], dtype=torch.int64).cuda()
    qo = torch.tensor([0, 0], dtype=torch.int64).cuda()
    p = hs2.make_problem(1, Hkv, Hkv, D, hs2.HS2_BF16, qo, ko, 0, rows, 0, rows, 0.1)
    K = torch.empty(rows, Hkv, D, dtype=torch.bfloat16, device="cuda")
    V = torch.empty_like(K)
    hs2.hs2_kv_bridge(p, to_device(H, "bf16"), hidden, to_device(Wk, "bf16"), to_device(Wv, "bf16"), K, V)
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
    f = lambda b: synth.stored_to_f64(b, "bf16")
    Kr, Vr = oracle.kv_bridge(f(H), f(Wk), f(Wv), Hkv, D)
    for got, ref in ((to_f64(K), Kr), (to_f64(V), Vr)):
        err = np.abs(got - ref)
        assert (err <= 2.0 ** -8 * np.abs(ref) + 1e-4).all(), float((err / (np.abs(ref) + 1e-4)).max())


def test_bridge_rejects_fp32_and_bad_hidden():
    ko = torch.tensor([0, 10], dtype=torch.int64).cuda()
    qo = torch.tensor([0, 0], dtype=torch.int64).cuda()
    x = torch.zeros(10, 128, dtype=torch.bfloat16, device="cuda")
    p32 = hs2.make_problem(1, 1, 1, 128, hs2.HS2_F32, qo, ko, 0, 10, 0, 10, 0.1)
    with pytest.raises(hs2.HS2Error) as e:
        hs2.hs2_kv_bridge(p32, x, 128, x, x, x, x)
    assert e.value.status == hs2.HS2_ERR_UNSUPPORTED
    p = hs2.make_problem(1, 1, 1, 128, hs2.HS2_BF16, qo, ko, 0, 10, 0, 10, 0.1)
    with pytest.raises(hs2.HS2Error) as e:
        hs2.hs2_kv_bridge(p, x, 100, x, x, x, x)
    assert e.value.status == hs2.HS2_ERR_INVALID_ARG
