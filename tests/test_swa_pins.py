"""Pins of oracle.swa_attention_row (CPU): brute force, the window covering the
whole context (= full attention), a window of one key, and planted mistakes."""
import inspect
import math

import numpy as np

import oracle
import oracle.swa as osw


def _brute(q, k, v, t, window, scale):
    """Pure-Python softmax attention over positions max(0, t-window+1)..t."""
    Hq, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    out = [[0.0] * D for _ in range(Hq)]
    pos = list(range(max(0, t - window + 1), t + 1))
    for h in range(Hq):
        g = h // G
        w = [math.exp(scale * sum(float(q[h, d]) * float(k[j, g, d]) for d in range(D))) for j in pos]
        s = math.fsum(w)
        for d in range(D):
            out[h][d] = math.fsum(w[i] * float(v[pos[i], g, d]) for i in range(len(pos))) / s
    return np.array(out)


def _case(seed, N=40, Hq=4, Hkv=2, D=6):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((Hq, D)), rng.standard_normal((N, Hkv, D)),
            rng.standard_normal((N, Hkv, D)))


def test_brute_force_tiny():
    for seed, t, W in [(1, 0, 3), (2, 5, 3), (3, 39, 7), (4, 20, 1), (5, 10, 100)]:
        q, k, v = _case(seed)
        got = oracle.swa_attention_row(q, k, v, t, W, 0.4)
        assert np.allclose(got, _brute(q, k, v, t, W, 0.4), rtol=1e-12, atol=1e-12), (seed, t, W)


def test_window_covering_the_context_is_full_attention():
    q, k, v = _case(6)
    for t in (0, 17, 39):
        O_full = oracle.full_attention_row(q, k, v, t, 0.3)[0]
        assert np.allclose(oracle.swa_attention_row(q, k, v, t, t + 1, 0.3), O_full, atol=1e-13)
        assert np.allclose(oracle.swa_attention_row(q, k, v, t, 10**6, 0.3), O_full, atol=1e-13)


def test_window_of_one_is_the_own_value_row():
    q, k, v = _case(7)
    O = oracle.swa_attention_row(q, k, v, 12, 1, 0.3)
    G = q.shape[0] // k.shape[1]
    for h in range(q.shape[0]):
        assert np.array_equal(O[h], v[12, h // G])


def test_keys_outside_the_window_do_not_matter():
    q, k, v = _case(8)
    t, W = 30, 5
    k2, v2 = k.copy(), v.copy()
    k2[: t - W + 1] = 1e3  # would dominate if visible
    k2[t + 1:] = 1e3
    assert np.allclose(oracle.swa_attention_row(q, k2, v2, t, W, 0.3),
                       oracle.swa_attention_row(q, k, v, t, W, 0.3), atol=1e-13)


def test_planted_mistakes_fail_a_pin():
    src = inspect.getsource(osw)
    mutants = [("lo, hi = max(0, t - window + 1), t + 1", "lo, hi = max(0, t - window), t + 1"),
               ("lo, hi = max(0, t - window + 1), t + 1", "lo, hi = max(0, t - window + 1), t"),
               ("x = scale * (Kg @ q_row[h])", "x = Kg @ q_row[h]"),
               ("for h in range(g * G, (g + 1) * G):", "for h in range(g, Hq, Hkv):")]
    pins = [test_brute_force_tiny, test_window_covering_the_context_is_full_attention,
            test_window_of_one_is_the_own_value_row]
    orig = oracle.swa_attention_row
    try:
        for old, new in mutants:
            assert old in src
            ns = {}
            exec(src.replace(old, new), ns)
            oracle.swa_attention_row = ns["swa_attention_row"]
            caught = 0
            for pin in pins:
                try:
                    pin()
                except (AssertionError, ValueError):
                    caught += 1
            assert caught > 0, new
    finally:
        oracle.swa_attention_row = orig
