"""Pins of oracle.kv_bridge (CPU): brute-force sums, weights that copy hidden
columns, linearity, and planted mistakes."""
import inspect

import numpy as np

import oracle
import oracle.bridge as ob


def _brute(H, W_t, Hkv, D):
    N, hidden = H.shape
    out = np.zeros((N, Hkv, D))
    for n in range(N):
        for g in range(Hkv):
            for d in range(D):
                out[n, g, d] = sum(float(H[n, i]) * float(W_t[g * D + d, i]) for i in range(hidden))
    return out


def test_brute_force_tiny():
    rng = np.random.default_rng(1)
    N, hidden, Hkv, D = 5, 7, 2, 3
    H = rng.standard_normal((N, hidden))
    Wk, Wv = rng.standard_normal((Hkv * D, hidden)), rng.standard_normal((Hkv * D, hidden))
    K, V = oracle.kv_bridge(H, Wk, Wv, Hkv, D)
    assert np.allclose(K, _brute(H, Wk, Hkv, D), atol=1e-12)
    assert np.allclose(V, _brute(H, Wv, Hkv, D), atol=1e-12)


def test_selection_weights_copy_hidden_columns():
    """Wk_t row c = unit vector e_{p(c)}: K[n, g, d] = H[n, p(g*D + d)] exactly."""
    rng = np.random.default_rng(2)
    N, hidden, Hkv, D = 4, 12, 2, 4
    H = rng.standard_normal((N, hidden))
    perm = rng.permutation(hidden)[: Hkv * D]
    W = np.zeros((Hkv * D, hidden))
    W[np.arange(Hkv * D), perm] = 1.0
    K, V = oracle.kv_bridge(H, W, 2.0 * W, Hkv, D)
    assert np.array_equal(K, H[:, perm].reshape(N, Hkv, D))
    assert np.array_equal(V, 2.0 * H[:, perm].reshape(N, Hkv, D))


def test_linear_in_the_hidden_states():
    rng = np.random.default_rng(3)
    H1, H2 = rng.standard_normal((3, 8)), rng.standard_normal((3, 8))
    W = rng.standard_normal((4, 8))
    K1, _ = oracle.kv_bridge(H1, W, W, 2, 2)
    K2, _ = oracle.kv_bridge(H2, W, W, 2, 2)
    K3, _ = oracle.kv_bridge(H1 + 3.0 * H2, W, W, 2, 2)
    assert np.allclose(K3, K1 + 3.0 * K2, atol=1e-12)


def test_planted_mistakes_fail_a_pin():
    src = inspect.getsource(ob)
    mutants = [("K = (H @ np.asarray(Wk_t, dtype=np.float64).T).reshape(N, Hkv, D)",
                "K = (H @ np.asarray(Wk_t, dtype=np.float64).T).reshape(N, D, Hkv).transpose(0, 2, 1)"),
               ("V = (H @ np.asarray(Wv_t, dtype=np.float64).T).reshape(N, Hkv, D)",
                "V = (H @ np.asarray(Wk_t, dtype=np.float64).T).reshape(N, Hkv, D)")]
    pins = [test_brute_force_tiny, test_selection_weights_copy_hidden_columns]
    orig = oracle.kv_bridge
    try:
        for old, new in mutants:
            assert old in src
            ns = {}
            exec(src.replace(old, new), ns)
            oracle.kv_bridge = ns["kv_bridge"]
            caught = 0
            for pin in pins:
                try:
                    pin()
                except AssertionError:
                    caught += 1
            assert caught > 0, new
    finally:
        oracle.kv_bridge = orig
