"""Pins of oracle.kv_append (CPU): the rows a step writes are exactly the new
tokens' own positions, and attention of a new query sees its own key as the
last visible one."""
import numpy as np

import oracle


def _case(rng, q_lens, kv_lens, Hkv=2, D=8):
    qo = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int64)
    ko = np.concatenate([[0], np.cumsum(kv_lens)]).astype(np.int64)
    K = rng.standard_normal((ko[-1], Hkv, D))
    V = rng.standard_normal((ko[-1], Hkv, D))
    Kn = rng.standard_normal((qo[-1], Hkv, D))
    Vn = rng.standard_normal((qo[-1], Hkv, D))
    return qo, ko, K, V, Kn, Vn


def test_only_the_last_tq_rows_of_each_sequence_change():
    rng = np.random.default_rng(3)
    q_lens, kv_lens = [1, 3, 0, 2], [5, 7, 4, 2]
    qo, ko, K, V, Kn, Vn = _case(rng, q_lens, kv_lens)
    K2, V2 = oracle.kv_append(K, V, Kn, Vn, qo, ko)
    changed = np.zeros(ko[-1], dtype=bool)
    for b in range(len(q_lens)):
        for i in range(q_lens[b]):
            r = ko[b + 1] - q_lens[b] + i  # brute force: the sequence's last Tq rows, in order
            changed[r] = True
            assert np.array_equal(K2[r], Kn[qo[b] + i]) and np.array_equal(V2[r], Vn[qo[b] + i])
    assert np.array_equal(K2[~changed], K[~changed]) and np.array_equal(V2[~changed], V[~changed])
    assert not np.shares_memory(K2, K)  # inputs untouched
    assert changed.sum() == sum(q_lens)


def test_new_query_sees_its_own_key_last():
    """A new key aligned with its own query (logit 60 above the rest) takes all
    the attention of that query: O = its own new V row, and positions past t
    (later new tokens) are not visible."""
    rng = np.random.default_rng(5)
    q_lens, kv_lens = [3], [9]
    Hkv, D = 1, 8
    qo, ko, K, V, Kn, Vn = _case(rng, q_lens, kv_lens, Hkv, D)
    K *= 0.01
    q = rng.standard_normal((q_lens[0], 1, D))
    scale = 1.0
    for i in range(q_lens[0]):
        Kn[i, 0] = q[i, 0] * 60.0 / (q[i, 0] @ q[i, 0])  # q . k_new = 60
    for i in range(q_lens[0]):
        Kn_i = Kn.copy()
        # keys of the later new tokens would dominate too if they were visible
        for i2 in range(i + 1, q_lens[0]):
            Kn_i[i2, 0] = q[i, 0] * 80.0 / (q[i, 0] @ q[i, 0])
        K2, V2 = oracle.kv_append(K, V, Kn_i, Vn, qo, ko)
        t = kv_lens[0] - q_lens[0] + i
        O, m, l, P = oracle.full_attention_row(q[i], K2, V2, t, scale)
        assert P.shape[1] == t + 1 and P[0, t] > 1 - 1e-12
        assert np.allclose(O[0], Vn[i, 0], atol=1e-12)


def test_empty_step_is_identity():
    rng = np.random.default_rng(7)
    qo, ko, K, V, Kn, Vn = _case(rng, [0, 0], [3, 4])
    K2, V2 = oracle.kv_append(K, V, Kn, Vn, qo, ko)
    assert np.array_equal(K2, K) and np.array_equal(V2, V)


def test_planted_mistakes_fail_a_pin():
    """Copies of the oracle with a plausible mistake (position off by one, the
    query's index used as the position, new rows in reverse order) each fail
    one of the pins above."""
    import inspect
    import oracle.cache as oc
    src = inspect.getsource(oc)
    mutants = [("t = n_kv - n_q + i", "t = n_kv - n_q + i - 1"),
               ("t = n_kv - n_q + i", "t = i"),
               ("K[ko[b] + t] = K_new[qo[b] + i]", "K[ko[b] + t] = K_new[qo[b] + n_q - 1 - i]")]
    pins = [test_only_the_last_tq_rows_of_each_sequence_change, test_new_query_sees_its_own_key_last]
    orig = oracle.kv_append
    try:
        for old, new in mutants:
            assert old in src
            ns = {}
            exec(src.replace(old, new), ns)
            oracle.kv_append = ns["kv_append"]
            caught = 0
            for pin in pins:
                try:
                    pin()
                except AssertionError:
                    caught += 1
            assert caught > 0, new
    finally:
        oracle.kv_append = orig
