"""The benchmark's algorithmic byte counts (the numerators of every roofline
fraction it reports) against sizes worked out by hand from the workload shapes."""
import types

import numpy as np

import bench


def _shape(kv, q, Hq=32, Hkv=4, D=128, dtype="bf16"):
    w = types.SimpleNamespace(dtype=dtype, kv_lens=np.asarray(kv), q_lens=np.asarray(q), Hq=Hq,
                              Hkv=Hkv, D=D)
    # decode rows sit at the end of their sequences
    w.query_positions = lambda: np.concatenate(
        [np.arange(n - t, n) for n, t in zip(w.kv_lens, w.q_lens)])
    return w


def test_decode_b8_128k_accounting():
    a = bench.workload_accounting(_shape([131072] * 8, [1] * 8), 4)
    kv = 2 * (8 * 131072) * 4 * 128 * 2          # K and V, bf16, read once
    qo = 2 * 8 * 32 * 128 * 2                      # Q read, O written
    scores = 8 * 131072 * 4 * 4                    # one float per visible key and KV group
    assert a["kv"] == kv == 2_147_483_648
    assert a["full"] == kv + qo + scores == 2_164_391_936
    sel = scores + 8 * 4 * (1152 + 1) * 4          # scores read, indices and counts written
    sparse = 8 * 4 * 1152 * 128 * 2 * 2 + qo       # selected K and V rows, Q_l and O_l
    assert a["select"] == sel and a["sparse_layer"] == sparse
    assert a["step"] == a["full"] + sel + 4 * sparse == 2_257_338_496
    assert a["flops"] == 4 * 128 * 32 * 8 * 131072


def test_needle_1m_and_short_rows_accounting():
    a = bench.workload_accounting(_shape([1048576], [1]), 4)
    assert a["step"] == 2_190_575_632
    # a sequence shorter than k + window gathers only its visible rows
    b = bench.workload_accounting(_shape([700], [1], Hq=8, Hkv=2), 1)
    assert b["sparse_layer"] == 2 * 700 * 128 * 2 * 2 + 2 * 8 * 128 * 2


def test_chunk_accounting_counts_causal_visibility():
    a = bench.workload_accounting(_shape([1000], [10]), 1)
    visible = sum(range(991, 1001))                # query i of the chunk sees 991 + i keys
    assert a["flops"] == 4 * 128 * 32 * visible
    assert a["full"] == 2 * 1000 * 4 * 128 * 2 + 2 * 10 * 32 * 128 * 2 + visible * 4 * 4
