"""Host logic of the seeded input generator (no attention arithmetic here)."""
import numpy as np
import torch

import synth


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).standard_normal(100_000).astype(np.float32) * 37.0
    x[:4] = [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0]  # ties to even, exact values
    ours = synth.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = synth.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(ours.view(np.int16)).view(torch.bfloat16).float().numpy())


def test_streams_are_deterministic_and_thread_independent():
    a = synth.normal_tokens(5, synth.TID_K, 3, 20000, (2, 8), "bf16")
    b = synth.normal_tokens(5, synth.TID_K, 3, 20000, (2, 8), "bf16")
    assert np.array_equal(a, b)
    c = synth.normal_tokens(5, synth.TID_K, 4, 20000, (2, 8), "bf16")
    assert not np.array_equal(a, c)
    # a prefix of the same stream gives the same rows
    d = synth.normal_tokens(5, synth.TID_K, 3, 9000, (2, 8), "bf16")
    assert np.array_equal(a[:9000], d)


def test_shard_draws_the_same_sequences():
    full = synth.make_workload("x", 7, "bf16", 4, 2, 16, [300, 200, 100], [1, 1, 1], 2)
    part = synth.make_workload("x", 7, "bf16", 4, 2, 16, [200, 100], [1, 1], 2, seq_ids=[1, 2])
    ko = full.kv_offsets
    assert np.array_equal(full.k[ko[1]:], part.k)
    assert np.array_equal(full.v[ko[1]:], part.v)
    assert np.array_equal(full.q[1:], part.q)
    assert np.array_equal(full.q_layers[1][1:], part.q_layers[1])


def test_needles_outside_window_and_aligned_with_query():
    w = synth.make_workload("n", 9, "bf16", 8, 2, 128, [5000], [1], 1, n_needles=64)
    pos = w.needle_pos[0]
    assert len(set(pos.tolist())) == 64 and pos.min() >= 0 and pos.max() <= 5000 - 129
    G = w.Hq // w.Hkv
    q = synth.stored_to_f64(w.q[0], "bf16")
    for g in range(w.Hkv):
        kn = synth.stored_to_f64(w.k[pos, g], "bf16")
        unit = q[g * G] / np.linalg.norm(q[g * G])
        proj = kn @ unit
        assert np.all(np.abs(proj - 4.0) < 1.0)


def test_ragged_lengths_in_range():
    n = synth.ragged_lengths(1239, 16, 8192, 524288)
    assert n.min() >= 8192 and n.max() <= 524288 and len(n) == 16
    assert np.array_equal(n, synth.ragged_lengths(1239, 16, 8192, 524288))


def test_query_positions():
    w = synth.make_workload("c", 3, "f32", 2, 1, 8, [10, 7], [3, 1], 0)
    assert list(w.query_positions()) == [7, 8, 9, 6]
    assert list(w.query_seq()) == [0, 0, 0, 1]
