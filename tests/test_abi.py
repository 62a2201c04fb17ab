"""The C-ABI library loads, exports every function include/hs2.h declares, and
rejects bad arguments on the host before touching the GPU."""
import ctypes
import os
import re

import pytest

from long_context_full_b200 import hs2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hs2.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hs2_[a-z_0-9]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from long_context_full_b200 import build
    build.build()
    return hs2.load()


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert "hs2_full_attn_scores" in names and "hs2_topk_select" in names
    assert "hs2_sparse_attn" in names and "hs2_block_select" in names
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(hs2.EXPORTED) == names


def test_status_strings_and_version(lib):
    assert hs2.status_string(0) == "ok"
    for code in range(-6, 0):
        assert hs2.status_string(code) not in ("ok", "unknown status")
    assert hs2.status_string(-99) == "unknown status"
    assert hs2.hs2_version() >= 1


def _problem(**kw):
    d = dict(B=1, Hq=8, Hkv=2, D=128, dtype=hs2.HS2_BF16, q_offsets=0x1000, kv_offsets=0x2000,
             total_q=1, total_kv=100, max_q_len=1, max_kv_len=100, scale=0.0884)
    d.update(kw)
    return hs2.make_problem(**d)


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=7), hs2.HS2_ERR_INVALID_ARG),          # Hq % Hkv != 0
    (dict(B=0), hs2.HS2_ERR_INVALID_ARG),
    (dict(dtype=5), hs2.HS2_ERR_INVALID_ARG),
    (dict(q_offsets=None), hs2.HS2_ERR_INVALID_ARG),
    (dict(total_kv=1000), hs2.HS2_ERR_INVALID_ARG),   # more keys than B * max_kv_len
    (dict(max_q_len=200), hs2.HS2_ERR_INVALID_ARG),   # queries longer than the cache
    (dict(scale=float("nan")), hs2.HS2_ERR_INVALID_ARG),
    (dict(D=64), hs2.HS2_ERR_UNSUPPORTED),
    (dict(Hq=32, Hkv=2), hs2.HS2_ERR_UNSUPPORTED),    # bf16 group of 16 heads
])
def test_problem_validation(lib, kw, code):
    p = _problem(**kw)
    n = ctypes.c_size_t(0)
    assert lib.hs2_topk_workspace_size(ctypes.byref(p), 1024, 128, ctypes.byref(n)) == code
    assert lib.hs2_full_attn_workspace_size(ctypes.byref(p), ctypes.byref(n)) == code
    rc = lib.hs2_topk_select(ctypes.byref(p), 0x3000, 128, 1024, 128, 0x4000, 0x5000, None, 0, None)
    assert rc == code


def test_null_problem_and_bad_call_arguments(lib):
    n = ctypes.c_size_t(0)
    assert lib.hs2_topk_workspace_size(None, 1024, 128, ctypes.byref(n)) == hs2.HS2_ERR_INVALID_ARG
    p = _problem()
    assert lib.hs2_topk_workspace_size(ctypes.byref(p), 0, 128, ctypes.byref(n)) == hs2.HS2_ERR_INVALID_ARG
    # score stride shorter than the longest sequence
    assert lib.hs2_topk_select(ctypes.byref(p), 0x3000, 50, 1024, 128, 0x4000, 0x5000, None, 0,
                               None) == hs2.HS2_ERR_INVALID_ARG
    # misaligned scores pointer
    assert lib.hs2_topk_select(ctypes.byref(p), 0x3004, 128, 1024, 128, 0x4000, 0x5000, None, 0,
                               None) == hs2.HS2_ERR_INVALID_ARG
    # null outputs
    assert lib.hs2_full_attn_scores(ctypes.byref(p), 0x1000, 0x1000, 0x1000, None, 0x1000, 128,
                                    None, 0, None) == hs2.HS2_ERR_INVALID_ARG


def test_workspace_sizes(lib):
    """Selection and sparse layers keep their state on chip; block selection
    needs the block maxima and the chosen block ids (each 256-byte rounded)."""
    p = _problem(total_q=3, B=3, max_kv_len=10000, total_kv=20000)
    n = ctypes.c_size_t(123)
    assert lib.hs2_topk_workspace_size(ctypes.byref(p), 1024, 128, ctypes.byref(n)) == 0
    assert n.value == 0
    assert lib.hs2_block_select_workspace_size(ctypes.byref(p), 16, 64, 128, ctypes.byref(n)) == 0
    rows = 3 * 2
    rnd = lambda b: (b + 255) // 256 * 256
    nb = (10000 + 63) // 64
    assert n.value == rnd(rows * nb * 4) + rnd(rows * 16 * 4)


def test_wait_selftest_rejects_bad_arguments_on_the_host(lib):
    """Checked before any CUDA call, so it runs without a GPU."""
    assert lib.hs2_wait_selftest(2, 1000, None) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_wait_selftest(-1, 1000, None) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_wait_selftest(0, -5, None) == hs2.HS2_ERR_INVALID_ARG


def test_context_parallel_calls_reject_bad_arguments_on_the_host(lib):
    """Checked before any CUDA call, so it runs without a GPU."""
    P = lambda **kw: ctypes.byref(_problem(**kw))
    # chunks are not split across ranks
    chunk = dict(max_q_len=4, total_q=4)
    assert lib.hs2_cp_attn_partial(P(**chunk), 0x1000, 0x1000, 0x1000, 0x2000, 0x3000, None, 0,
                                   None) == hs2.HS2_ERR_UNSUPPORTED
    assert lib.hs2_cp_scores(P(**chunk), 0x3000, 0x4000, 128, None, 0, None) == hs2.HS2_ERR_UNSUPPORTED
    assert lib.hs2_cp_topk_local(P(**chunk), 0x4000, 128, 1024, 128, 0x5000, 0x6000, 0x7000, 0x8000,
                                 0x9000, None) == hs2.HS2_ERR_UNSUPPORTED
    assert lib.hs2_cp_sparse_partial(P(**chunk), 0x1000, 0x1000, 0x1000, 0x6000, 0x7000, 1152,
                                     0x5000, 0x2000, 0x3000, None) == hs2.HS2_ERR_UNSUPPORTED
    # missing buffers, bad sizes
    assert lib.hs2_cp_attn_partial(P(), 0x1000, 0x1000, 0x1000, None, 0x3000, None, 0,
                                   None) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_cp_scores(P(), 0x3000, 0x4000, 50, None, 0, None) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_cp_topk_local(P(), 0x4000, 128, 1024, 128, None, 0x6000, 0x7000, 0x8000, 0x9000,
                                 None) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_cp_topk_local(P(), 0x4000, 128, 0, 128, 0x5000, 0x6000, 0x7000, 0x8000, 0x9000,
                                 None) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_cp_sparse_partial(P(), 0x1000, 0x1000, 0x1000, 0x6000, 0x7000, 1152, None,
                                     0x2000, 0x3000, None) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_cp_merge(-1, 2, 0x1000, 0x2000, hs2.HS2_BF16, 0x3000, None, None) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_cp_merge(8, 0, 0x1000, 0x2000, hs2.HS2_BF16, 0x3000, None, None) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_cp_merge(8, 2, 0x1000, 0x2000, 7, 0x3000, None, None) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_cp_merge(0, 2, 0x1000, 0x2000, hs2.HS2_BF16, 0x3000, None, None) == hs2.HS2_OK
    # the merged selection's shared-memory limits: k <= 2048, R (k + window) <= 16384
    assert lib.hs2_cp_topk_merge(P(), 2, 4096, 128, 0x1000, 0x2000, 0x3000, 0x4000,
                                 None) == hs2.HS2_ERR_UNSUPPORTED
    assert lib.hs2_cp_topk_merge(P(), 16, 1024, 128, 0x1000, 0x2000, 0x3000, 0x4000,
                                 None) == hs2.HS2_ERR_UNSUPPORTED
    assert lib.hs2_cp_topk_merge(P(), 0, 1024, 128, 0x1000, 0x2000, 0x3000, 0x4000,
                                 None) == hs2.HS2_ERR_INVALID_ARG


def test_empty_step_returns_ok_without_pointers(lib):
    """total_q = 0: every call checks the problem and its scalars, launches
    nothing and returns HS2_OK with null tensor and workspace pointers (no
    device is touched, so this runs without a GPU)."""
    P = lambda **kw: ctypes.byref(_problem(**dict(dict(total_q=0, B=2, total_kv=150), **kw)))
    assert lib.hs2_full_attn_scores(P(), None, None, None, None, None, 128, None, 0, None) == hs2.HS2_OK
    assert lib.hs2_full_attn_scores(P(max_q_len=0), None, None, None, None, None, 128, None, 0,
                                    None) == hs2.HS2_OK
    assert lib.hs2_topk_select(P(), None, 128, 1024, 128, None, None, None, 0, None) == hs2.HS2_OK
    assert lib.hs2_block_select(P(), None, 128, 16, 64, 128, None, None, None, 0, None) == hs2.HS2_OK
    assert lib.hs2_block_select_noalloc(P(), None, 128, 16, 64, 128, None, None, None) == hs2.HS2_OK
    assert lib.hs2_sparse_attn(P(), None, None, None, None, None, 1152, None, None, 0, None) == hs2.HS2_OK
    assert lib.hs2_swa_attn(P(), None, None, None, 128, None, None) == hs2.HS2_OK
    assert lib.hs2_kv_append(P(), None, None, None, None, None) == hs2.HS2_OK
    assert lib.hs2_cp_attn_partial(P(), None, None, None, None, None, None, 0, None) == hs2.HS2_OK
    assert lib.hs2_cp_scores(P(), None, None, 128, None, 0, None) == hs2.HS2_OK
    assert lib.hs2_cp_topk_local(P(), None, 128, 1024, 128, None, None, None, None, None,
                                 None) == hs2.HS2_OK
    assert lib.hs2_cp_topk_merge(P(), 2, 1024, 128, None, None, None, None, None) == hs2.HS2_OK
    assert lib.hs2_cp_sparse_partial(P(), None, None, None, None, None, 1152, None, None, None,
                                     None) == hs2.HS2_OK
    # the scalar arguments are still checked
    assert lib.hs2_topk_select(P(), None, 128, 0, 128, None, None, None, 0, None) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_block_select(P(), None, 128, 16, 0, 128, None, None, None, 0,
                                None) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_sparse_attn(P(), None, None, None, None, None, 0, None, None, 0,
                               None) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_swa_attn(P(), None, None, None, 0, None, None) == hs2.HS2_ERR_INVALID_ARG
    assert lib.hs2_full_attn_scores(P(Hq=7), None, None, None, None, None, 128, None, 0,
                                    None) == hs2.HS2_ERR_INVALID_ARG
