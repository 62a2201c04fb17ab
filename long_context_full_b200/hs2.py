"""Python binding of the hs2 C ABI (include/hs2.h): argument marshalling only.

Every step of the path runs in the CUDA kernels of ``libhs2.so``; this module
turns torch tensors into device pointers and checks status codes.  There is
no fallback: if the library is missing or fails, the call raises.

The functions keep the C names.  Tensors are passed as torch CUDA tensors (or
raw integer device addresses); ``stream`` defaults to torch's current stream.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhs2.so")

HS2_OK = 0
HS2_ERR_INVALID_ARG = -1
HS2_ERR_UNSUPPORTED = -2
HS2_ERR_WORKSPACE = -3
HS2_ERR_CUDA = -4
HS2_ERR_TIMEOUT = -5
HS2_ERR_DEVICE_INPUT = -6

HS2_F32 = 0
HS2_BF16 = 1

EXPORTED = [
    "hs2_full_attn_workspace_size", "hs2_full_attn_launches", "hs2_full_attn_scores",
    "hs2_topk_workspace_size", "hs2_topk_select",
    "hs2_block_select_workspace_size", "hs2_block_select", "hs2_block_select_noalloc",
    "hs2_sparse_attn_workspace_size", "hs2_sparse_attn", "hs2_kv_append", "hs2_swa_attn",
    "hs2_kv_bridge", "hs2_wait_selftest",
    "hs2_cp_attn_partial", "hs2_cp_merge", "hs2_cp_scores", "hs2_cp_topk_local",
    "hs2_cp_topk_merge", "hs2_cp_sparse_partial",
    "hs2_get_last_device_error", "hs2_status_string", "hs2_version",
]


class Problem(ctypes.Structure):
    """Mirror of ``hs2_problem``."""
    _fields_ = [
        ("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
        ("D", ctypes.c_int32), ("dtype", ctypes.c_int32), ("reserved", ctypes.c_int32),
        ("q_offsets", ctypes.c_void_p), ("kv_offsets", ctypes.c_void_p),
        ("total_q", ctypes.c_int64), ("total_kv", ctypes.c_int64),
        ("max_q_len", ctypes.c_int64), ("max_kv_len", ctypes.c_int64),
        ("scale", ctypes.c_float),
    ]


class HS2Error(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


_lib = None


def load() -> ctypes.CDLL:
    """Loads libhs2.so (built in place by ``long_context_full_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"hs2 CUDA library not built: {LIB_PATH} is missing "
                           "(run python -m long_context_full_b200.build)")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(Problem)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    psz = ctypes.POINTER(ctypes.c_size_t)
    sig = {
        "hs2_full_attn_workspace_size": [P, psz],
        "hs2_full_attn_launches": [P, ctypes.POINTER(i32)],
        "hs2_full_attn_scores": [P, vp, vp, vp, vp, vp, i64, vp, sz, vp],
        "hs2_topk_workspace_size": [P, i32, i32, psz],
        "hs2_topk_select": [P, vp, i64, i32, i32, vp, vp, vp, sz, vp],
        "hs2_block_select_workspace_size": [P, i32, i32, i32, psz],
        "hs2_block_select": [P, vp, i64, i32, i32, i32, vp, vp, vp, sz, vp],
        "hs2_block_select_noalloc": [P, vp, i64, i32, i32, i32, vp, vp, vp],
        "hs2_sparse_attn_workspace_size": [P, i32, psz],
        "hs2_sparse_attn": [P, vp, vp, vp, vp, vp, i32, vp, vp, sz, vp],
        "hs2_kv_append": [P, vp, vp, vp, vp, vp],
        "hs2_swa_attn": [P, vp, vp, vp, i32, vp, vp],
        "hs2_kv_bridge": [P, vp, i32, vp, vp, vp, vp, vp],
        "hs2_wait_selftest": [i32, i64, vp],
        "hs2_cp_attn_partial": [P, vp, vp, vp, vp, vp, vp, sz, vp],
        "hs2_cp_merge": [i64, i32, vp, vp, i32, vp, vp, vp],
        "hs2_cp_scores": [P, vp, vp, i64, vp, sz, vp],
        "hs2_cp_topk_local": [P, vp, i64, i32, i32, vp, vp, vp, vp, vp, vp],
        "hs2_cp_topk_merge": [P, i32, i32, i32, vp, vp, vp, vp, vp],
        "hs2_cp_sparse_partial": [P, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp],
        "hs2_get_last_device_error": [vp],
        "hs2_status_string": [ctypes.c_int],
        "hs2_version": [],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_char_p if name == "hs2_status_string" else ctypes.c_int
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().hs2_status_string(int(status)).decode()


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if isinstance(x, torch.Tensor):
        if x.numel() and not x.is_cuda:
            raise ValueError("hs2 takes device tensors")
        return x.data_ptr() if x.numel() else None
    raise TypeError(f"cannot pass {type(x)} as a device pointer")


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(status: int, what: str) -> None:
    if status != HS2_OK:
        raise HS2Error(status, what)


def dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return HS2_BF16
    if t == torch.float32:
        return HS2_F32
    raise ValueError(f"hs2 supports bf16 and fp32, not {t}")


def make_problem(B, Hq, Hkv, D, dtype, q_offsets, kv_offsets, total_q, total_kv,
                 max_q_len, max_kv_len, scale) -> Problem:
    """Fills an ``hs2_problem``; offsets are int64 device tensors of B+1 entries."""
    code = dtype if isinstance(dtype, int) else dtype_code(dtype)
    return Problem(int(B), int(Hq), int(Hkv), int(D), code, 0, _ptr(q_offsets),
                   _ptr(kv_offsets), int(total_q), int(total_kv), int(max_q_len),
                   int(max_kv_len), float(scale))


def _size(fn, *args) -> int:
    n = ctypes.c_size_t(0)
    _check(fn(*args, ctypes.byref(n)), fn.__name__)
    return int(n.value)


def _ws(workspace):
    if workspace is None:
        return None, 0
    if isinstance(workspace, torch.Tensor):
        return _ptr(workspace), workspace.numel() * workspace.element_size()
    addr, nbytes = workspace
    return int(addr), int(nbytes)


def hs2_full_attn_workspace_size(p: Problem) -> int:
    return _size(load().hs2_full_attn_workspace_size, ctypes.byref(p))


def hs2_full_attn_launches(p: Problem) -> int:
    n = ctypes.c_int32(0)
    _check(load().hs2_full_attn_launches(ctypes.byref(p), ctypes.byref(n)), "hs2_full_attn_launches")
    return int(n.value)


def hs2_full_attn_scores(p: Problem, Q, K, V, O, scores, score_stride, workspace, stream=None):
    w, n = _ws(workspace)
    _check(load().hs2_full_attn_scores(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(O),
                                       _ptr(scores), int(score_stride), w, n, _stream(stream)),
           "hs2_full_attn_scores")


def hs2_topk_workspace_size(p: Problem, k: int, window: int) -> int:
    return _size(load().hs2_topk_workspace_size, ctypes.byref(p), int(k), int(window))


def hs2_topk_select(p: Problem, scores, score_stride, k, window, idx, count, workspace,
                    stream=None):
    w, n = _ws(workspace)
    _check(load().hs2_topk_select(ctypes.byref(p), _ptr(scores), int(score_stride), int(k),
                                  int(window), _ptr(idx), _ptr(count), w, n, _stream(stream)),
           "hs2_topk_select")


def hs2_block_select_workspace_size(p: Problem, n_blocks: int, block: int, window: int) -> int:
    return _size(load().hs2_block_select_workspace_size, ctypes.byref(p), int(n_blocks),
                 int(block), int(window))


def hs2_block_select(p: Problem, scores, score_stride, n_blocks, block, window, idx, count,
                     workspace, stream=None):
    w, n = _ws(workspace)
    _check(load().hs2_block_select(ctypes.byref(p), _ptr(scores), int(score_stride),
                                   int(n_blocks), int(block), int(window), _ptr(idx),
                                   _ptr(count), w, n, _stream(stream)), "hs2_block_select")


# Fixed scratch behind hs2_block_select_noalloc (bytes).
NOALLOC_SCRATCH_BYTES = 16 << 20


def hs2_block_select_noalloc(p: Problem, scores, score_stride, n_blocks, block, window, idx,
                             count, stream=None):
    """hs2_block_select without a workspace, for callers that cannot provide
    device memory; the library's fixed 16 MiB scratch is shared by all calls
    on a device, so calls must not overlap on the GPU."""
    _check(load().hs2_block_select_noalloc(ctypes.byref(p), _ptr(scores), int(score_stride),
                                           int(n_blocks), int(block), int(window), _ptr(idx),
                                           _ptr(count), _stream(stream)),
           "hs2_block_select_noalloc")


def hs2_sparse_attn_workspace_size(p: Problem, idx_stride: int) -> int:
    return _size(load().hs2_sparse_attn_workspace_size, ctypes.byref(p), int(idx_stride))


def hs2_sparse_attn(p: Problem, Q_l, K, V, idx, count, idx_stride, O_l, workspace, stream=None):
    w, n = _ws(workspace)
    _check(load().hs2_sparse_attn(ctypes.byref(p), _ptr(Q_l), _ptr(K), _ptr(V), _ptr(idx),
                                  _ptr(count), int(idx_stride), _ptr(O_l), w, n,
                                  _stream(stream)), "hs2_sparse_attn")


def hs2_kv_append(p: Problem, K_new, V_new, K, V, stream=None):
    """Writes the new tokens' K/V rows into the cache at their own positions."""
    _check(load().hs2_kv_append(ctypes.byref(p), _ptr(K_new), _ptr(V_new), _ptr(K), _ptr(V),
                                _stream(stream)), "hs2_kv_append")


def hs2_swa_attn(p: Problem, Q, K, V, window, O, stream=None):
    """Sliding-window attention over positions max(0, t-window+1) .. t."""
    _check(load().hs2_swa_attn(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), int(window), _ptr(O),
                               _stream(stream)), "hs2_swa_attn")


def hs2_kv_bridge(p: Problem, H, hidden, Wk_t, Wv_t, K, V, stream=None):
    """K = H Wk, V = H Wv into the cache layout (Wk_t, Wv_t: [Hkv*D, hidden])."""
    _check(load().hs2_kv_bridge(ctypes.byref(p), _ptr(H), int(hidden), _ptr(Wk_t), _ptr(Wv_t),
                                _ptr(K), _ptr(V), _stream(stream)), "hs2_kv_bridge")


def hs2_wait_selftest(mode: int, limit_cycles: int, stream=None):
    """Queues a bounded wait that nothing ends; it records HS2_ERR_TIMEOUT."""
    _check(load().hs2_wait_selftest(int(mode), int(limit_cycles), _stream(stream)),
           "hs2_wait_selftest")


def hs2_cp_attn_partial(p: Problem, Q, K, V, O_part, ml_part, workspace, stream=None):
    ws, n = _ws(workspace)
    _check(load().hs2_cp_attn_partial(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(O_part),
                                      _ptr(ml_part), ws, n, _stream(stream)), "hs2_cp_attn_partial")


def hs2_cp_merge(rows: int, R: int, O_parts, ml_parts, dtype, O, ml=None, stream=None):
    code = dtype if isinstance(dtype, int) else dtype_code(dtype)
    _check(load().hs2_cp_merge(int(rows), int(R), _ptr(O_parts), _ptr(ml_parts), code, _ptr(O),
                               _ptr(ml), _stream(stream)), "hs2_cp_merge")


def hs2_cp_scores(p: Problem, ml, scores, score_stride, workspace, stream=None):
    ws, n = _ws(workspace)
    _check(load().hs2_cp_scores(ctypes.byref(p), _ptr(ml), _ptr(scores), int(score_stride), ws, n,
                                _stream(stream)), "hs2_cp_scores")


def hs2_cp_topk_local(p: Problem, scores, score_stride, k, window, pos0, idx_tmp, count_tmp,
                      pair_score, pair_pos, stream=None):
    _check(load().hs2_cp_topk_local(ctypes.byref(p), _ptr(scores), int(score_stride), int(k),
                                    int(window), _ptr(pos0), _ptr(idx_tmp), _ptr(count_tmp),
                                    _ptr(pair_score), _ptr(pair_pos), _stream(stream)),
           "hs2_cp_topk_local")


def hs2_cp_topk_merge(p: Problem, R, k, window, pair_score, pair_pos, idx, count, stream=None):
    _check(load().hs2_cp_topk_merge(ctypes.byref(p), int(R), int(k), int(window), _ptr(pair_score),
                                    _ptr(pair_pos), _ptr(idx), _ptr(count), _stream(stream)),
           "hs2_cp_topk_merge")


def hs2_cp_sparse_partial(p: Problem, Q_l, K, V, idx, count, idx_stride, pos0, O_part, ml_part,
                          stream=None):
    _check(load().hs2_cp_sparse_partial(ctypes.byref(p), _ptr(Q_l), _ptr(K), _ptr(V), _ptr(idx),
                                        _ptr(count), int(idx_stride), _ptr(pos0), _ptr(O_part),
                                        _ptr(ml_part), _stream(stream)), "hs2_cp_sparse_partial")


def hs2_get_last_device_error(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device error word."""
    return int(load().hs2_get_last_device_error(_stream(stream)))


def hs2_version() -> int:
    return int(load().hs2_version())
