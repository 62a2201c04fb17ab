#!/usr/bin/env python
"""Throughput of one HySparse2 hybrid-block decode step on B200.

A step is one pass of the whole path over one batch: the full-attention
layer over the shared KV cache with per-key selection scores, token-level
top-1024 + 128-window selection, and 4 sparse-attention layers that reuse the
cache and the indices.  Workload per GPU (weak scaling, independent sequences,
no collective on the data path): 8 decode sequences x 131072 cached tokens,
32 query / 4 KV heads, head dim 128, bf16, synthetic N(0,1) inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 is launched with torch.distributed.run (one process per GPU, NCCL only
for the barrier and the max-over-ranks timing).  Rank 0 prints one JSON line.
``--impl reference`` times the CPU oracle (float64, the host cores) on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "query-tok/s & KV-scan HBM GB/s (vs ~8 TB/s), select+sparse attn, 128K–1M ctx"
UNIT = "query-tok/s"
BATCH, CONTEXT, HQ, HKV, D, LAYERS, TOPK, WINDOW = 8, 131072, 32, 4, 128, 4, 1024, 128
WORKLOAD = "decode_b8_128k_bf16"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-subrecords", action="store_true",
                    help="skip the needle 1M, chunk 262K and ragged 16 records of the default run")
    ap.add_argument("--batch", type=int, default=BATCH,
                    help="sequences per GPU (smaller only for profiling captures)")
    ap.add_argument("--context", type=int, default=CONTEXT,
                    help="cached tokens per sequence (smaller only for profiling captures)")
    ap.add_argument("--workload", default="decode_b8_128k",
                    choices=["decode_b8_128k", "needle_1m", "ragged_16", "chunk_256k",
                             "multiblock_4x_decode_b8_128k", "hybrid_swa_decode_b8_128k",
                             "kv_bridge_262k", "cp8_needle_1m"],
                    help="other shapes of the pages' workloads (one GPU); the default is the "
                         "benchmark line")
    return ap.parse_args()


def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def rank_first_sequence(rank: int, batch: int) -> int:
    """Weak scaling: rank r owns global sequences [r * batch, (r + 1) * batch)."""
    return rank * batch


def max_over_ranks(x: float, world: int, device) -> float:
    """The slowest rank's value (device timings are combined by max)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(batch: int, world: int, steps: int, elapsed_ms: float) -> float:
    """Whole-job query tokens per second: every rank's queries over the slowest rank's time."""
    return batch * world * steps / (elapsed_ms / 1e3)


# ---------------------------------------------------------------------------
# workload accounting
# ---------------------------------------------------------------------------
def workload_accounting(w, n_layers: int, count=TOPK + WINDOW):
    """Algorithmic bytes and flops of one step of a synthetic workload: K/V
    read once, Q read and O written, every visible score written once and read
    once by the selection, and the selected rows gathered once per layer."""
    e = 2 if w.dtype == "bf16" else 4
    tpos = w.query_positions()
    visible = int((tpos + 1).sum())
    rows_sel = int(np.minimum(tpos + 1, count).sum())  # selected rows per KV group
    kv = 2 * int(w.kv_lens.sum()) * w.Hkv * w.D * e
    q = int(w.q_lens.sum()) * w.Hq * w.D * e
    scores = visible * w.Hkv * 4
    full = kv + 2 * q + scores
    select = scores + int(w.q_lens.sum()) * w.Hkv * (count + 1) * 4
    sparse = rows_sel * w.Hkv * w.D * e * 2 + 2 * q
    flops = 4 * w.D * w.Hq * visible
    return dict(full=full, select=select, sparse_layer=sparse, step=full + select + n_layers * sparse,
                kv=kv, flops=flops, queries=int(w.q_lens.sum()))


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    """Sustained bf16 tensor throughput (TFLOP/s) for a kernel timed inside a long step."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops_sustained"]), "measured sustained"
    except Exception:
        return 1400.0, "fallback sustained"


def profiled_traffic(kernel_src_hash: str):
    """DRAM bytes per launch of the full-attention call from the committed ncu
    summary, or None if it was taken on different kernel sources."""
    path = os.path.join(ROOT, "profiles", "full_attn_decode_b8_128k.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m = re.search(r"traffic_bytes_per_call:\s*([0-9.eE+]+)", text)
    h = re.search(r"kernel_sources_sha256:\s*([0-9a-f]+)", text)
    if not m or not h or h.group(1) != kernel_src_hash:
        return None
    return float(m.group(1))


# the sources of the kernels of the decode full-attention call (their traffic
# is what the committed summary records)
DECODE_SOURCES = ("common.cuh", "ptx.cuh", "decode_attn.cuh")


def kernel_sources_hash() -> str:
    csrc = os.path.join(ROOT, "long_context_full_b200", "csrc")
    h = hashlib.sha256()
    for f in DECODE_SOURCES:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML sampler thread)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, index: int, period: float = 0.02):
        self.samples, self.reasons = [], 0
        self.ok = False
        self.max_mhz = None
        self.period = period
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
        self._stop = threading.Event()
        self._t = None

    def _sample(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        try:
            self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            self.reasons |= nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if not self.ok:
            return None
        self._stop.set()
        self._t.join()
        self._sample()
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": float(self.max_mhz),
                "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# CPU oracle on a bounded sample (the baseline leg and the reference arm)
# ---------------------------------------------------------------------------
def oracle_unit(w, r: int, g: int, n_keys: int | None = None):
    """The oracle's full step for one (query row, KV group): full attention of
    the group's heads over the first n_keys cached tokens (all by default),
    scores, top-k select, and every sparse layer."""
    import oracle
    import synth
    b = int(w.query_seq()[r])
    ko = w.kv_offsets
    n = int(w.kv_lens[b]) if n_keys is None else n_keys
    G = w.Hq // w.Hkv
    ks = synth.stored_to_f64(w.k[ko[b]:ko[b] + n, g:g + 1], w.dtype)
    vs = synth.stored_to_f64(w.v[ko[b]:ko[b] + n, g:g + 1], w.dtype)
    q = synth.stored_to_f64(w.q[r, g * G:(g + 1) * G], w.dtype)
    t = n - 1
    O, m, l, P = oracle.full_attention_row(q, ks, vs, t, w.scale)
    s = oracle.selection_scores(P, 1)
    idx, c = oracle.topk_select(s[0], t, w.topk, w.window)
    for layer in range(w.n_layers):
        ql = synth.stored_to_f64(w.q_layers[layer][r, g * G:(g + 1) * G], w.dtype)
        oracle.sparse_attention_row(ql, ks, vs, [idx[:c]], w.scale)


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


def cpu_baseline(w, budget_s: float = 12.0):
    """Oracle throughput in query-tok/s on whole (query, KV group) units, the
    batch's units in turn (again from the first when all are done) until
    ``budget_s`` of CPU time has been spent (at least one unit)."""
    n = w.q.shape[0] * w.Hkv
    units, t0 = 0, time.perf_counter()
    while True:
        r, g = divmod(units % n, w.Hkv)
        oracle_unit(w, r, g)
        units += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": (units / w.Hkv) / dt, "unit": UNIT, "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"{units} (query, KV-group) units, the batch's {n} in turn: full attention "
                      f"of the group's {w.Hq // w.Hkv} heads over {int(w.kv_lens[0])} keys, scores, top-k "
                      f"select, {w.n_layers} sparse layers; float64 numpy, {dt:.1f} s"}


def run_reference(args, rank, world):
    """--impl reference: the CPU oracle as it stands, on a bounded sample of
    this workload; rank 0 only."""
    if rank != 0:
        return
    import synth
    w = synth.decode_128k(batch=1)
    # sample size per step: one (query, KV group) unit over the first n_keys
    # cached tokens, shrunk so that all steps fit in about two minutes
    t0 = time.perf_counter()
    oracle_unit(w, 0, 0)
    unit_s = time.perf_counter() - t0
    steps = args.steps + args.warmup
    n_keys = CONTEXT
    if steps * unit_s > 120.0:
        n_keys = max(4096, int(CONTEXT * 120.0 / (steps * unit_s)))
    for _ in range(args.warmup):
        oracle_unit(w, 0, 0, n_keys)
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle_unit(w, 0, i % HKV, n_keys)
    dt = (time.perf_counter() - t0) / max(1, args.steps)
    # throughput of the sample scaled to whole queries over the full context
    value = (1.0 / HKV) * (n_keys / CONTEXT) / dt
    sample = (f"one (query, KV group) unit per step: full attention of 8 heads over the first "
              f"{n_keys} of {CONTEXT} keys, scores, top-k select, {LAYERS} sparse layers; "
              f"value scaled by (1/{HKV}) x ({n_keys}/{CONTEXT}) per step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "batch_per_gpu": BATCH, "context": CONTEXT,
                       "Hq": HQ, "Hkv": HKV, "D": D, "k": TOPK, "window": WINDOW,
                       "reuse_layers": LAYERS},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------
def time_steps(step, Q, K, V, QL, n_steps: int, local: int, barrier=lambda: None):
    """Times exactly ``n_steps`` hybrid-block steps on the current stream with
    CUDA events around the whole region only (the kernels of consecutive calls
    overlap their launches; an event between them would serialise that), then
    ``n_steps`` more with events around each phase (full attention, selection,
    the sparse layers) for the breakdown.  Returns (elapsed ms of the first
    region, per-step phase ms [n_steps, 3], clock record of the first region)."""
    import torch
    stream = torch.cuda.current_stream()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    start.record(stream)
    for _ in range(n_steps):
        step.run(Q, K, V, QL)
    end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_steps)]
    for i in range(n_steps):
        e = ev[i]
        e[0].record(stream)
        step.full_attention(Q, K, V)
        e[1].record(stream)
        step.select_tokens()
        e[2].record(stream)
        for layer in range(step.n_layers):
            step.sparse_layer(layer, QL[layer], K, V)
        e[3].record(stream)
    torch.cuda.synchronize()
    ph = np.array([[e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2]), e[2].elapsed_time(e[3])]
                   for e in ev])
    return start.elapsed_time(end), ph, clk


def time_calls(fn, n: int) -> float:
    """Mean ms of ``n`` back-to-back calls of ``fn`` between two CUDA events on
    the current stream (consecutive launches overlap as they do inside a step;
    no event between the calls)."""
    import torch
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(n):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / n


def load_workload(w, select: str = "token"):
    """Device copies of a synthetic bf16 workload and a HybridBlockStep for it."""
    import torch
    from long_context_full_b200.block import HybridBlockStep

    def dev(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()

    Q, K, V = dev(w.q), dev(w.k), dev(w.v)
    QL = [dev(x) for x in w.q_layers]
    step = HybridBlockStep(w.Hq, w.Hkv, w.D, torch.bfloat16, w.q_lens, w.kv_lens, w.n_layers,
                           k=TOPK, window=WINDOW, select=select)
    return step, Q, K, V, QL


def warm(step, Q, K, V, QL, n: int):
    """``n`` untimed steps (at least 3), then a check of the device error word."""
    import torch
    from long_context_full_b200 import hs2
    for _ in range(max(3, n)):
        step.run(Q, K, V, QL)
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK


def needle_recall(w, idx, count):
    """Needle recall per KV group of the GPU's index sets (idx / count of the
    decode row) beside that of the oracle's own selection on its own scores."""
    import oracle
    import synth
    G = w.Hq // w.Hkv
    n = int(w.kv_lens[0])
    t = n - 1
    needles = set(w.needle_pos[0].tolist())
    gpu, ora = [], []
    for g in range(w.Hkv):
        ks = synth.stored_to_f64(w.k[:n, g:g + 1], w.dtype)
        vs = synth.stored_to_f64(w.v[:n, g:g + 1], w.dtype)
        q = synth.stored_to_f64(w.q[0, g * G:(g + 1) * G], w.dtype)
        _, _, _, P = oracle.full_attention_row(q, ks, vs, t, w.scale)
        s = oracle.selection_scores(P, 1)[0]
        oi, oc = oracle.topk_select(s, t, w.topk, w.window)
        ora.append(len(needles & set(oi[:oc].tolist())) / len(needles))
        gpu.append(len(needles & set(idx[g, :int(count[g])].tolist())) / len(needles))
    return gpu, ora


def subrecord(w, args, local, hbm, select_compare: bool = False, recall: bool = False):
    """One more of the pages' workload shapes, timed like the headline (same
    steps and warm-up, its own clock record): ms per step, phase times and its
    roofline figures."""
    import torch
    from long_context_full_b200 import hs2
    step, Q, K, V, QL = load_workload(w)
    warm(step, Q, K, V, QL, args.warmup)
    el, ph, clk = time_steps(step, Q, K, V, QL, args.steps, local)
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
    ms = el / args.steps
    t_full, t_sel, t_sp = (float(x) for x in ph.mean(axis=0))
    t_call = time_calls(lambda: step.full_attention(Q, K, V), args.steps)  # back to back
    ab = workload_accounting(w, w.n_layers)
    rec = {"workload": w.name, "query_tokens": ab["queries"], "context": int(w.kv_lens.max()),
           "ms_per_step": ms, "query_tok_s": ab["queries"] / (ms * 1e-3),
           "phase_ms": {"full_attn_scores": t_full, "topk_select": t_sel,
                        f"sparse_attn_x{w.n_layers}": t_sp},
           "full_attn_ms_per_call": t_call,
           "clocks": clk}
    if int(w.q_lens.max()) > 1:
        tf, tf_kind = tensor_peak()
        achieved = ab["flops"] / (t_call * 1e-3) / 1e12
        rec["full_attn_tflops"] = achieved
        rec["full_attn_frac_of_tensor_peak"] = achieved / tf
        rec["tensor_peak"] = {"value": tf, "unit": "TFLOP/s", "kind": tf_kind}
        rec["score_write_gbs"] = (ab["full"] - ab["kv"]) / (t_call * 1e-3) / 1e9
    else:
        step_gbs = ab["step"] / (ms * 1e-3) / 1e9
        rec["algorithmic_bytes_per_step"] = ab["step"]
        rec["step_gbs"] = step_gbs
        rec["step_frac_of_hbm"] = step_gbs / hbm
        rec["step_frac_of_8TBps"] = step_gbs / 8000.0
        rec["full_attn_gbs"] = ab["full"] / (t_call * 1e-3) / 1e9
        rec["full_attn_frac_of_hbm"] = rec["full_attn_gbs"] / hbm
        ss = ab["select"] + w.n_layers * ab["sparse_layer"]
        rec["select_sparse_gbs"] = ss / ((t_sel + t_sp) * 1e-3) / 1e9
    if recall:
        gpu, ora = needle_recall(w, step.idx.cpu().numpy(), step.count.cpu().numpy())
        rec["needle_recall"] = {"gpu": gpu, "oracle": ora,
                                "note": "per KV group; parity means equal index sets, not recall 1"}
    if select_compare:
        del step
        bstep, Q, K, V, QL = load_workload(w, select="block")
        warm(bstep, Q, K, V, QL, args.warmup)
        bel, bph, bclk = time_steps(bstep, Q, K, V, QL, args.steps, local)
        assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
        rec["block_select_path"] = {
            "ms_per_step": bel / args.steps,
            "phase_ms": {"full_attn_scores": float(bph[:, 0].mean()),
                         "block_select": float(bph[:, 1].mean()),
                         f"sparse_attn_x{w.n_layers}": float(bph[:, 2].mean())},
            "clocks": bclk}
    torch.cuda.synchronize()
    return rec


def run_multiblock(args, local: int, n_blocks: int = 4):
    """A decode step through ``n_blocks`` Hybrid Blocks, each with its own
    8 x 131072-token cache (8 GiB of K/V in all), replayed as one CUDA graph:
    per block, the new token's K/V appended, full attention with scores, top-k
    selection and 4 sparse layers.  Throughput = the 8 query tokens of the step
    / step time.  End to end: the step's inputs (queries of every layer and the
    new K/V rows of every block) copied from pinned host memory and the last
    sparse layer's output of every block read back; the caches stay resident."""
    import torch
    import synth
    from long_context_full_b200 import hs2
    from long_context_full_b200.multiblock import BlockInputs, MultiBlockDecodeStep

    ws = [synth.decode_128k(batch=BATCH, first_seq=BATCH * i, context=CONTEXT) for i in range(n_blocks)]
    rng = np.random.default_rng(2026)
    news = [(synth.f32_to_bf16_bits(rng.standard_normal((BATCH, HKV, D)).astype(np.float32)),
             synth.f32_to_bf16_bits(rng.standard_normal((BATCH, HKV, D)).astype(np.float32)))
            for _ in range(n_blocks)]
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).pin_memory()
    ins = [BlockInputs(dev(w.k), dev(w.v), dev(kn), dev(vn), dev(w.q), [dev(x) for x in w.q_layers])
           for w, (kn, vn) in zip(ws, news)]
    w0 = ws[0]
    mb = MultiBlockDecodeStep(n_blocks, w0.Hq, w0.Hkv, w0.D, torch.bfloat16, w0.q_lens, w0.kv_lens,
                              w0.n_layers, k=TOPK, window=WINDOW)
    outs = mb.capture(ins)
    for _ in range(max(3, args.warmup)):
        mb.replay()
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
    stream = torch.cuda.current_stream()
    Kst = args.steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    torch.cuda.synchronize()
    clocks.start()
    start.record(stream)
    for _ in range(Kst):
        mb.replay()
    end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
    ms_step = start.elapsed_time(end) / Kst
    value = BATCH / (ms_step * 1e-3)
    ab = workload_accounting(w0, w0.n_layers)
    append_bytes = 2 * 2 * BATCH * HKV * D * 2  # new rows read and written, K and V
    step_bytes = n_blocks * (ab["step"] + append_bytes)
    hbm, hbm_kind = peaks()
    achieved = step_bytes / (ms_step * 1e-3) / 1e9

    # end to end: inputs from pinned host memory, outputs back, graph replay between
    hin = [(pin(w.q), [pin(x) for x in w.q_layers], pin(kn), pin(vn)) for w, (kn, vn) in zip(ws, news)]
    dpairs = []
    for x, (hq, hql, hkn, hvn) in zip(ins, hin):
        dpairs += [(x.Q, hq), (x.K_new, hkn), (x.V_new, hvn)] + list(zip(x.Q_layers, hql))
    douts = [o.O_layers[-1] for o in outs]
    houts = [torch.empty_like(o, device="cpu").pin_memory() for o in douts]
    h2d = sum(h.numel() * h.element_size() for _, h in dpairs)
    d2h = sum(h.numel() * h.element_size() for h in houts)

    def e2e_step():
        for d_, h_ in dpairs:
            d_.copy_(h_, non_blocking=True)
        mb.replay()
        for h_, d_ in zip(houts, douts):
            h_.copy_(d_, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    E = max(1, min(args.e2e_steps, Kst))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(E):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_value = BATCH * E / (e0.elapsed_time(e1) * 1e-3)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": Kst,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) Q/K/V, Philox streams)",
        "config": {"workload": f"multiblock_{n_blocks}x_decode_b8_128k_bf16 (CUDA graph)",
                   "blocks": n_blocks, "query_tokens_per_gpu": BATCH, "context": CONTEXT,
                   "Hq": HQ, "Hkv": HKV, "D": D, "k": TOPK, "window": WINDOW,
                   "reuse_layers": w0.n_layers,
                   "l2": f"inputs larger than L2: {n_blocks * ab['kv'] / 2**30:.2f} GiB of K/V per step",
                   "parallelism": "dp1"},
        "roofline": {"kernel": "whole step (all blocks)", "bound": "hbm", "achieved": achieved,
                     "peak": hbm, "unit": "GB/s", "frac": achieved / hbm, "peak_kind": hbm_kind,
                     "traffic": None, "algorithmic_bytes": step_bytes},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": E},
        "gpu_launches": Kst * mb.launches_per_step(),
        "clocks": clk,
        "cpu_baseline": None,
    }
    print(json.dumps(line), flush=True)


SWA_WINDOW = 128  # the pages give no window for the Hybrid SWA baseline: declared


def run_hybrid_swa(args, local: int):
    """The Hybrid SWA baseline's block on the benchmark workload, timed at the
    kernel level beside the Hybrid Block: the same full-attention call (with
    its scores) followed by 4 sliding-window layers (window SWA_WINDOW) instead
    of the selection and 4 sparse layers.  Per step: 8 query tokens."""
    import torch
    import synth
    from long_context_full_b200 import hs2
    from long_context_full_b200.block import HybridBlockStep

    w = synth.decode_128k(batch=BATCH, first_seq=0, context=CONTEXT)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    Q, K, V = dev(w.q), dev(w.k), dev(w.v)
    QL = [dev(x) for x in w.q_layers]
    step = HybridBlockStep(w.Hq, w.Hkv, w.D, torch.bfloat16, w.q_lens, w.kv_lens, w.n_layers,
                           k=TOPK, window=WINDOW)
    OL = [torch.empty_like(Q) for _ in range(w.n_layers)]

    def swa_layers():
        for l in range(w.n_layers):
            hs2.hs2_swa_attn(step.problem, QL[l], K, V, SWA_WINDOW, OL[l])

    for _ in range(max(3, args.warmup)):
        step.full_attention(Q, K, V)
        swa_layers()
        step.select_tokens()
        for l in range(w.n_layers):
            step.sparse_layer(l, QL[l], K, V)
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
    stream = torch.cuda.current_stream()
    Kst = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(Kst)]
    clocks = ClockSampler(local)
    torch.cuda.synchronize()
    clocks.start()
    for i in range(Kst):
        e = ev[i]
        e[0].record(stream)
        step.full_attention(Q, K, V)
        e[1].record(stream)
        swa_layers()
        e[2].record(stream)
        step.select_tokens()
        e[3].record(stream)
        for l in range(w.n_layers):
            step.sparse_layer(l, QL[l], K, V)
        e[4].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
    ph = np.array([[e[j].elapsed_time(e[j + 1]) for j in range(4)] for e in ev]).mean(axis=0)
    t_full, t_swa, t_sel, t_sp = (float(x) for x in ph)
    ms_step = t_full + t_swa  # the Hybrid SWA block: full attention + its SWA layers
    value = BATCH / (ms_step * 1e-3)
    ab = workload_accounting(w, w.n_layers)
    hbm, hbm_kind = peaks()
    swa_bytes = w.n_layers * (2 * BATCH * HKV * min(SWA_WINDOW, CONTEXT) * D * 2 + 2 * BATCH * HQ * D * 2)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": Kst,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) Q/K/V, Philox streams)",
        "config": {"workload": f"hybrid_swa_decode_b8_128k_bf16 (window {SWA_WINDOW}, comparison)",
                   "query_tokens_per_gpu": BATCH, "context": CONTEXT, "Hq": HQ, "Hkv": HKV, "D": D,
                   "swa_window": SWA_WINDOW, "swa_layers": w.n_layers,
                   "l2": f"inputs larger than L2: {ab['kv'] / 2**30:.2f} GiB of K/V per step",
                   "parallelism": "dp1"},
        "phase_ms": {"full_attn_scores": t_full, "swa_x4": t_swa,
                     "hybrid_block_select": t_sel, "hybrid_block_sparse_x4": t_sp},
        "hybrid_block_ms_per_step": t_full + t_sel + t_sp,
        "roofline": {"kernel": "hs2_swa_attn x4 (window rows gathered)", "bound": "hbm",
                     "achieved": swa_bytes / (t_swa * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
                     "frac": swa_bytes / (t_swa * 1e-3) / 1e9 / hbm, "peak_kind": hbm_kind,
                     "traffic": None, "algorithmic_bytes": swa_bytes},
        "gpu_launches": Kst * (3 + w.n_layers),
        "clocks": clk,
        "cpu_baseline": None,
    }
    print(json.dumps(line), flush=True)


CP_RANKS = 8


def run_cp_rank(args, local: int):
    """Context-parallel decode of the 1M-token needle workload split by position
    into CP_RANKS equal ranges: all ranks run on this GPU in turn for warm-up
    (and to fill the exchanged partials), then one rank's own work per step -
    its full-attention partial, the merges, its scores and local top-k, the
    merged selection and the 4 sparse partials with their merges - is timed.
    The all-gathers between the phases are not timed (one GPU here); their
    size per rank and step is reported."""
    import torch
    import synth
    from long_context_full_b200 import hs2
    from long_context_full_b200.context_parallel import (ContextParallelDecodeStep, LocalRanks,
                                                         shard_offsets)

    w = synth.needle_1m()
    R, N = CP_RANKS, int(w.kv_lens[0])
    lens = [[N // R + (1 if r < N % R else 0)] for r in range(R)]
    pos0 = shard_offsets(lens)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    Ks = [dev(w.k[pos0[r][0]:pos0[r][0] + lens[r][0]]) for r in range(R)]
    Vs = [dev(w.v[pos0[r][0]:pos0[r][0] + lens[r][0]]) for r in range(R)]
    Q = dev(w.q)
    QL = [dev(x) for x in w.q_layers]
    steps = [ContextParallelDecodeStep(r, R, w.Hq, w.Hkv, w.D, torch.bfloat16, lens, w.n_layers,
                                       k=TOPK, window=WINDOW, scale=w.scale) for r in range(R)]
    ranks = LocalRanks(steps)
    for _ in range(max(3, args.warmup)):
        ranks.run(Q, Ks, Vs, QL)
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
    O_parts = torch.stack([st.O_part for st in steps])
    ml_parts = torch.stack([st.ml_part for st in steps])
    ps = torch.stack([st.pair_score for st in steps])
    pp = torch.stack([st.pair_pos for st in steps])
    st = steps[0]
    stream = torch.cuda.current_stream()
    Kst = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(Kst)]
    clocks = ClockSampler(local)
    torch.cuda.synchronize()
    clocks.start()
    for i in range(Kst):
        e = ev[i]
        e[0].record(stream)
        st.attention_partial(Q, Ks[0], Vs[0])
        e[1].record(stream)
        st.attention_merge(O_parts, ml_parts)
        e[2].record(stream)
        st.local_selection()
        e[3].record(stream)
        st.selection_merge(ps, pp)
        e[4].record(stream)
        for l in range(w.n_layers):
            st.sparse_partial(QL[l], Ks[0], Vs[0])
            st.sparse_merge(l, O_parts, ml_parts)
        e[5].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
    ph = np.array([[e[j].elapsed_time(e[j + 1]) for j in range(5)] for e in ev]).mean(axis=0)
    t_attn, t_merge, t_lsel, t_smerge, t_sparse = (float(x) for x in ph)
    ms_step = float(ph.sum())
    B = int(w.q_lens.sum())
    kv_bytes = 2 * lens[0][0] * w.Hkv * w.D * 2
    hbm, hbm_kind = peaks()
    exch = 4 * B * w.Hq * (w.D + 2) * (2 + w.n_layers) + 8 * B * w.Hkv * (TOPK + WINDOW)
    line = {
        "metric": METRIC, "value": B / (ms_step * 1e-3), "unit": UNIT, "n_gpus": 1, "steps": Kst,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) Q/K/V with 64 needles, Philox streams)",
        "config": {"workload": f"cp{R}_needle_b1_1m_bf16 (rank 0 of {R} context-parallel ranks; "
                               f"all ranks run on this one GPU, the all-gathers are not timed)",
                   "query_tokens": B, "context": N, "keys_per_rank": lens[0][0], "Hq": w.Hq,
                   "Hkv": w.Hkv, "D": w.D, "k": TOPK, "window": WINDOW, "reuse_layers": w.n_layers,
                   "l2": f"inputs larger than L2: {kv_bytes / 2**20:.0f} MiB of K/V per rank-step",
                   "parallelism": f"cp{R} (emulated)"},
        "phase_ms": {"attn_partial": t_attn, "attn_merge": t_merge, "scores_and_local_topk": t_lsel,
                     "topk_merge": t_smerge, "sparse_partial_and_merge_x4": t_sparse},
        "exchange_bytes_per_rank_step": exch,
        "roofline": {"kernel": "hs2_cp_attn_partial (decode pass + combine on the rank's keys)",
                     "bound": "hbm", "achieved": kv_bytes / (t_attn * 1e-3) / 1e9, "peak": hbm,
                     "unit": "GB/s", "frac": kv_bytes / (t_attn * 1e-3) / 1e9 / hbm,
                     "peak_kind": hbm_kind, "traffic": None, "algorithmic_bytes": kv_bytes},
        "gpu_launches": Kst * (2 + 1 + 3 + 1 + 2 * w.n_layers),
        "clocks": clk,
        "cpu_baseline": None,
    }
    print(json.dumps(line), flush=True)


BRIDGE_HIDDEN = 4096  # the pages give no hidden size: declared


def run_kv_bridge(args, local: int):
    """KV Bridging GEMM: K and V of 264,192 cache rows (the chunk workload's
    cache) from hidden states of width BRIDGE_HIDDEN, Hkv = 4, D = 128.
    Tensor-bound: 2 * rows * hidden * 2 * Hkv * D flops per call."""
    import torch
    from long_context_full_b200 import hs2

    rows, hidden, ncols = 264192, BRIDGE_HIDDEN, HKV * D
    g = torch.Generator(device="cuda")
    g.manual_seed(1250)
    H = torch.randn(rows, hidden, device="cuda", generator=g).to(torch.bfloat16)
    Wk = (torch.randn(ncols, hidden, device="cuda", generator=g) / math.sqrt(hidden)).to(torch.bfloat16)
    Wv = (torch.randn(ncols, hidden, device="cuda", generator=g) / math.sqrt(hidden)).to(torch.bfloat16)
    K = torch.empty(rows, HKV, D, dtype=torch.bfloat16, device="cuda")
    V = torch.empty_like(K)
    ko = torch.tensor([0, rows], dtype=torch.int64, device="cuda")
    qo = torch.tensor([0, 0], dtype=torch.int64, device="cuda")
    p = hs2.make_problem(1, HQ, HKV, D, hs2.HS2_BF16, qo, ko, 0, rows, 0, rows, 0.088)
    for _ in range(max(3, args.warmup)):
        hs2.hs2_kv_bridge(p, H, hidden, Wk, Wv, K, V)
    torch.cuda.synchronize()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
    stream = torch.cuda.current_stream()
    Kst = args.steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    torch.cuda.synchronize()
    clocks.start()
    start.record(stream)
    for _ in range(Kst):
        hs2.hs2_kv_bridge(p, H, hidden, Wk, Wv, K, V)
    end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
    ms = start.elapsed_time(end) / Kst
    flops = 2.0 * rows * hidden * 2 * ncols
    tf, tf_kind = tensor_peak()
    achieved = flops / (ms * 1e-3) / 1e12
    line = {
        "metric": "KV Bridging: cache rows built per second (K and V projections)",
        "value": rows / (ms * 1e-3), "unit": "cache-tok/s", "n_gpus": 1, "steps": Kst,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) hidden states and weights)",
        "config": {"workload": f"kv_bridge_262k (hidden {hidden}, declared)", "rows": rows,
                   "hidden": hidden, "Hkv": HKV, "D": D, "parallelism": "dp1",
                   "l2": f"inputs larger than L2: {rows * hidden * 2 / 2**30:.2f} GiB of hidden states"},
        "roofline": {"kernel": "k_kv_bridge<256>", "bound": "tensor", "achieved": achieved,
                     "peak": tf, "unit": "TFLOP/s", "frac": achieved / tf, "peak_kind": tf_kind,
                     "traffic": None, "algorithmic_flops": flops},
        "gpu_launches": Kst,
        "clocks": clk,
        "cpu_baseline": None,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank, world, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import torch.distributed as dist
    import synth
    from long_context_full_b200 import hs2

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    hs2.load()
    if args.workload == "multiblock_4x_decode_b8_128k":
        if world > 1:
            raise SystemExit("--workload other than the default runs on one GPU")
        return run_multiblock(args, local)
    if args.workload == "kv_bridge_262k":
        if world > 1:
            raise SystemExit("--workload other than the default runs on one GPU")
        return run_kv_bridge(args, local)
    if args.workload == "hybrid_swa_decode_b8_128k":
        if world > 1:
            raise SystemExit("--workload other than the default runs on one GPU")
        return run_hybrid_swa(args, local)
    if args.workload == "cp8_needle_1m":
        if world > 1:
            raise SystemExit("--workload other than the default runs on one GPU")
        return run_cp_rank(args, local)

    batch, context = args.batch, args.context
    if args.workload == "decode_b8_128k":
        w = synth.decode_128k(batch=batch, first_seq=rank_first_sequence(rank, batch),
                              context=context)
        workload = WORKLOAD if (batch, context) == (BATCH, CONTEXT) else \
            f"decode_b{batch}_{context}_bf16 (profiling case)"
    else:
        if world > 1:
            raise SystemExit("--workload other than the default runs on one GPU")
        if args.workload == "chunk_256k" and context != CONTEXT:
            w = synth.chunk_256k(cached=context)  # smaller cache: profiling captures only
            workload = f"chunk_{context}_plus_2k_bf16 (profiling case)"
        else:
            w = {"needle_1m": synth.needle_1m, "ragged_16": synth.ragged_16,
                 "chunk_256k": synth.chunk_256k}[args.workload]()
            workload = w.name
    batch = int(w.q_lens.sum())  # query tokens per step
    step, Q, K, V, QL = load_workload(w)
    n_layers = w.n_layers
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()

    # ---- warm-up, then the device-timed region: exactly K steps, events per phase
    warm(step, Q, K, V, QL, args.warmup)
    Kst = args.steps
    elapsed_ms, ph, clk = time_steps(step, Q, K, V, QL, Kst, local, barrier)
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
    elapsed_ms = max_over_ranks(elapsed_ms, world, "cuda")
    ms_step = elapsed_ms / Kst
    value = job_throughput(batch, world, Kst, elapsed_ms)
    launches = step.launches_per_step()

    ab = workload_accounting(w, n_layers)
    t_full = float(ph[:, 0].mean())
    t_sel = float(ph[:, 1].mean())
    t_sp = float(ph[:, 2].mean())
    # the dominant call on its own: Kst calls back to back (the phase times
    # above carry the cost of an event between phases)
    t_call = time_calls(lambda: step.full_attention(Q, K, V), Kst)
    assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
    hbm, hbm_kind = peaks()
    chunk = int(w.q_lens.max()) > 1
    if chunk:  # dense QK^T / PV: the tensor pipe bounds the full-attention call
        tf, tf_kind = tensor_peak()
        achieved = ab["flops"] / (t_call * 1e-3) / 1e12
        roof = {"kernel": "hs2_full_attn_scores (chunk: attention pass + score pass)",
                "bound": "tensor", "achieved": achieved, "peak": tf, "unit": "TFLOP/s",
                "frac": achieved / tf, "peak_kind": tf_kind, "traffic": None,
                "algorithmic_flops": ab["flops"]}
    else:
        achieved = ab["full"] / (t_call * 1e-3) / 1e9
        traffic = profiled_traffic(kernel_sources_hash()) if workload == WORKLOAD else None
        roof = {"kernel": "hs2_full_attn_scores (decode pass + O merge and score finalize: 2 kernels)",
                "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                "frac": achieved / hbm, "peak_kind": hbm_kind,
                "traffic": traffic, "algorithmic_bytes": ab["full"],
                "frac_of_8TBps": achieved / 8000.0,
                "ms_per_call": t_call, "calls_timed": Kst,
                "frac_from_phase_events": ab["full"] / (t_full * 1e-3) / 1e9 / hbm}

    # ---- end to end through the public API with host buffers
    pin = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory()
    hQ, hK, hV = pin(w.q), pin(w.k), pin(w.v)
    hQL = [pin(x) for x in w.q_layers]
    outs = [step.O] + step.O_layers + [step.idx, step.count]
    hout = [torch.empty_like(o, device="cpu").pin_memory() for o in outs]
    h2d = sum(t.numel() * t.element_size() for t in [hQ, hK, hV] + hQL)
    d2h = sum(t.numel() * t.element_size() for t in hout)

    def e2e_step():
        for d_, h_ in zip([Q, K, V] + QL, [hQ, hK, hV] + hQL):
            d_.copy_(h_, non_blocking=True)
        step.run(Q, K, V, QL)
        for h_, d_ in zip(hout, outs):
            h_.copy_(d_, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    E = max(1, min(args.e2e_steps, Kst))
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(E):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, "cuda")
    e2e_value = job_throughput(batch, world, E, e2e_ms)

    # ---- end to end with the cache resident (a decode server's case): per step
    # the queries of every layer and each new token's K/V row come from pinned
    # host memory, the rows are appended with hs2_kv_append (the same bytes at
    # the same positions, so the cache does not change), the step runs, and
    # its outputs are read back
    e2e_res = None
    if int(w.q_lens.max()) == 1:
        last = w.kv_offsets[1:] - 1
        hKn, hVn = pin(np.ascontiguousarray(w.k[last])), pin(np.ascontiguousarray(w.v[last]))
        Kn, Vn = torch.empty_like(hKn, device="cuda"), torch.empty_like(hVn, device="cuda")
        h2d_res = sum(t.numel() * t.element_size() for t in [hQ, hKn, hVn] + hQL)

        def e2e_resident_step():
            for d_, h_ in zip([Q, Kn, Vn] + QL, [hQ, hKn, hVn] + hQL):
                d_.copy_(h_, non_blocking=True)
            hs2.hs2_kv_append(step.problem, Kn, Vn, K, V)
            step.run(Q, K, V, QL)
            for h_, d_ in zip(hout, outs):
                h_.copy_(d_, non_blocking=True)

        e2e_resident_step()
        torch.cuda.synchronize()
        barrier()
        e0.record(stream)
        for _ in range(E):
            e2e_resident_step()
        e1.record(stream)
        torch.cuda.synchronize()
        assert hs2.hs2_get_last_device_error() == hs2.HS2_OK
        res_ms = max_over_ranks(e0.elapsed_time(e1), world, "cuda")
        e2e_res = {"value": job_throughput(batch, world, E, res_ms), "unit": UNIT,
                   "h2d_bytes_per_step": h2d_res, "d2h_bytes_per_step": d2h, "steps": E,
                   "note": "K/V cache resident; the new tokens' K/V rows appended each step"}

    # ---- the other workloads of the metric's range, one GPU, default run only
    subs = None
    if (world == 1 and args.workload == "decode_b8_128k" and workload == WORKLOAD
            and not args.no_subrecords):
        del hK, hV
        step = None
        Q = K = V = None
        QL = []
        torch.cuda.empty_cache()
        subs = {}
        subs["needle_1m"] = subrecord(synth.needle_1m(), args, local, hbm, recall=True)
        torch.cuda.empty_cache()
        subs["chunk_262k"] = subrecord(synth.chunk_256k(), args, local, hbm)
        torch.cuda.empty_cache()
        subs["ragged_16"] = subrecord(synth.ragged_16(), args, local, hbm, select_compare=True)
        torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.workload == "decode_b8_128k":
        cpu = cpu_baseline(w)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": Kst,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) Q/K/V, Philox streams)",
            "config": {"workload": workload, "query_tokens_per_gpu": batch,
                       "context": int(w.kv_lens.max()), "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D,
                       "k": TOPK, "window": WINDOW, "reuse_layers": n_layers,
                       "l2": f"inputs larger than L2: {ab['kv'] / 2**30:.2f} GiB of K/V streamed per step",
                       "parallelism": f"dp{world} (independent sequences per GPU)"},
            "kv_scan_gbs": ab["kv"] / (t_call * 1e-3) / 1e9,
            "step_gbs": ab["step"] / (ms_step * 1e-3) / 1e9,
            "step_frac_of_hbm": ab["step"] / (ms_step * 1e-3) / 1e9 / hbm,
            "phase_ms": {"full_attn_scores": t_full, "topk_select": t_sel,
                         f"sparse_attn_x{n_layers}": t_sp},
            "roofline": roof,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": E},
            "gpu_launches": Kst * launches,
            "clocks": clk,
        }
        if e2e_res is not None:
            line["e2e_resident_cache"] = e2e_res
        if subs is not None:
            line["workloads"] = subs
        if cpu is not None:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
