"""Throughput of the exact-attention hot path on B200, one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python -m torch.distributed.run --nproc-per-node N ... bench.py --gpus N ...

A step is one pass of the whole prefill hot path over the workload "prefill B8 H16 N2048 d128"
(bf16 Q/K/V i.i.d. N(0,1), seeded): one non-causal and one causal fa_fwd launch (tile scheduler,
TMA loads, Q K^T, mask, online softmax, rescale, P V and epilogue all run inside them).
`value` is attention TFLOP/s (4 B H N^2 d per non-causal pass, half that causal) over all ranks;
the L2 is flushed (a 256 MiB write) before every timed step and the flush is outside the timed
events.  With N ranks each rank runs the same independent (b, h) workload (weak scaling; heads are
independent, so there is no collective on the data path).

Extra keys: `roofline` (prefill kernel vs the measured dense bf16 peak), `cpu_baseline` (the fp64
oracle on this host's cores, a bounded row sample), `e2e` (the same metric through the Python API
with Q/K/V copied from pinned host memory and O/LSE copied back inside the timed region), `sweep`
(the sequence-length grid, d = 128 and d = 64), `decode` (paged decode GB/s vs HBM),
`paged_prefill` (chunked prefill through the block table, TFLOP/s), `backward` (fa_bwd TFLOP/s),
`tree` (draft-tree verification TFLOP/s), `sequence_parallel` (one long sequence with its keys
split over ranks: partials, all-gather, merge) and `clocks`.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "attention fwd TFLOP/s (and % of B200 dense BF16 peak) vs seqlen; decode GB/s"
UNIT = "TFLOP/s"
WORKLOAD = "prefill B8 H16 N2048 d128, causal + non-causal"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "source": "fallback"}
KERNEL_SOURCES = ["exact_attention_158_b200/csrc/fa_prefill.cuh",
                  "exact_attention_158_b200/csrc/sm100_ptx.cuh"]
DECODE_SOURCES = ["exact_attention_158_b200/csrc/fa_decode.cuh",
                  "exact_attention_158_b200/csrc/sm100_ptx.cuh"]


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        p["source"] = "measured"
        return p
    return dict(FALLBACK_PEAKS)


def source_hash(paths) -> str:
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def committed_traffic(name: str, paths):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken on this source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f).get(name)
    if not t or t.get("source_hash") != source_hash(paths):
        return None
    return t.get("bytes_per_launch")


# ---------------------------------------------------------------------------------------------
# clocks during the timed region (NVML reads only)
# ---------------------------------------------------------------------------------------------
class ClockSampler:
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.001):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # no NVML: report no clocks rather than guess
            self._nv = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                r = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._nv is not None:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._nv is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ---------------------------------------------------------------------------------------------
# timing helpers
# ---------------------------------------------------------------------------------------------
class Flusher:
    def __init__(self, device):
        self.buf = torch.empty(256 << 20, dtype=torch.uint8, device=device)

    def __call__(self):
        self.buf.fill_(1)


def time_launches(fn, steps, warmup, flush, stream):
    """Run fn() warmup times, then `steps` times with an L2 flush before each; returns the list of
    per-step device times (ms) from CUDA events recorded on `stream`."""
    for _ in range(warmup):
        flush()
        fn()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for a, b in evs:
        flush()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def dist_max(x: float) -> float:
    """Max over ranks (every rank calls it at the same point; identity without a process group)."""
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        return float(t.item())
    return x


def aggregate(step_ms_local: float, flops_per_rank_step: float, world: int):
    """Whole-job throughput: every rank runs the same independent workload (weak scaling), so the
    job does world * flops per step in the slowest rank's step time.  Returns (TFLOP/s, max ms)."""
    step_ms = dist_max(step_ms_local)
    return world * flops_per_rank_step / (step_ms * 1e-3) / 1e12, step_ms


def barrier():
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.barrier()


# ---------------------------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on this host's cores, bounded sample of rows
# ---------------------------------------------------------------------------------------------
_CPU_INPUTS = None


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _oracle_rows_rate(qb, kb, vb, threads, target_s, rng, BH, N, d):
    """Time the oracle over random (head, row) samples, half causal; returns (TFLOP/s, rows, s)."""
    from oracle import oracle as orc
    flops = 0.0
    rows = 0
    t0 = time.perf_counter()
    batch = max(64, threads * 16)
    while time.perf_counter() - t0 < target_s:
        for causal in (False, True):
            pairs = np.stack([rng.integers(0, BH, batch), rng.integers(0, N, batch)], 1)
            orc.attention_rows(qb, kb, vb, causal, 1 / math.sqrt(d), pairs, threads)
            # exact FLOPs of these rows: 4 d per visible key
            vis = (pairs[:, 1] + 1) if causal else np.full(batch, N)
            flops += float(4.0 * d * vis.sum())
            rows += batch
    el = time.perf_counter() - t0
    return flops / el / 1e12, rows, el


def cpu_baseline(target_s: float = 12.0, one_thread_s: float = 3.0):
    """The fp64 oracle on this host: all its threads over a bounded row sample of the headline
    workload (the reported value), plus a 1-thread figure on the same kind of sample."""
    from oracle import oracle as orc
    global _CPU_INPUTS
    BH, N, d = 8 * 16, 2048, 128
    if _CPU_INPUTS is None:
        q, k, v = W.make_prefill(W.prefill_cases()[0], device="cpu")
        _CPU_INPUTS = tuple(W.bf16_bits(t).reshape(BH, N, d) for t in (q, k, v))
    qb, kb, vb = _CPU_INPUTS
    threads = orc.default_threads()
    rng = np.random.default_rng(0)
    value, rows, el = _oracle_rows_rate(qb, kb, vb, threads, target_s, rng, BH, N, d)
    out = {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
           "sample": f"{rows} query rows of {WORKLOAD} (half causal), fp64, {el:.1f} s; "
                     "throughput scaled by the exact FLOPs of the sampled rows",
           "cpu_model": cpu_model(), "nproc": os.cpu_count()}
    if one_thread_s > 0:
        v1, rows1, el1 = _oracle_rows_rate(qb, kb, vb, 1, one_thread_s, rng, BH, N, d)
        out["value_1thread"] = v1
        out["sample_1thread"] = f"{rows1} query rows, 1 thread, {el1:.1f} s"
    return out


def cpu_sweep_point(case, target_s: float = 0.25):
    """The oracle (all host threads) on sampled rows of two (b, h) slices of one sweep point, its
    time extrapolated to the whole point by the exact FLOPs of the sampled rows."""
    from oracle import oracle as orc
    heads = [0, case.B * case.H - 1]
    q, k, v = (W.bf16_bits(t) for t in W.make_prefill_heads(case, heads))
    threads = orc.default_threads()
    rng = np.random.default_rng(1)
    flops, rows, t0 = 0.0, 0, time.perf_counter()
    batch = max(32, threads * 4)
    while time.perf_counter() - t0 < target_s:
        pairs = np.stack([rng.integers(0, 2, batch), rng.integers(0, case.N, batch)], 1)
        orc.attention_rows(q, k, v, case.causal, case.scale, pairs, threads)
        vis = (pairs[:, 1] + 1) if case.causal else np.full(batch, case.N)
        flops += float(4.0 * case.d * vis.sum())
        rows += batch
    el = time.perf_counter() - t0
    tf = flops / el / 1e12
    return {"tflops": tf, "ms_extrapolated": case.flops / (tf * 1e12) * 1e3, "rows": rows,
            "cores": threads, "extrapolated": True}


# ---------------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------------
def run_prefill_case(fa, case, steps, warmup, flush, stream, out_dtype=torch.bfloat16):
    q, k, v = W.make_prefill(case, device="cuda")
    o = torch.empty_like(q) if out_dtype == torch.bfloat16 else torch.empty(q.shape, dtype=out_dtype, device="cuda")
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    fn = lambda: fa.fa_fwd(q, k, v, causal=case.causal, scale=case.scale, out=o, lse=lse,
                           out_dtype=out_dtype)
    ts = time_launches(fn, steps, warmup, flush, stream)
    if fa.device_status() != 0:
        raise RuntimeError("device status set during the bench")
    return ts


def bench_decode(fa, args, dev, flush, stream, pk):
    case = W.DecodeCase("decode", S=args.decode_seqs)
    inp = W.make_decode(case, device=dev)
    o = torch.empty_like(inp["q"])
    lse = torch.empty(inp["q"].shape[:2], dtype=torch.float32, device=dev)
    ws = torch.empty(fa.fa_decode_workspace_size(case.S, case.H, case.d, inp["max_blocks"]),
                     dtype=torch.uint8, device=dev)
    fn = lambda: fa.fa_decode_paged(inp["q"], inp["k_pool"], inp["v_pool"], inp["block_table"],
                                    inp["seq_lens"], scale=case.scale, out=o, lse=lse,
                                    workspace=ws)
    torch.cuda.nvtx.range_push("bench_decode_timed")
    ts = time_launches(fn, args.sweep_steps, 3, flush, stream)
    torch.cuda.nvtx.range_pop()
    if fa.device_status() != 0:
        raise RuntimeError("device status set during the decode bench")
    ms = statistics.median(ts)
    nbytes = W.decode_bytes(inp["lens"], case.H, case.d, inp["max_blocks"])
    gbs = nbytes / (ms * 1e-3) / 1e9
    # the decode only reads: its denominator is the read-only bandwidth measured here with the
    # same streaming loads over a 4 GiB buffer (best of five), besides the copy figure
    tokens = sum(inp["lens"])
    del inp, o, lse, ws
    torch.cuda.empty_cache()
    rbuf = torch.empty(4 << 30, dtype=torch.uint8, device=dev)
    fa.probe_read_rate(rbuf)
    read_gbs = max(rbuf.numel() / (fa.probe_read_rate(rbuf) * 1e-3) / 1e9 for _ in range(5))
    _MEASURED["read_gbs"] = read_gbs
    del rbuf
    torch.cuda.empty_cache()
    return {"metric": "paged decode GB/s", "workload": f"{case.S} seqs, q len 1, H32 d128, "
            "context U[512,8192], 16-token pages, permuted block table",
            "ms": round(ms, 4), "value": round(gbs, 1), "unit": "GB/s",
            "algorithmic_bytes": nbytes, "tokens": tokens,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": round(read_gbs, 1),
                         "unit": "GB/s", "frac": round(gbs / read_gbs, 4),
                         "peak_source": "read-only bandwidth measured in this run "
                                        "(fa_probe_read_rate, 4 GiB, best of 5)",
                         "frac_of_copy_peak": round(gbs / pk["hbm_gbs"], 4),
                         "copy_peak": pk["hbm_gbs"],
                         "frac_of_nominal_7700": round(gbs / 7700.0, 4),
                         "traffic": committed_traffic("decode", DECODE_SOURCES)},
            "launches_per_step": 2}


# figures measured earlier in the same run that later rows reuse (the read-only bandwidth)
_MEASURED = {}


def bench_paged_prefill(fa, args, dev, flush, stream, pk):
    case = W.DecodeCase("paged_prefill", S=16, H=32, d=128, len_lo=2048, len_hi=8192)
    Lq = 512
    inp = W.make_paged_prefill(case, Lq, device=dev)
    o = torch.empty_like(inp["q"])
    lse = torch.empty(inp["q"].shape[:3], dtype=torch.float32, device=dev)
    fn = lambda: fa.fa_prefill_paged(inp["q"], inp["k_pool"], inp["v_pool"], inp["block_table"],
                                     inp["seq_lens"], causal=True, scale=case.scale, out=o,
                                     lse=lse)
    torch.cuda.nvtx.range_push("bench_paged_prefill_timed")
    ts = time_launches(fn, args.sweep_steps, 3, flush, stream)
    torch.cuda.nvtx.range_pop()
    if fa.device_status() != 0:
        raise RuntimeError("device status set during the paged prefill bench")
    ms = statistics.median(ts)
    flops = W.paged_prefill_flops(inp["lens"], case.H, case.d, Lq, True)
    tf = flops / (ms * 1e-3) / 1e12
    return {"metric": "chunked prefill over a paged cache, TFLOP/s",
            "workload": f"{case.S} seqs, chunk {Lq}, H32 d128, context U[2048,8192], "
            "16-token pages, permuted block table, causal (bottom-right)",
            "ms": round(ms, 4), "value": round(tf, 1), "unit": "TFLOP/s",
            "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": pk["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": round(tf / pk["bf16_tflops"], 4)},
            "launches_per_step": 1}


def bench_tree(fa, args, dev, flush, stream, pk):
    """Draft-tree verification: 32 sequences, 64-node seeded random trees after contexts of
    U[2048, 8192] tokens, H32 d128, one fa_tree_attention launch per step."""
    T = 64
    case = W.DecodeCase("tree_verify", S=32, H=32, d=128, len_lo=2048 + T, len_hi=8192 + T)
    inp = W.make_tree_verify(case, T, "random", device=dev)
    o = torch.empty_like(inp["q"])
    lse = torch.empty(inp["q"].shape[:3], dtype=torch.float32, device=dev)
    fn = lambda: fa.fa_tree_attention(inp["q"], inp["k_pool"], inp["v_pool"], inp["block_table"],
                                      inp["seq_lens"], inp["tree_mask"], scale=case.scale, out=o,
                                      lse=lse)
    torch.cuda.nvtx.range_push("bench_tree_timed")
    ts = time_launches(fn, args.sweep_steps, 3, flush, stream)
    torch.cuda.nvtx.range_pop()
    if fa.device_status() != 0:
        raise RuntimeError("device status set during the tree bench")
    ms = statistics.median(ts)
    masks = [W.tree_visibility(p) for p in inp["parents"]]
    flops = W.tree_verify_flops(inp["lens"], masks, case.H, case.d)
    nbytes = W.tree_verify_bytes(inp["lens"], case.H, case.d, T)
    tf = flops / (ms * 1e-3) / 1e12
    gbs = nbytes / (ms * 1e-3) / 1e9
    # 64 queries per (sequence, head) against every cached key: about 64 FLOP per byte of K/V,
    # below the ridge point (measured peak FLOP/s over measured bandwidth), so HBM bounds it
    return {"metric": "draft-tree verification over a paged cache, TFLOP/s",
            "workload": "32 seqs, 64-node random draft trees, context U[2048,8192], H32 d128, "
            "16-token pages, permuted block table",
            "ms": round(ms, 4), "value": round(tf, 2), "unit": "TFLOP/s",
            "algorithmic_bytes": nbytes, "flop_per_byte": round(flops / nbytes, 1),
            "roofline": dict({"bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm_gbs"],
                              "unit": "GB/s", "frac": round(gbs / pk["hbm_gbs"], 4),
                              "peak_source": "measured copy bandwidth"},
                             **({"frac_of_read_peak": round(gbs / _MEASURED["read_gbs"], 4),
                                 "read_peak": round(_MEASURED["read_gbs"], 1)}
                                if "read_gbs" in _MEASURED else {})),
            "launches_per_step": 1}


def bench_sequence_parallel(fa, args, dev, flush, stream, pk, rank, world):
    """One long causal sequence, B1 H16 N32768 d128, with its keys split into contiguous ranges.
    With N GPUs each rank holds one range: partial of every query over it (fa_fwd_keyrange), an
    NCCL all-gather of the partials, and the merge (fa_merge_partials) on every rank.  On one GPU
    the four ranges of a 4-way split run one after another before the same merge."""
    from exact_attention_158_b200 import sequence_parallel as sp
    case = W.PrefillCase("seqpar", 1, 16, 32768, 128, True)
    q, k, v = W.make_prefill(case, device=dev)
    G = world if world > 1 else 4
    ranges = sp.key_ranges(case.N, G)
    mine = [ranges[rank]] if world > 1 else ranges
    shards = [(a, k[:, :, a:b].contiguous(), v[:, :, a:b].contiguous()) for a, b in mine]
    del k, v
    o_all = torch.empty((G, *q.shape), dtype=torch.float32, device=dev)
    l_all = torch.empty((G, *q.shape[:3]), dtype=torch.float32, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    lib = fa.load_library()
    st = stream.cuda_stream

    def merge():
        rc = lib.fa_merge_partials(o_all.data_ptr(), l_all.data_ptr(), G, lse.numel(), case.d,
                                   o.data_ptr(), 0, lse.data_ptr(), st)
        if rc != 0:
            raise RuntimeError(f"fa_merge_partials: {rc}")

    def step():
        if world > 1:
            a, ks, vs = shards[0]
            fa.fa_fwd_keyrange(q, ks, vs, k_pos0=a, causal=True, out=o_all[rank], lse=l_all[rank])
            # in place: this rank's slice of the gathered buffer is its input
            torch.distributed.all_gather_into_tensor(o_all, o_all[rank])
            torch.distributed.all_gather_into_tensor(l_all, l_all[rank])
        else:
            for r, (a, ks, vs) in enumerate(shards):
                fa.fa_fwd_keyrange(q, ks, vs, k_pos0=a, causal=True, out=o_all[r], lse=l_all[r])
        merge()

    torch.cuda.nvtx.range_push("bench_sequence_parallel_timed")
    ts = time_launches(step, args.sweep_steps, 3, flush, stream)
    merge_ts = time_launches(merge, args.sweep_steps, 3, flush, stream)
    torch.cuda.nvtx.range_pop()
    if fa.device_status() != 0:
        raise RuntimeError("device status set during the sequence-parallel bench")
    ms = dist_max(statistics.median(ts))
    mms = dist_max(statistics.median(merge_ts))
    tf = case.flops / (ms * 1e-3) / 1e12
    rows = lse.numel()
    merge_bytes = G * rows * (case.d + 1) * 4 + rows * case.d * 2 + rows * 4
    mgbs = merge_bytes / (mms * 1e-3) / 1e9
    return {"metric": "sequence-sharded causal forward TFLOP/s (whole sequence, all ranks)",
            "workload": "B1 H16 N32768 d128 causal, keys and values split into contiguous ranges",
            "ranges": G, "emulated_on_one_gpu": world == 1,
            "ms": round(ms, 4), "value": round(tf, 1), "unit": "TFLOP/s",
            "roofline": {"bound": "tensor", "achieved": round(tf, 1),
                         "peak": pk["bf16_tflops"] * (world if world > 1 else 1), "unit": "TFLOP/s",
                         "frac": round(tf / (pk["bf16_tflops"] * (world if world > 1 else 1)), 4)},
            "merge": {"ms": round(mms, 4), "algorithmic_bytes": merge_bytes,
                      "roofline": {"bound": "hbm", "achieved": round(mgbs, 1), "peak": pk["hbm_gbs"],
                                   "unit": "GB/s", "frac": round(mgbs / pk["hbm_gbs"], 4)}},
            "launches_per_step": (1 if world > 1 else G) + 1}


def bench_backward(fa, args, dev, flush, stream, pk):
    """fa_bwd on the headline shape (B8 H16 N2048 d128), non-causal and causal.  FLOPs are the five
    matmuls per (query, key) pair: 2.5x the forward's 4 B H N^2 d (halved causal)."""
    out = {}
    for causal in (False, True):
        case = W.PrefillCase("bwd", 8, 16, 2048, 128, causal)
        q, k, v = W.make_prefill(case, device=dev)
        do = W.make_dout(case, device=dev)
        o, lse = fa.fa_fwd(q, k, v, causal=causal, scale=case.scale)
        ws = torch.empty(fa.load_library().fa_bwd_workspace_size(case.B, case.H, case.N, case.d),
                         dtype=torch.uint8, device=dev)
        fn = lambda: fa.fa_bwd(q, k, v, o, do, lse, causal=causal, scale=case.scale, workspace=ws)
        torch.cuda.nvtx.range_push("bench_backward_timed")
        ts = time_launches(fn, args.sweep_steps, 3, flush, stream)
        torch.cuda.nvtx.range_pop()
        if fa.device_status() != 0:
            raise RuntimeError("device status set during the backward bench")
        ms = statistics.median(ts)
        tf = 2.5 * case.flops / (ms * 1e-3) / 1e12
        out["causal" if causal else "non_causal"] = {"ms": round(ms, 4), "tflops": round(tf, 1),
                                                     "frac": round(tf / pk["bf16_tflops"], 4)}
    tot_ms = out["causal"]["ms"] + out["non_causal"]["ms"]
    tot_tf = 2.5 * 1.5 * W.PrefillCase("bwd", 8, 16, 2048, 128, False).flops / (tot_ms * 1e-3) / 1e12
    return {"metric": "attention backward TFLOP/s (dQ, dK, dV; 2.5x forward FLOPs)",
            "workload": "B8 H16 N2048 d128, dO ~ N(0,1), O and LSE from fa_fwd, causal + non-causal",
            "value": round(tot_tf, 1), "unit": "TFLOP/s", "per_variant": out,
            "roofline": {"bound": "tensor", "achieved": round(tot_tf, 1), "peak": pk["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": round(tot_tf / pk["bf16_tflops"], 4)},
            "launches_per_step": 6}


def measure_ex2(fa, dev):
    """Exponentials per second on the special-function unit (best of three ~0.1 s probes), and
    per SM per clock at the SM clock sampled meanwhile."""
    fa.probe_ex2_rate(2000)
    with ClockSampler(dev.index) as clk:
        best = max(n / (ms * 1e-3) for n, ms in (fa.probe_ex2_rate(200_000) for _ in range(3)))
    c = clk.summary()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    mhz = c["sm_mhz"] or c["sm_max_mhz"]
    return {"exps_per_s": best, "sms": sms, "sm_mhz": mhz,
            "per_sm_per_clk": round(best / (sms * mhz * 1e6), 3) if mhz else None,
            "how": "fa_probe_ex2_rate: 4 CTAs x 256 threads per SM, 16 independent ex2 chains "
                   "per thread, CUDA events; one exponential per 4 d FLOP of the forward"}


def bench_ours(args, rank, world):
    import exact_attention_158_b200 as fa
    fa.load_library()
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    flush = Flusher(dev)
    pk = peaks()
    if args.only == "decode":
        return {"metric": METRIC, "decode": bench_decode(fa, args, dev, flush, stream, pk)}
    if args.only == "tree":
        return {"metric": METRIC, "tree": bench_tree(fa, args, dev, flush, stream, pk)}
    if args.only == "seqpar":
        return {"metric": METRIC,
                "sequence_parallel": bench_sequence_parallel(fa, args, dev, flush, stream, pk,
                                                             rank, world)}
    if args.only == "backward":
        return {"metric": METRIC, "backward": bench_backward(fa, args, dev, flush, stream, pk)}
    if args.only == "paged":
        return {"metric": METRIC,
                "paged_prefill": bench_paged_prefill(fa, args, dev, flush, stream, pk)}
    if args.only == "point":
        # one sweep point alone (for profiling): d, N and the mask from the command line
        case = next(c for c in W.sweep_cases(args.point_d)
                    if c.N == args.point_n and c.causal == bool(args.point_causal))
        ts = run_prefill_case(fa, case, args.steps, args.warmup, flush, stream)
        ms = statistics.median(ts)
        return {"metric": METRIC, "point": {"d": case.d, "N": case.N, "B": case.B, "H": case.H,
                                            "causal": case.causal, "ms": round(ms, 4),
                                            "tflops": round(case.flops / (ms * 1e-3) / 1e12, 1)}}

    # ---- headline: prefill config, non-causal + causal per step
    cases = W.prefill_cases()
    inputs = [W.make_prefill(c, device=dev) for c in cases]
    outs = [(torch.empty_like(q), torch.empty(q.shape[:3], dtype=torch.float32, device=dev))
            for q, _, _ in inputs]
    kernel_ms = {False: [], True: []}

    def step():
        for c, (q, k, v), (o, lse) in zip(cases, inputs, outs):
            fa.fa_fwd(q, k, v, causal=c.causal, scale=c.scale, out=o, lse=lse)

    for _ in range(args.warmup):
        flush()
        step()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in cases] for _ in range(args.steps)]
    torch.cuda.nvtx.range_push("bench_timed")
    with ClockSampler(dev.index) as clk:
        for st in range(args.steps):
            flush()
            for ci, (c, (q, k, v), (o, lse)) in enumerate(zip(cases, inputs, outs)):
                a, b = evs[st][ci]
                a.record(stream)
                fa.fa_fwd(q, k, v, causal=c.causal, scale=c.scale, out=o, lse=lse)
                b.record(stream)
        torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    barrier()
    torch.cuda.synchronize()
    if fa.device_status() != 0:
        raise RuntimeError("device status set during the timed region")
    for st in range(args.steps):
        for ci, c in enumerate(cases):
            kernel_ms[c.causal].append(evs[st][ci][0].elapsed_time(evs[st][ci][1]))
    step_ms = statistics.mean(kernel_ms[False]) + statistics.mean(kernel_ms[True])
    flops_step = sum(c.flops for c in cases)
    value, step_ms_max = aggregate(step_ms, flops_step, world)
    peak_key = "bf16_tflops"
    achieved = flops_step / (step_ms * 1e-3) / 1e12
    traffic = committed_traffic("prefill", KERNEL_SOURCES)
    roofline = {"bound": "tensor", "achieved": round(achieved, 1), "peak": pk[peak_key],
                "unit": "TFLOP/s", "frac": round(achieved / pk[peak_key], 4),
                "peak_source": f"{pk['source']} {peak_key} (burst: the kernel is timed alone)",
                "traffic": traffic,
                "per_variant": {
                    ("causal" if c else "non_causal"): {
                        "ms": round(statistics.mean(kernel_ms[c]), 4),
                        "tflops": round(cases[int(c)].flops / (statistics.mean(kernel_ms[c]) * 1e-3) / 1e12, 1)}
                    for c in (False, True)}}
    clocks = clk.summary()

    result = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms_max, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16, counter-based generator)",
        "config": {"workload": WORKLOAD, "B": 8, "H": 16, "N": 2048, "d": 128,
                   "causal": "both (one launch each per step)", "o_dtype": "bf16",
                   "parallelism": f"replicas x{world} (independent heads per GPU)",
                   "l2": "flushed (256 MiB write) before every timed step, outside the events"},
        "roofline": roofline, "gpu_launches": 2 * args.steps, "clocks": clocks,
    }
    if args.only == "prefill":
        return result

    # ---- e2e through the Python API with host buffers: both launches of a step read the same
    # Q, K, V (the two cases share one seed), so a step copies them to the device once (pinned
    # host -> device), runs the non-causal and the causal forward, and copies both outputs (O and
    # LSE) back to pinned host memory.  Steps are pipelined over three streams with two device
    # buffer sets: step t+1's inputs travel while step t computes and step t-1's outputs return
    # (PCIe carries both directions at once).  The inputs (201 MB) exceed L2, so no flush is
    # needed between steps; the time is the whole run's, divided by the step count.
    assert all(torch.equal(a, b) for a, b in zip(inputs[0], inputs[1]))
    host_in = [t.cpu().pin_memory() for t in inputs[0]]
    host_out = [(torch.empty(inputs[0][0].shape, dtype=torch.bfloat16).pin_memory(),
                 torch.empty(inputs[0][0].shape[:3], dtype=torch.float32).pin_memory()) for _ in cases]
    dev_in = [[torch.empty_like(t) for t in inputs[0]] for _ in range(2)]
    dev_out = [[(torch.empty_like(inputs[0][0]),
                 torch.empty(inputs[0][0].shape[:3], dtype=torch.float32, device=dev))
                for _ in cases] for _ in range(2)]
    del inputs, outs
    torch.cuda.empty_cache()
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for e in ev_comp + ev_out:
        e.record(stream)
    e2e_steps = max(4, min(args.steps, 20))

    def e2e_run(n_steps):
        for t in range(n_steps):
            b = t % 2
            s_in.wait_event(ev_comp[b])          # step t-2 has finished reading dev_in[b]
            with torch.cuda.stream(s_in):
                for h, d_ in zip(host_in, dev_in[b]):
                    d_.copy_(h, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_out[b])         # step t-2's outputs have left dev_out[b]
            q_, k_, v_ = dev_in[b]
            for c, (o_, l_) in zip(cases, dev_out[b]):
                fa.fa_fwd(q_, k_, v_, causal=c.causal, scale=c.scale, out=o_, lse=l_)
            ev_comp[b].record(stream)
            s_out.wait_event(ev_comp[b])
            with torch.cuda.stream(s_out):
                for (ho, hl), (o_, l_) in zip(host_out, dev_out[b]):
                    ho.copy_(o_, non_blocking=True)
                    hl.copy_(l_, non_blocking=True)
                ev_out[b].record(s_out)

    e2e_run(2)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    e2e_run(e2e_steps)
    s_out.wait_event(ev_comp[(e2e_steps - 1) % 2])
    t1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = dist_max(t0.elapsed_time(t1) / e2e_steps)
    if fa.device_status() != 0:
        raise RuntimeError("device status set during the e2e run")
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(o.numel() * o.element_size() + l.numel() * l.element_size() for o, l in host_out)
    e2e = {"value": round(world * flops_step / (e2e_ms * 1e-3) / 1e12, 2), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 3),
           "pipelined": "3 streams, 2 device buffer sets: copy-in, compute and copy-out of "
                        "consecutive steps overlap",
           "gpu_launches_per_step": 2}
    del host_in, host_out, dev_in, dev_out
    torch.cuda.empty_cache()

    # ---- sequence-length sweep (the pages' benchmark grid)
    # Ceilings per point: the dense bf16 peak, HBM (algorithmic bytes x measured bandwidth) and the
    # exponentials (one per 4 d FLOP, at the special-function unit's rate measured on this GPU by
    # fa_probe_ex2_rate, scaled to the SM clock sampled during the sweep).
    sweep, mufu = [], None
    if not args.no_sweep:
        mufu = measure_ex2(fa, dev)
        with ClockSampler(dev.index) as sclk:
            for d in (128, 64):
                for case in W.sweep_cases(d):
                    ts = run_prefill_case(fa, case, args.sweep_steps, 3, flush, stream)
                    sweep.append((case, statistics.median(ts)))
                    torch.cuda.empty_cache()
        sweep_mhz = sclk.summary()["sm_mhz"] or mufu["sm_mhz"]
        mufu["sweep_sm_mhz"] = sweep_mhz
        rows = []
        for case, ms in sweep:
            tf = case.flops / (ms * 1e-3) / 1e12
            intensity = case.flops / (4 * case.B * case.H * case.N * case.d * 2 + case.B * case.H * case.N * 4)
            hbm_ceiling = intensity * pk["hbm_gbs"] / 1e3
            if mufu["per_sm_per_clk"] and sweep_mhz:
                exps_s = mufu["per_sm_per_clk"] * mufu["sms"] * sweep_mhz * 1e6
            else:
                exps_s = mufu["exps_per_s"]
            mufu_ceiling = exps_s * 4 * case.d / 1e12
            attainable = min(pk["bf16_tflops"], hbm_ceiling, mufu_ceiling)
            row = {"d": case.d, "N": case.N, "B": case.B, "H": case.H, "causal": case.causal,
                   "ms": round(ms, 4), "tflops": round(tf, 1),
                   "frac_peak": round(tf / pk["bf16_tflops"], 4),
                   "mufu_ceiling_tflops": round(mufu_ceiling, 1),
                   "frac_mufu": round(tf / mufu_ceiling, 4),
                   "frac_attainable": round(tf / attainable, 4),
                   "bound_by": ("tensor" if attainable == pk["bf16_tflops"] else
                                "hbm" if attainable == hbm_ceiling else "mufu")}
            if not args.no_cpu_baseline and rank == 0:
                row["cpu_oracle"] = cpu_sweep_point(case)
            rows.append(row)
        sweep = rows

    # ---- paged decode (HBM bound)
    dec = None if args.no_decode else bench_decode(fa, args, dev, flush, stream, pk)

    # ---- chunked prefill over the paged cache (tensor bound)
    paged = None if args.no_paged else bench_paged_prefill(fa, args, dev, flush, stream, pk)

    # ---- backward (tensor bound)
    bwd = None if args.no_backward else bench_backward(fa, args, dev, flush, stream, pk)

    # ---- draft-tree verification (tensor bound, short query tiles)
    tree = None if args.no_tree else bench_tree(fa, args, dev, flush, stream, pk)

    # ---- sequence-sharded forward (partials + merge; ranks emulated on one GPU)
    seqpar = (None if args.no_seqpar else
              bench_sequence_parallel(fa, args, dev, flush, stream, pk, rank, world))

    result.update({"e2e": e2e, "sweep": sweep, "mufu": mufu, "decode": dec, "paged_prefill": paged,
                   "backward": bwd, "tree": tree, "sequence_parallel": seqpar})
    return result


# ---------------------------------------------------------------------------------------------
def bench_reference(args):
    """The oracle as it stands, on this host's cores, for the same metric and workload."""
    steps = []
    cb = None
    for _ in range(args.warmup):
        cpu_baseline(target_s=2.0)
    for _ in range(args.steps):
        cb = cpu_baseline(target_s=max(2.0, 20.0 / max(args.steps, 1)))
        steps.append(cb["value"])
    value = statistics.mean(steps)
    cb = dict(cb, value=value)
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "B": 8, "H": 16, "N": 2048, "d": 128},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--sweep-steps", type=int, default=20)
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-paged", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-tree", action="store_true")
    ap.add_argument("--no-seqpar", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--decode-seqs", type=int, default=64,
                    help="sequences in the decode workload (64 is the benchmark; fewer for profiling)")
    ap.add_argument("--point-d", type=int, default=64, help="--only point: head dim")
    ap.add_argument("--point-n", type=int, default=4096, help="--only point: sequence length")
    ap.add_argument("--point-causal", type=int, default=0, help="--only point: causal (0/1)")
    ap.add_argument("--only", choices=["all", "prefill", "decode", "paged", "backward", "tree",
                                       "seqpar", "point"],
                    default="all",
                    help="prefill: the headline loop alone; decode / paged: the paged decode or "
                    "chunked prefill loop alone")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(bench_reference(args)), flush=True)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    out = bench_ours(args, rank, world)
    if rank == 0 and world == 1 and args.only == "all" and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline()
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
