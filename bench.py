#!/usr/bin/env python
"""Benchmark of the SSA hot path on B200 through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config mha|tiny|mla|varlen] [--no-decode] [--no-prefill]
                    [--no-cpu-baseline] [--decode-extra N] [--decode-mtp Q]

One JSON line on rank 0.  A step is one SSA prefill call over the chosen
workload (default: B=1, H=32, L=32768, d=128, 1 sink + 7 local blocks of 128);
``value`` is useful TFLOP/s = 2 (d_qk + d_v) * (number of unmasked (i, j)
pairs) per step / device time, summed over ranks.  The same run also times the
paged decode workload (32 sequences, 128 heads, 576/512, random page table over
a ~20 GB pool) and reports it under ``decode`` in GB/s of algorithmic bytes,
and the same decode with 8 distinct selected pages per sequence on top of the
window under ``decode_selected`` (``--decode-extra``), and the decode with 2
query tokens per sequence under ``decode_mtp`` (``--decode-mtp``), and the decode
over an FP8 cache under ``decode_fp8`` (``--decode-fp8``).  The
prefill's backward pass on the same workload is timed under ``backward``, and
full-attention against SSA decode layers at 128K tokens of context under
``decode_context`` (``--decode-context``), and a full-attention against an SSA
prefill layer at 128K tokens under ``prefill_context`` (``--prefill-context``).

Under torchrun every rank runs its own replica of the workload (weak scaling,
no collective on the data path; NCCL only reduces the timing).
``--impl reference`` times the CPU oracle on a bounded sample of the same
workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "SSA prefill TFLOPS & tokens/s (frac of BF16 peak); decode GB/s (frac of HBM)"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_BYTES = 126 * 1024 * 1024


# ------------------------------------------------------------------ helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def window_pairs(L: int, blk=128, n_sink=1, n_local=7) -> int:
    """Number of (i, j) pairs the SSA mask keeps for one sequence of length L
    (closed form of the row count: min(i+1, blk*(n_sink+n_local-1) + i%blk + 1))."""
    i = np.arange(L, dtype=np.int64)
    return int(np.minimum(i + 1, blk * (n_sink + n_local - 1) + (i % blk) + 1).sum())


def row_pairs(i: np.ndarray, blk=128, n_sink=1, n_local=7) -> np.ndarray:
    i = np.asarray(i, dtype=np.int64)
    return np.minimum(i + 1, blk * (n_sink + n_local - 1) + (i % blk) + 1)


# Kernel sources each profiled kernel is built from: a committed traffic figure
# stays valid only while these files are unchanged.
KERNEL_SOURCES = {
    "ssa_prefill_kernel": ("prefill.cuh", "ptx.cuh", "schedule.cuh"),
    "ssa_decode_split_kernel": ("decode.cuh", "ptx.cuh", "schedule.cuh"),
    "ssa_decode_merge_kernel": ("decode.cuh", "ptx.cuh", "schedule.cuh"),
    "ssa_decode_long_kernel": ("decode_long.cuh", "decode.cuh", "ptx.cuh", "schedule.cuh"),
}


def code_only(src: str) -> str:
    """A source file without its comments, whitespace runs collapsed: an edit of
    comments alone leaves source_hash, and the traffic records keyed by it, as
    they were (the kernel sources hold no comment markers inside strings)."""
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return re.sub(r"\s+", " ", src).strip()


def source_hash(kernel: str) -> str:
    """Hash of the code (comments left out) of the files a kernel is built from."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_sparse_streaming_ssa_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update((name + "\n" + code_only(f.read())).encode())
    return h.hexdigest()[:12]


REST_S = 1.0


def rest():
    """Idle the GPU for REST_S seconds between two workloads' measurements, so
    that each starts as it would alone (the power limiter of a 1 kW part reacts
    to the last tens of ms of load; the pause is outside every timed region)."""
    import torch
    torch.cuda.synchronize()
    time.sleep(REST_S)


def traffic_lookup(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None
    cur = source_hash(kernel)
    for ln in lines:
        parts = ln.split()
        if len(parts) == 4 and not ln.startswith("#") and parts[0] == kernel and \
                parts[1] == workload and parts[2] == cur:
            return int(float(parts[3]))
    return None


class ClockSampler:
    """Polls SM clock and throttle reasons through NVML on a background thread
    while the timed region runs."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s=0.002):
        self.period = period_s
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# ------------------------------------------------------------ multi-rank

def max_over_ranks(ms: float) -> float:
    """Slowest rank's device time (every rank times its own replica; the job
    is done when the slowest one is).  Single process: the value itself."""
    import torch
    import torch.distributed as td
    if not (td.is_available() and td.is_initialized()):
        return ms
    dev = "cuda" if td.get_backend() == "nccl" else "cpu"
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    td.all_reduce(t, op=td.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, units_per_rank_step: float, steps: int, max_ms: float) -> float:
    """Whole-job rate: the units all ranks processed / the slowest rank's time."""
    return world * units_per_rank_step * steps / (max_ms * 1e-3)


# ---------------------------------------------------------------- prefill

def workload_name(config, seed=0, heads=None):
    """The prefill workload's description, as the detailed record gives it (no
    device work: the packed workload's lengths come from the seeded host draw)."""
    from block_sparse_streaming_ssa_b200 import synth
    if config == "varlen":
        sp = synth.VARLEN
        lengths = synth.varlen_lengths(seed, sp.n_seqs, sp.len_lo, sp.len_hi, sp.total_cap)
        return (f"ssa_prefill_varlen {sp.n_seqs} seqs (total {sum(lengths)} tokens) "
                f"H={sp.H} d_qk=d_v={sp.d_qk} bf16, 1 sink + 7 local blocks of 128")
    sp = {"tiny": synth.TINY, "mha": synth.MHA, "mla": synth.MLA}[config]
    H = heads or sp.H
    return (f"ssa_prefill_{sp.name} B={sp.B} H={H} L={sp.L} d_qk={sp.d_qk} "
            f"d_v={sp.d_v} bf16, 1 sink + 7 local blocks of 128")


def line_config(workload):
    """The JSON line's `config` for a prefill workload (both arms give the same)."""
    return {"workload": workload.replace(" bf16, 1 sink + 7 local blocks of 128", " 1+7x128"),
            "parallelism": "replicas", "l2": "inputs > L2"}


def make_prefill(config, device, seed, heads=None):
    """The prefill workload ``config``; ``heads`` (dense workloads only) keeps
    the shapes but takes that many heads, for profiler captures of a smaller
    case whose per-head work is the same."""
    import dataclasses
    from block_sparse_streaming_ssa_b200 import synth
    if config == "varlen":
        sp = synth.VARLEN
        lengths = synth.varlen_lengths(seed, sp.n_seqs, sp.len_lo, sp.len_hi, sp.total_cap)
        q, k, v, cu = synth.varlen_inputs(lengths, sp.H, sp.d_qk, sp.d_v, seed=seed, device=device)
        pairs = sp.H * sum(window_pairs(n) for n in lengths)
        desc = {"workload": workload_name(config, seed),
                "lengths": lengths, "H": sp.H, "d_qk": sp.d_qk, "d_v": sp.d_v}
        tokens = sum(lengths)
        return dict(spec=sp, q=q, k=k, v=v, cu=cu, max_len=max(lengths), pairs=pairs,
                    tokens=tokens, desc=desc, varlen=True)
    sp = {"tiny": synth.TINY, "mha": synth.MHA, "mla": synth.MLA}[config]
    if heads:
        sp = dataclasses.replace(sp, H=heads)
    q, k, v = synth.prefill_spec_inputs(sp, seed=seed, device=device)
    pairs = sp.B * sp.H * window_pairs(sp.L)
    desc = {"workload": workload_name(config, seed, heads),
            "B": sp.B, "H": sp.H, "L": sp.L, "d_qk": sp.d_qk, "d_v": sp.d_v}
    return dict(spec=sp, q=q, k=k, v=v, cu=None, pairs=pairs, tokens=sp.B * sp.L, desc=desc,
                varlen=False)


def prefill_call(w, q=None, k=None, v=None, o=None, lse=None):
    from block_sparse_streaming_ssa_b200.loza_ssa import (loza_ssa_prefill,
                                                          loza_ssa_prefill_varlen)
    q = w["q"] if q is None else q
    k = w["k"] if k is None else k
    v = w["v"] if v is None else v
    if w["varlen"]:
        return loza_ssa_prefill_varlen(q, k, v, w["cu"], w["max_len"], o=o, lse=lse,
                                       scale=w["spec"].scale)
    return loza_ssa_prefill(q, k, v, o=o, lse=lse, scale=w["spec"].scale)


def prefill_bytes(w) -> int:
    q, k, v = w["q"], w["k"], w["v"]
    out = v.numel() * 2 + (v.numel() // v.shape[-1]) * 4
    return q.numel() * 2 + k.numel() * 2 + v.numel() * 2 + out


def time_prefill(w, steps, warmup, dist):
    import torch
    o, lse = prefill_call(w)
    for _ in range(warmup):
        prefill_call(w, o=o, lse=lse)
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        t0.record()
        for i in range(steps):
            starts[i].record()
            prefill_call(w, o=o, lse=lse)
            ends[i].record()
        t1.record()
        torch.cuda.synchronize()
    if dist:
        torch.distributed.barrier()
    total_ms = t0.elapsed_time(t1)
    per = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    return total_ms, per, clk.summary()


def backward_bench(w, steps, warmup, peaks, world=1):
    """The prefill's backward (loza_ssa_prefill_bwd) on the same workload,
    with o and lse from the forward pass and a seeded random dO.  Useful FLOPs
    follow the usual attention-backward count: the five products dP = dO V^T
    (2 d_v per unmasked (i, j) pair), dV += P^T dO (2 d_v), dQ += dS K
    (2 d_qk), dK += dS^T Q (2 d_qk) and one recomputation of S = Q K^T
    (2 d_qk), i.e. 2.5x the forward when d_qk = d_v (the dK/dV kernel
    recomputes S and dP a second time; that work is not counted)."""
    import torch
    from block_sparse_streaming_ssa_b200.loza_ssa import (loza_ssa_prefill_bwd,
                                                          loza_ssa_prefill_varlen_bwd)
    sp = w["spec"]
    if (sp.d_qk, sp.d_v) not in ((64, 64), (128, 128), (192, 128)):
        return None
    o, lse = prefill_call(w)
    g = torch.Generator(device="cuda").manual_seed(4242)
    dout = torch.randn(w["v"].shape, generator=g, device="cuda").to(torch.bfloat16)

    def bwd(grads=()):
        if w["varlen"]:
            return loza_ssa_prefill_varlen_bwd(w["q"], w["k"], w["v"], o, lse, dout, w["cu"],
                                               w["max_len"], *grads, scale=sp.scale)
        return loza_ssa_prefill_bwd(w["q"], w["k"], w["v"], o, lse, dout, *grads,
                                    scale=sp.scale)

    grads = bwd()
    for _ in range(warmup):
        bwd(grads)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        bwd(grads)
    t1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1) / steps)
    flops = 2 * (3 * sp.d_qk + 2 * sp.d_v) * w["pairs"]
    tf = flops / (ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]
    return {"workload": w["desc"]["workload"] + ", backward (dQ, dK, dV)",
            "value": round(job_throughput(world, flops, 1, ms) / 1e12, 2), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 4), "useful_tflop_per_step": round(flops / 1e12, 4),
            "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": peak,
                         "unit": "TFLOP/s", "frac": round(tf / peak, 4), "traffic": None,
                         "peak_source": peaks["source"] + " (burst bf16 GEMM)",
                         "note": "whole call: D preprocess, dQ kernel, dK/dV kernel, sink reduce"
                                 + (" (and the packed-sequence prefix setup)" if w["varlen"] else "")},
            "gpu_launches": (5 if w["varlen"] else 4) * steps}


def e2e_prefill(w, steps):
    """Same metric through the public call with host buffers: for the dense
    workloads loza_ssa_prefill_host (pinned host q, k, v in, pinned host o,
    lse out, copies inside the call, overlapped over chunks of planes); for the
    packed workload pinned-host copies around loza_ssa_prefill_varlen."""
    import torch
    from block_sparse_streaming_ssa_b200.loza_ssa import (loza_ssa_prefill_host,
                                                          loza_ssa_prefill_host_workspace_size)
    hq, hk, hv = (t.cpu().pin_memory() for t in (w["q"], w["k"], w["v"]))
    o, lse = prefill_call(w)
    ho, hl = o.cpu().pin_memory(), lse.cpu().pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    d2h = ho.numel() * ho.element_size() + hl.numel() * hl.element_size()
    if not w["varlen"]:
        sp = w["spec"]
        ws = torch.empty(loza_ssa_prefill_host_workspace_size(sp.B, sp.H, sp.L, sp.d_qk, sp.d_v),
                         dtype=torch.uint8, device="cuda")
        del o, lse
        torch.cuda.empty_cache()

        def step():
            loza_ssa_prefill_host(hq, hk, hv, o=ho, lse=hl, scale=sp.scale, workspace=ws)
    else:
        dq, dk, dv = (torch.empty_like(t) for t in (w["q"], w["k"], w["v"]))

        def step():
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            prefill_call(w, dq, dk, dv, o=o, lse=lse)
            ho.copy_(o, non_blocking=True)
            hl.copy_(lse, non_blocking=True)
    step()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        step()
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    return ms, h2d, d2h


# ----------------------------------------------------------------- decode

def decode_extra_pages(lens, n_extra, seed, n_sink=1, n_local=7, blk=128):
    """Per sequence, ``n_extra`` distinct logical pages drawn uniformly from the
    pages between the sink and the local run (fewer when there are not that
    many); -1 pads.  Returns the [B, n_extra] int32 list and the keys it adds."""
    rng = np.random.default_rng(2000 + seed)
    ex = np.full((len(lens), n_extra), -1, np.int32)
    added = 0
    for b, n in enumerate(lens):
        qb = (n - 1) // blk
        lo = max(n_sink, qb - n_local + 1)
        pool = np.arange(n_sink, lo)
        pick = rng.choice(pool, size=min(n_extra, pool.size), replace=False)
        ex[b, :pick.size] = pick
        added += pick.size * blk
    return ex, added


def union_window_keys(n: int, q_len: int, blk=128, n_sink=1, n_local=7) -> int:
    """Distinct keys the last q_len positions of a length-n sequence attend
    (the union of their SSA key sets), counted block by block."""
    keys = set()
    for t in range(n - q_len, n):
        qb = t // blk
        for kb in range(qb + 1):
            if kb < n_sink or qb - kb < n_local:
                keys.update(range(kb * blk, min((kb + 1) * blk, t + 1)))
    return len(keys)


def decode_bench(iters, warmup, peaks, seed=0, len_hi=None, n_sets=8, world=1, n_extra=0,
                 q_len=1, fp8=False):
    """Paged decode through the public call.  ``value``: algorithmic bytes per
    call / device time per call, with the calls captured in a CUDA graph (the
    way a serving loop issues decode steps) and rotating over ``n_sets``
    batches that share the page pool but read different pages (own page
    table and queries each), so that consecutive calls find nothing of their
    inputs in L2.  ``n_extra`` > 0: the selected-pages decode, each sequence
    also attending ``n_extra`` distinct pages chosen between its sink and its
    local run.  ``q_len`` > 1: several query tokens per sequence (the
    multi-token decode); the bytes count the union of the tokens' key sets
    once, the FLOPs every token's own set.  ``fp8``: the same workload over an
    FP8 cache (e4m3 codes + one fp32 scale per token, 580 bytes per key).  ``eager_flush_us``: one eager call per step after a 2x L2
    write, for comparison (it also pays the write-back of the flushed lines
    and, when the GPU runs dry, the host-side cost of the call)."""
    import torch
    from block_sparse_streaming_ssa_b200 import synth
    from block_sparse_streaming_ssa_b200.loza_ssa import (loza_ssa_decode, loza_ssa_decode_fp8,
                                                          loza_ssa_decode_mtp,
                                                          loza_ssa_decode_mtp_workspace_size,
                                                          loza_ssa_decode_selected,
                                                          loza_ssa_decode_selected_workspace_size)
    s = synth.DECODE
    lens = synth.decode_seq_lens(seed, s.B, s.len_lo, len_hi or s.len_hi)
    ksc = None
    if fp8:
        q, kv, ksc, pt, sl = synth.decode_inputs_fp8(lens, s.H_q, s.d_qk, seed=seed,
                                                     device="cuda")
    else:
        q, kv, pt, sl = synth.decode_inputs(lens, s.H_q, s.d_qk, seed=seed, device="cuda",
                                            q_len=q_len if q_len > 1 else None)
    key_bytes = s.d_qk + 4 if fp8 else s.d_qk * 2
    ex_h, extra_keys = decode_extra_pages(lens, n_extra, seed)
    extra = torch.as_tensor(ex_h, device="cuda")
    ws_bytes = (loza_ssa_decode_mtp_workspace_size(s.B, q_len, s.H_q, s.d_v, 1, 7) if q_len > 1
                else loza_ssa_decode_selected_workspace_size(s.B, s.H_q, s.d_v, 1, 7, n_extra))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")

    def decode(qq, pp, **kw):
        if fp8:
            return loza_ssa_decode_fp8(qq, kv, ksc, pp, sl, s.d_v, scale=s.scale, workspace=ws,
                                       **kw)
        if q_len > 1:
            return loza_ssa_decode_mtp(qq, kv, pp, sl, s.d_v, scale=s.scale, workspace=ws, **kw)
        if n_extra:
            return loza_ssa_decode_selected(qq, kv, pp, sl, extra, s.d_v, scale=s.scale,
                                            workspace=ws, **kw)
        return loza_ssa_decode(qq, kv, pp, sl, s.d_v, scale=s.scale, workspace=ws, **kw)

    o, lse = decode(q, pt)
    keys = int(sum(row_pairs(np.arange(n - q_len, n)).sum() for n in lens)) + extra_keys
    read_keys = (int(sum(union_window_keys(n, q_len) for n in lens)) + extra_keys if q_len > 1
                 else keys)
    algo_bytes = read_keys * key_bytes + q.numel() * 2 + o.numel() * 2 + lse.numel() * 4
    flops = 2 * (s.d_qk + s.d_v) * keys * s.H_q

    gen = torch.Generator(device="cpu").manual_seed(1000 + seed)
    sets = [(q, pt)]
    for _ in range(n_sets - 1):
        perm = torch.randperm(kv.shape[0], generator=gen).to(torch.int32).cuda()
        sets.append((torch.randn(q.shape, generator=gen).to(torch.bfloat16).cuda(),
                     torch.where(pt >= 0, perm[pt.clamp(min=0).long()], pt)))
    distinct_kv = n_sets * keys * key_bytes

    def call(i):
        qq, pp = sets[i % n_sets]
        decode(qq, pp, o=o, lse=lse)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for i in range(max(warmup, n_sets)):
            call(i)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        for i in range(iters):
            call(i)
    torch.cuda.synchronize()
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    reps = []
    for _ in range(5):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        graph.replay()
        b.record()
        torch.cuda.synchronize()
        reps.append(a.elapsed_time(b) / iters)
    ms = max_over_ranks(statistics.median(reps))

    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")
    eager = []
    for i in range(iters):
        flush.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        call(i)
        b.record()
        eager.append((a, b))
    torch.cuda.synchronize()
    eager_ms = statistics.median([a.elapsed_time(b) for a, b in eager])
    del graph

    gbs = job_throughput(world, algo_bytes, 1, ms) / 1e9
    return {
        "workload": f"ssa_decode B={s.B} H_q={s.H_q} d_qk={s.d_qk} d_v={s.d_v} paged 128, "
                    f"seq_len U[{s.len_lo},{len_hi or s.len_hi}] seed {seed}, random page permutation "
                    f"over {kv.shape[0]} pages"
                    + (f", plus {n_extra} distinct selected pages per sequence" if n_extra else "")
                    + (f", {q_len} query tokens per sequence" if q_len > 1 else "")
                    + (", FP8 e4m3 cache with one fp32 scale per token" if fp8 else ""),
        "value": round(gbs, 1), "unit": "GB/s", "us_per_step": round(ms * 1e3, 2),
        "algorithmic_bytes_per_step": algo_bytes, "useful_gflop_per_step": round(flops / 1e9, 3),
        "tflops": round(flops / (ms * 1e-3) / 1e12, 1),
        "l2": f"inputs larger than L2: {n_sets} rotating batches with their own page tables "
              f"and queries ({distinct_kv / 2**20:.0f} MiB of distinct KV pages), "
              f"{iters} calls per CUDA graph replay",
        "eager_flush_us": round(eager_ms * 1e3, 2),
        "roofline": {"bound": "hbm", "achieved": round(gbs / world, 1), "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": round(gbs / world / peaks["hbm_gbs"], 4),
                     "traffic": traffic_lookup("ssa_decode_split_kernel",
                                               "decode_fp8" if fp8 else
                                               "decode_selected" if n_extra else
                                               f"decode_mtp{q_len}" if q_len > 1 else "decode"),
                     "peak_source": peaks["source"],
                     "note": "time of the whole call: split kernel + LSE merge kernel"},
        "gpu_launches": 2 * iters * 5 + 2 * iters,
    }


def prefill_context_bench(peaks, L=131072, world=1, seed=0):
    """Prefill of one layer at a long context: full causal attention (a kept
    MLA layer of the ZigZag stack: no sink, a window of every block) against
    SSA, on the MLA-dims workload shape (B=1, H=64, d_qk=192, d_v=128) at L
    tokens.  One warm-up and two timed calls of the full layer (each is a long
    call, so it runs under the power cap); five of the SSA layer."""
    import dataclasses
    import torch
    from block_sparse_streaming_ssa_b200 import synth
    from block_sparse_streaming_ssa_b200.loza_ssa import loza_ssa_prefill
    sp = dataclasses.replace(synth.MLA, L=L)
    q, k, v = synth.prefill_spec_inputs(sp, seed=seed, device="cuda")
    nb = (L + 127) // 128
    o = torch.empty((sp.B, sp.H, L, sp.d_v), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((sp.B, sp.H, L), dtype=torch.float32, device="cuda")

    def timed(n_sink, n_local, warmup, iters):
        for _ in range(warmup):
            loza_ssa_prefill(q, k, v, o=o, lse=lse, n_sink=n_sink, n_local=n_local,
                             scale=sp.scale)
        ev = []
        for _ in range(iters):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            loza_ssa_prefill(q, k, v, o=o, lse=lse, n_sink=n_sink, n_local=n_local,
                             scale=sp.scale)
            b.record()
            ev.append((a, b))
        torch.cuda.synchronize()
        return max_over_ranks(statistics.median([a.elapsed_time(b) for a, b in ev]))

    ssa_ms = timed(1, 7, 3, 5)
    full_ms = timed(0, nb, 1, 2)
    full_flops = 2 * (sp.d_qk + sp.d_v) * sp.B * sp.H * (L * (L + 1) // 2)
    ssa_flops = 2 * (sp.d_qk + sp.d_v) * sp.B * sp.H * window_pairs(L)
    full_tf = full_flops / (full_ms * 1e-3) / 1e12
    del q, k, v, o, lse
    torch.cuda.empty_cache()
    return {
        "workload": f"prefill at {L} tokens: B={sp.B} H={sp.H} d_qk={sp.d_qk} d_v={sp.d_v} bf16; "
                    f"full causal layer (window of all {nb} blocks) vs SSA layer (1 sink + 7 local)",
        "full_layer_ms": round(full_ms, 3), "ssa_layer_ms": round(ssa_ms, 4),
        "layer_speedup": round(full_ms / ssa_ms, 1),
        "zigzag_pair_speedup": round(2 * full_ms / (full_ms + ssa_ms), 2),
        "full_layer_tflops": round(full_tf, 1),
        "ssa_layer_tflops": round(ssa_flops / (ssa_ms * 1e-3) / 1e12, 1),
        "full_layer_roofline": {"bound": "tensor", "achieved": round(full_tf, 1),
                                "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                                "frac": round(full_tf / peaks["bf16_tflops_sustained"], 4),
                                "peak_source": peaks["source"] + " (sustained bf16 GEMM)"},
        "gpu_launches": 8 + 3,
    }


def context_bench(peaks, context=131072, iters=5, warmup=3, world=1, seed=0):
    """Decode at one long context through the layer-stack call: a full-attention
    (MLA) layer against an SSA layer, and a 4-layer ZigZag stack (full, SSA,
    full, SSA -- the QbitAI LoZA article's layout, half the layers SSA) against
    4 full layers.  32 sequences of ``context`` tokens each, 128 heads, 576/512,
    every layer with its own query and page pool; a 2x L2 write before every
    timed call.  Full-attention layers run as the SSA decode with a window of
    every page."""
    import torch
    from block_sparse_streaming_ssa_b200 import synth
    from block_sparse_streaming_ssa_b200.loza_ssa import (loza_ssa_decode_layers,
                                                          loza_ssa_decode_layers_workspace_size)
    s = synth.DECODE
    lens = [context] * s.B
    pools = []
    for i in range(4):
        q, kv, pt, sl = synth.decode_inputs(lens, s.H_q, s.d_qk, seed=seed + 17 * i,
                                            device="cuda")
        pools.append((q, kv))
        if i == 0:
            table, seq_lens = pt, sl
    max_pages = table.shape[1]
    ws = torch.empty(loza_ssa_decode_layers_workspace_size(s.B, s.H_q, s.d_v, max_pages, 1, 7,
                                                           True), dtype=torch.uint8,
                     device="cuda")
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")

    def timed(pattern):
        layers = [(pools[i][0], pools[i][1], full) for i, full in enumerate(pattern)]
        for _ in range(warmup):
            loza_ssa_decode_layers(layers, table, seq_lens, s.d_v, scale=s.scale, workspace=ws)
        ev = []
        for _ in range(iters):
            flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            loza_ssa_decode_layers(layers, table, seq_lens, s.d_v, scale=s.scale, workspace=ws)
            b.record()
            ev.append((a, b))
        torch.cuda.synchronize()
        return max_over_ranks(statistics.median([a.elapsed_time(b) for a, b in ev]))

    full_ms = timed((True,))
    ssa_ms = timed((False,))
    zigzag_ms = timed((True, False, True, False))
    all_full_ms = timed((True, True, True, True))
    full_bytes = s.B * (context * s.d_qk * 2 + s.H_q * (s.d_qk * 2 + s.d_v * 2 + 4))
    t16 = traffic_lookup("ssa_decode_long_kernel", "ctx16k")
    traffic = None if t16 is None else int(t16 * context / 16384)
    full_flops = 2 * (s.d_qk + s.d_v) * s.B * s.H_q * context
    gbs = full_bytes / (full_ms * 1e-3) / 1e9
    del pools, ws, flush
    torch.cuda.empty_cache()
    return {
        "workload": f"decode at {context} tokens of context: B={s.B} H_q={s.H_q} d_qk={s.d_qk} "
                    f"d_v={s.d_v} paged 128, random page permutation, own pool per layer",
        "full_layer_ms": round(full_ms, 4), "ssa_layer_ms": round(ssa_ms, 4),
        "layer_speedup": round(full_ms / ssa_ms, 1),
        "zigzag4_ms": round(zigzag_ms, 4), "full4_ms": round(all_full_ms, 4),
        "stack_speedup": round(all_full_ms / zigzag_ms, 2),
        "full_layer_gbs": round(gbs, 1),
        "full_layer_tflops": round(full_flops / (full_ms * 1e-3) / 1e12, 1),
        "full_layer_roofline": {"bound": "hbm", "achieved": round(gbs, 1),
                                "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                "frac": round(gbs / peaks["hbm_gbs"], 4),
                                "peak_source": peaks["source"],
                                "kernel": "ssa_decode_long_kernel",
                                "traffic": traffic,
                                "traffic_note": "ncu DRAM bytes of one launch at 16384 tokens, "
                                                "scaled by the context length"},
        "l2": "2x L2 write before every timed call",
        # a full-attention layer: plan, long-window and merge kernels; an SSA
        # layer: the split kernel with its in-cluster merge
        "gpu_launches": (3 + 1 + (3 + 1 + 3 + 1) + 4 * 3) * (iters + warmup),
    }


# ----------------------------------------------------------- CPU oracle

def oracle_sample(config, budget_s, seed=0):
    """Time the CPU oracle (as it stands) on a bounded row sample of the
    workload; returns (useful flops, seconds, rows, threads, description)."""
    import torch
    from block_sparse_streaming_ssa_b200 import synth
    from oracle import ssa_oracle as orc
    sp = {"tiny": synth.TINY, "mha": synth.MHA, "mla": synth.MLA, "varlen": synth.MHA}[config]
    H = 2 if sp.H >= 2 else 1
    q, k, v = synth.prefill_inputs(1, H, sp.L, sp.d_qk, sp.d_v, seed=seed, device="cpu",
                                   std=sp.std, sink_boost=sp.sink_boost)
    qb, kb, vb = (synth.bf16_bits(t) for t in (q, k, v))
    rng = np.random.default_rng(seed)

    def run(n):
        rows = np.sort(rng.choice(H * sp.L, size=n, replace=False))
        t = time.perf_counter()
        orc.prefill(qb, kb, vb, 128, 1, 7, sp.scale, rows=rows)
        dt = time.perf_counter() - t
        fl = 2 * (sp.d_qk + sp.d_v) * int(row_pairs(rows % sp.L).sum())
        return fl, dt, n

    fl, dt, n = run(64)
    n2 = int(min(H * sp.L, max(64, 64 * budget_s / max(dt, 1e-3))))
    fl, dt, n = run(n2)
    passes = 1
    while dt < budget_s:  # every row of the sample already taken: run fresh samples
        f2, d2, _ = run(n2)
        fl, dt, passes = fl + f2, dt + d2, passes + 1
    return fl, dt, n * passes, orc.num_threads(), (
        f"{passes} x {n} random query rows of {H} heads of the {sp.name} workload (B=1, "
        f"L={sp.L}, d_qk={sp.d_qk}, d_v={sp.d_v}), each against its full SSA window, float64")


# ------------------------------------------------------------------- main

def prefill_leg(config, steps, warmup, peaks, dist, world, rank, heads=None):
    """Time one prefill workload: (compact entry, detail, raw timing)."""
    import torch
    w = make_prefill(config, "cuda", seed=rank, heads=heads)
    total_ms, per, clocks = time_prefill(w, steps, warmup, dist)
    max_ms = max_over_ranks(total_ms)
    flops = 2 * (w["spec"].d_qk + w["spec"].d_v) * w["pairs"]
    avg_launch_ms = sum(per) / len(per)
    achieved = flops / (avg_launch_ms * 1e-3) / 1e12
    value = job_throughput(world, flops, steps, max_ms) / 1e12
    tok_s = job_throughput(world, w["tokens"], steps, max_ms)
    entry = {"tflops": round(value, 1), "frac": round(achieved / peaks["bf16_tflops"], 3),
             "ms": round(max_ms / steps, 4), "mtok_s": round(tok_s / 1e6, 2)}
    return w, entry, dict(total_ms=total_ms, max_ms=max_ms, flops=flops, achieved=achieved,
                          value=value, tok_s=tok_s, avg_launch_ms=avg_launch_ms, clocks=clocks)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", choices=["mla", "mha", "tiny", "varlen"], default="mla",
                    help="the headline prefill workload (default: the MLA-dims one, the largest "
                         "that fits one GPU)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-prefill", action="store_true",
                    help="time only the decode workload (for profiler captures of it)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip timing the prefill's backward pass")
    ap.add_argument("--no-other-prefill", action="store_true",
                    help="time only the headline prefill workload")
    ap.add_argument("--prefill-heads", type=int, default=None,
                    help="headline prefill with this many heads instead (a smaller case of the "
                         "same shapes, for profiler captures)")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the host-buffer call (for profiler captures)")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--decode-iters", type=int, default=30)
    ap.add_argument("--decode-len-hi", type=int, default=None,
                    help="shorter decode contexts (smaller page pool), for profiler captures")
    ap.add_argument("--decode-extra", type=int, default=8,
                    help="also time the selected-pages decode with this many chosen pages per "
                         "sequence (0: skip it)")
    ap.add_argument("--decode-mtp", type=int, default=2,
                    help="also time the decode with this many query tokens per sequence "
                         "(<= 1: skip it)")
    ap.add_argument("--decode-fp8", type=int, default=1,
                    help="also time the decode over an FP8 cache (0: skip it)")
    ap.add_argument("--decode-context", type=int, default=131072,
                    help="also time full-attention vs SSA decode layers at this context "
                         "(0: skip it)")
    ap.add_argument("--prefill-context", type=int, default=131072,
                    help="also time a full-attention vs an SSA prefill layer at this length "
                         "(0: skip it)")
    ap.add_argument("--cpu-budget-s", type=float, default=10.0)
    ap.add_argument("--ref-budget-s", type=float, default=60.0,
                    help="--impl reference: CPU seconds over all warm-up and timed steps")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    peaks = load_peaks()

    if args.impl == "reference":
        if rank != 0:
            return
        per_step_budget = max(0.1, args.ref_budget_s / (args.steps + args.warmup))
        fl_tot, t_tot, rows_tot = 0, 0.0, 0
        threads, desc = 1, ""
        for i in range(args.warmup + args.steps):
            fl, dt, n, threads, desc = oracle_sample(args.config, per_step_budget, seed=i)
            if i >= args.warmup:
                fl_tot, t_tot, rows_tot = fl_tot + fl, t_tot + dt, rows_tot + n
        val = fl_tot / t_tot / 1e12
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t_tot / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": line_config(workload_name(args.config)),
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
        }), flush=True)
        return

    import torch
    from block_sparse_streaming_ssa_b200 import build as cuda_build
    cuda_build.build()
    dist = world > 1
    if dist:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)

    def decode_legs():
        rest()
        legs = {"decode": decode_bench(args.decode_iters, args.warmup, peaks, seed=rank,
                                       len_hi=args.decode_len_hi, world=world)}
        if args.decode_extra:
            legs[f"dec_sel{args.decode_extra}"] = decode_bench(
                args.decode_iters, args.warmup, peaks, seed=rank, len_hi=args.decode_len_hi,
                world=world, n_extra=args.decode_extra)
        if args.decode_mtp > 1:
            legs[f"dec_mtp{args.decode_mtp}"] = decode_bench(
                args.decode_iters, args.warmup, peaks, seed=rank, len_hi=args.decode_len_hi,
                world=world, q_len=args.decode_mtp)
        if args.decode_fp8:
            legs["dec_fp8"] = decode_bench(args.decode_iters, args.warmup, peaks, seed=rank,
                                           len_hi=args.decode_len_hi, world=world, fp8=True)
        if args.decode_context:
            rest()
            legs["ctx_dec"] = context_bench(peaks, args.decode_context, world=world, seed=rank)
        return legs

    def compact(name, d):
        if d is None:
            return None
        if name == "ctx_dec":
            return {"full_ms": round(d["full_layer_ms"], 3),
                    "ssa_us": round(d["ssa_layer_ms"] * 1e3, 1), "stack4_x": d["stack_speedup"],
                    "full_frac": round(d["full_layer_roofline"]["frac"], 3)}
        if name.startswith("bwd"):
            return {"tflops": round(d["value"], 1), "frac": round(d["roofline"]["frac"], 3)}
        return {"gbs": round(d["value"]), "frac": round(d["roofline"]["frac"], 3)}

    if args.no_prefill:
        legs = decode_legs()
        if rank == 0:
            print(json.dumps({"metric": METRIC, **legs}), file=sys.stderr, flush=True)
            print(json.dumps({"metric": METRIC,
                              "configs": {k: compact(k, v) for k, v in legs.items()}}),
                  flush=True)
        if dist:
            torch.distributed.destroy_process_group()
        return

    # ---- headline prefill workload
    w, head_entry, t = prefill_leg(args.config, args.steps, args.warmup, peaks, dist, world, rank,
                                   heads=args.prefill_heads)
    e2e_ms, h2d, d2h = (None, 0, 0) if args.no_e2e else e2e_prefill(w, args.e2e_steps)
    # every rank runs the same e2e loop
    e2e_val = None if e2e_ms is None else world * t["flops"] / (e2e_ms * 1e-3) / 1e12
    w_desc, w_spec = w["desc"], w["spec"]
    detail = {"headline": {"workload": w_desc, **head_entry,
                           "e2e_ms": e2e_ms and round(e2e_ms, 3), "clocks": t["clocks"]},
              "idle_s_before_each_other_workload": REST_S}
    configs = {}
    backwards = {}
    if not args.no_backward:
        rest()
        b = backward_bench(w, max(3, args.steps // 4), args.warmup, peaks, world)
        if b is not None:
            backwards[f"bwd_{args.config}"] = b
    del w
    torch.cuda.empty_cache()

    # ---- the other prefill workloads (each its own timed region, same timing rules)
    if not args.no_other_prefill:
        for other in ("mha", "varlen", "mla"):
            if other == args.config:
                continue
            rest()
            w2, entry, _ = prefill_leg(other, args.steps, args.warmup, peaks, dist, world, rank)
            # the line keeps rates and fractions; times and workloads go to the detail
            configs[other] = {k: entry[k] for k in ("tflops", "frac", "mtok_s")}
            detail[other] = {"workload": w2["desc"]["workload"], **entry}
            if other == "mha" and not args.no_backward:
                rest()
                backwards["bwd_mha"] = backward_bench(w2, max(3, args.steps // 4), args.warmup,
                                                      peaks, world)
            del w2
            torch.cuda.empty_cache()
    for name, b in backwards.items():
        configs[name] = compact("bwd", b)
        detail[name] = b
    if args.prefill_context:
        rest()
        pctx = prefill_context_bench(peaks, args.prefill_context, world=world, seed=rank)
        detail["ctx_pre"] = pctx
    if not args.no_decode:
        for k, v in decode_legs().items():
            configs[k] = compact(k, v)
            detail[k] = v

    if rank != 0:
        if dist:
            torch.distributed.destroy_process_group()
        return

    cpu = None
    if not args.no_cpu_baseline and world == 1:
        fl, dt, n, threads, desc = oracle_sample(args.config, args.cpu_budget_s)
        cpu = {"value": round(fl / dt / 1e12, 5), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{n} rows of {args.config}, f64, {dt:.0f} s"}
        detail["cpu_baseline"] = {**cpu, "sample": desc + f", {dt:.1f} s"}
    kname = "ssa_prefill_kernel"
    peak = peaks["bf16_tflops"]
    clocks = t["clocks"]
    line = {
        "metric": METRIC, "value": round(t["value"], 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(t["max_ms"] / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": line_config(w_desc["workload"]),
        "tokens_per_s": round(t["tok_s"]),
        "roofline": {"bound": "tensor", "achieved": round(t["achieved"], 1), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(t["achieved"] / peak, 4),
                     "traffic": traffic_lookup(kname, args.config)},
        "cpu_baseline": cpu,
        "e2e": None if e2e_val is None else {
            "value": round(e2e_val, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h},
        "clocks": {k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
        "gpu_launches": args.steps,
        "configs": configs,
    }
    detail["headline"]["roofline"] = {
        **line["roofline"], "kernel": kname, "avg_launch_ms": round(t["avg_launch_ms"], 4),
        "peak_source": peaks["source"],
        "frac_of_sustained": round(t["achieved"] / peaks["bf16_tflops_sustained"], 4)}
    print(json.dumps(detail), file=sys.stderr, flush=True)
    print(json.dumps(line), flush=True)
    if dist:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
