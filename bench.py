#!/usr/bin/env python
"""Benchmark of the fused causal GQA + RoPE attention forward on B200.

One step = one call of the public C-ABI entry point (prologue kernel +
attention kernel) over one batch of synthetic, seeded inputs already resident
in HBM. Default workload: Llama-3-8B-shaped causal prefill (B=1, T=8192,
32 query / 8 KV heads, d=128, theta=5e5, bf16). Metric: TFLOP/s counting
4*T*T*d per query head, halved for causal.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   (the float64 CPU oracle, timed)
  --workload decode_llama8b | decode_qwen3b | ...   one decoding step
  --workload bwd_llama8b | bwd_varlen | bwd_nano    the backward (dq, dk, dv)
  --workload qkv_llama8b | qkv_nano                 the QKV projection with its RoPE epilogue
  --workload masked_llama8b | masked_nano           the forward with an additive mask
  --workload rot_llama8b | rot_varlen | ...          the forward on already rotated q and k

Under torchrun each rank runs its own replica of the workload (independent
problems, weak scaling); the elapsed time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "causal GQA+RoPE attention fwd TFLOP/s on 1 B200; % of dense-BF16 tensor peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


KERNEL_SOURCES = ("attn_kernel.cuh", "prep_kernel.cuh", "common.cuh", "ptx.cuh", "rope_round.cuh",
                  "exp2_poly.cuh", "gqa_rope_attn.cu")


def recorded_traffic(workload: str):
    """DRAM bytes (read + write) per launch of the attention kernel from the
    committed ncu capture for this workload, or None when there is none or
    when the kernel sources have changed since it was taken (the capture
    records a SHA-256 over the sources)."""
    import hashlib
    p = os.path.join(ROOT, "profiles", f"gqa_attn_fwd_kernel.{workload}.traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "transformer_attention_gqa_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    if rec.get("sources_sha256") != h.hexdigest():
        return None
    return int(rec["dram_bytes_per_launch"])


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        import shutil
        import tempfile
        if not shutil.which("nvidia-smi"):
            return
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        self.fh = open(self.path, "w")
        self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                      "--format=csv,noheader,nounits", "-lms", "200"],
                                     stdout=self.fh, stderr=subprocess.DEVNULL)
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ oracle timing
_INPUTS = {}


def _cached_inputs(workload):
    from transformer_attention_gqa_b200 import workloads as wl

    if workload.name not in _INPUTS:
        _INPUTS[workload.name] = wl.make_inputs(workload)
    return _INPUTS[workload.name]


def _oracle_rows(inp, w, rows):
    import oracle.gqa_oracle as orc

    t0 = time.perf_counter()
    orc.gqa_rope_attention(inp.q, inp.k, inp.v, inp.cu_seqlens, w.n_q_heads, w.n_kv_heads, w.rope_theta,
                           causal=w.causal, query_rows=rows)
    dt = time.perf_counter() - t0
    cu = inp.cu_seqlens
    seq = np.searchsorted(cu, rows, side="right") - 1
    tok = rows - cu[seq]
    L = cu[seq + 1] - cu[seq]
    keys = (tok + 1) if w.causal else L
    # metric convention: 4*Tq*Tk*d per head, halved for causal == 4*d per (row, visible key, head)
    return dt, float(np.sum(4.0 * keys * w.head_dim * w.n_q_heads))


_PROBES = {}


def _oracle_probe(w, inp):
    """(fixed seconds, seconds per query row) of one oracle call on this
    workload, from two small probes (8 and 64 random rows), once per process.
    The fixed part is the call's work that does not depend on the number of
    rows (the rotation of the sequences' q and k)."""
    if w.name not in _PROBES:
        rng = np.random.default_rng(12345)
        pick = lambda n: np.sort(rng.choice(w.total_tokens, size=min(n, w.total_tokens), replace=False))
        t8, _ = _oracle_rows(inp, w, pick(8))
        t64, _ = _oracle_rows(inp, w, pick(64))
        per_row = max((t64 - t8) / 56.0, 1e-6)
        _PROBES[w.name] = (max(t8 - 8 * per_row, 0.0), per_row)
    return _PROBES[w.name]


def cpu_baseline(workload, budget_s: float = 15.0, seed_rows: int = 0, beyond_fixed: bool = False):
    """Times the float64 oracle, as it stands, on a bounded sample of random
    query rows of the workload (the probes size the sample to about budget_s
    seconds, or to budget_s seconds of per-row work beyond the call's fixed
    part with beyond_fixed); returns its TFLOP/s by the metric's convention."""
    w = workload
    inp = _cached_inputs(w)
    fixed, per_row = _oracle_probe(w, inp)
    rng = np.random.default_rng(seed_rows)
    pick = lambda n: np.sort(rng.choice(w.total_tokens, size=min(n, w.total_tokens), replace=False))
    work_s = budget_s if beyond_fixed else budget_s - fixed
    n = int(max(8, min(w.total_tokens, work_s / per_row)))
    dt, flops = _oracle_rows(inp, w, pick(n))
    cores = len(os.sched_getaffinity(0))
    threads = None
    try:
        from threadpoolctl import threadpool_info
        threads = max((x.get("num_threads", 0) for x in threadpool_info()), default=None)
    except Exception:
        pass
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": threads or cores, "kind": "oracle",
            "sample": f"{n} random query rows x {w.n_q_heads} heads of {w.name} (all their visible keys), "
                      f"float64 NumPy, {dt:.1f} s", "host_cores": cores}


# ------------------------------------------------------------------ shared timing
def _rt_events():
    """cudaEvent_t create / elapsed-ms / destroy through cuda.bindings (for
    events handed to the library, which records them on its own stream)."""
    from cuda.bindings import runtime as rt

    def create():
        err, e = rt.cudaEventCreate()
        assert int(err) == 0
        return e

    def elapsed(a, b):
        err, ms = rt.cudaEventElapsedTime(a, b)
        assert int(err) == 0
        return float(ms)

    return create, elapsed, rt.cudaEventDestroy


def _timed_steps(step, steps, stream, flush=None):
    """Total device ms of `steps` calls of step(), each between CUDA events on
    `stream`, with the L2 flushed before each outside its events, bracketed
    by barriers and synchronisation."""
    import torch
    from transformer_attention_gqa_b200 import replicas

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    replicas.barrier()
    torch.cuda.synchronize()
    for i in range(steps):
        if flush is not None:
            flush.zero_()
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    replicas.barrier()
    return sum(a.elapsed_time(b) for a, b in ev)


def _library_kernel_ms(step, calls, flush=None):
    """Median durations (ms) of the first and the second kernel of the library
    call step() makes, from events the library records around them on its
    stream (gqa_rope_attn_set_profile_events), over `calls` calls."""
    import torch
    from transformer_attention_gqa_b200 import _abi

    create, elapsed, destroy = _rt_events()
    kern = []
    for _ in range(calls):
        e = [create() for _ in range(3)]
        if flush is not None:
            flush.zero_()
        _abi.set_profile_events(int(e[0]), int(e[1]), int(e[2]))
        step()
        kern.append(e)
    torch.cuda.synchronize()
    first = statistics.median(elapsed(a, b) for a, b, _ in kern)
    second = statistics.median(elapsed(b, c) for _, b, c in kern)
    for e in kern:
        for x in e:
            destroy(x)
    return first, second


def _e2e_serial_ms(step, ins, outs, stream, steps):
    """Mean ms per end-to-end step on `stream`: every step copies each
    (device, pinned host) pair of `ins` to the device, runs step(), and
    copies each (pinned host, device) pair of `outs` back."""
    import torch
    from transformer_attention_gqa_b200 import replicas

    def one():
        for d_, h_ in ins:
            d_.copy_(h_, non_blocking=True)
        step()
        for h_, d_ in outs:
            h_.copy_(d_, non_blocking=True)

    for _ in range(2):
        one()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    replicas.barrier()
    e0.record(stream)
    for _ in range(steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def _nbytes(tensors):
    return sum(t.numel() * t.element_size() for t in tensors)


def _reference_line(args, world, metric, unit, config, sample, digits=6):
    """The --impl reference JSON line: the oracle, as it stands, on bounded
    samples of the workload (sample(budget_s, index) -> cpu_baseline dict;
    index 1000 + i for the args.warmup short warm-up samples, i for the
    args.steps timed ones), reporting the median. ``config`` is the GPU
    arm's config dict for the same workload."""
    for i in range(args.warmup):
        sample(0.5, 1000 + i)
    vals, info = [], None
    for i in range(args.steps):
        info = sample(max(1.0, min(5.0, 60.0 / max(args.steps, 1))), i)
        vals.append(info["value"])
    val = round(statistics.median(vals), digits)
    return {"impl": "reference", "metric": metric, "value": val, "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
            "cpu_baseline": {"value": val, "unit": unit, "cores": info["cores"], "kind": "oracle",
                             "sample": info["sample"]},
            "e2e": {"value": val, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------ decoding
DECODE_METRIC = "GQA+RoPE decode step (KV cache read, new row appended) algorithmic HBM GB/s on 1 B200"
DECODE_UNIT = "GB/s"


def _decode_sample_bytes(w, sel):
    lens = np.asarray(w.cache_lens)[sel]
    return float(np.sum(lens + 1)) * w.n_kv_heads * w.head_dim * 2 * 2


def decode_config(w, world):
    big = w.kv_bytes() > 2 * (126 << 20)
    return {"workload": w.name, "shape": w.description, "batch": w.batch, "max_cache_len": w.max_cache_len,
            "n_q_heads": w.n_q_heads, "n_kv_heads": w.n_kv_heads, "head_dim": w.head_dim,
            "algorithmic_bytes_per_step": w.step_bytes(), "tokens_per_step": w.batch,
            "parallelism": f"replicas x{world}",
            "l2": "K/V read per step larger than L2" if big else "256 MiB written before every timed step"}


def cpu_baseline_decode(w, inp, budget_s: float = 15.0, seed: int = 0):
    """Times the float64 oracle's decoding step on a bounded random sample of
    the batch's sequences; returns the algorithmic K/V bytes of the sample
    per second (GB/s), the decode metric's convention."""
    import oracle.gqa_oracle as orc

    rng = np.random.default_rng(seed)

    def run(n):
        sel = np.sort(rng.choice(w.batch, size=min(n, w.batch), replace=False))
        t0 = time.perf_counter()
        orc.gqa_rope_decode(inp.q[sel], inp.k_new[sel], inp.v_new[sel], inp.k_cache[sel], inp.v_cache[sel],
                            inp.cache_seqlens[sel], w.n_q_heads, w.n_kv_heads, w.rope_theta)
        return time.perf_counter() - t0, sel

    t1, _ = run(1)
    n = int(max(1, min(w.batch, budget_s / max(t1, 1e-3))))
    dt, sel = run(n)
    cores = len(os.sched_getaffinity(0))
    return {"value": _decode_sample_bytes(w, sel) / dt / 1e9, "unit": DECODE_UNIT, "cores": cores,
            "kind": "oracle", "sample": f"{len(sel)} of {w.batch} sequences of {w.name}, float64 NumPy, {dt:.1f} s"}


def run_decode(args, rank, world, local_rank):
    import torch
    import transformer_attention_gqa_b200 as g
    from transformer_attention_gqa_b200 import _abi, replicas, workloads as wl

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = wl.DECODE_WORKLOADS[args.workload]
    inp = wl.make_decode_inputs(w, seed=w.seed if rank == 0 else replicas.replica_seed(w.seed, rank), nan_tail=False)
    bf = torch.bfloat16
    q = torch.from_numpy(inp.q).to(bf).to(dev)
    kn = torch.from_numpy(inp.k_new).to(bf).to(dev)
    vn = torch.from_numpy(inp.v_new).to(bf).to(dev)
    kc = torch.from_numpy(inp.k_cache).to(bf).to(dev)
    vc = torch.from_numpy(inp.v_cache).to(bf).to(dev)
    lens = torch.from_numpy(inp.cache_seqlens).to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((w.n_q_heads, w.batch), dtype=torch.float32, device=dev)
    ws = g.Workspace(dev)
    stream = torch.cuda.current_stream(dev)
    big = w.kv_bytes() > 2 * (126 << 20)
    flush = None if big else torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step():  # the same token each step: row p is rewritten with the same values
        g.gqa_rope_attn_decode(q, kn, vn, kc, vc, lens, w.rope_theta, out=out, lse=lse, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert g.get_device_status() == 0
    launches_per_step = _abi.last_launch_count()
    clocks = ClockSampler(local_rank)
    clocks.start()
    total_ms = _timed_steps(step, args.steps, stream, flush)
    split_ms, merge_ms = _library_kernel_ms(step, max(3, min(args.steps, 10)), flush)
    clk = clocks.stop()

    # end to end: the token's q, k_new, v_new and the lengths from pinned host
    # memory, out and lse back; the cache stays resident on the device
    ins = [(d_, d_.cpu().pin_memory()) for d_ in (q, kn, vn, lens)]
    outs = [(torch.empty(d_.shape, dtype=d_.dtype).pin_memory(), d_) for d_ in (out, lse)]
    h2d, d2h = _nbytes(h_ for _, h_ in ins), _nbytes(h_ for h_, _ in outs)
    e2e_ms = _e2e_serial_ms(step, ins, outs, stream, max(3, min(args.steps, 10)))
    assert g.get_device_status() == 0

    total_ms, e2e_ms, split_ms, merge_ms = replicas.max_over_ranks([total_ms, e2e_ms, split_ms, merge_ms], device=dev)
    ms_per_step = total_ms / args.steps
    nbytes = w.step_bytes()
    peaks, src = load_peaks()
    peak = float(peaks["hbm_gbs"])
    achieved = nbytes / ((split_ms + merge_ms) * 1e-3) / 1e9
    res = {
        "metric": DECODE_METRIC, "value": round(nbytes * world / (ms_per_step * 1e-3) / 1e9, 1),
        "unit": DECODE_UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": decode_config(w, world),
        "tokens_per_s": round(w.batch * world / (ms_per_step * 1e-3), 1),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": None,
                     "peak_source": f"{src} hbm_gbs (copy)", "kernel": "gqa_decode_split_kernel + gqa_decode_combine_kernel",
                     "split_ms": round(split_ms, 5), "merge_ms": round(merge_ms, 5)},
        "e2e": {"value": round(nbytes * world / (e2e_ms * 1e-3) / 1e9, 1), "unit": DECODE_UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 5)},
        "gpu_launches": launches_per_step * args.steps,
    }
    if clk:
        res["clocks"] = clk
    res["_inputs"] = inp
    return res


# ------------------------------------------------------------------ backward
# Backward workloads: the gradients of a forward workload's shape. One step =
# one gqa_rope_attn_bwd call (prologue, attention backward, dq rotation) on
# the forward's out and lse, computed once before timing.
BWD_WORKLOADS = {"bwd_llama8b": "llama8b", "bwd_varlen": "varlen", "bwd_nano": "nano"}
BWD_METRIC = "causal GQA+RoPE attention bwd (dq, dk, dv) TFLOP/s on 1 B200; % of dense-BF16 tensor peak"
BWD_FLOP_FACTOR = 2.5  # five products of the forward's two sizes (S recomputed, dP, dV, dK, dQ)


def cpu_baseline_bwd(w, budget_s: float = 15.0, max_len: int = 1024):
    """Times the float64 oracle's backward, as it stands, on a prefix of the
    workload's first sequence (its length sized by two probes to about
    budget_s, at most max_len tokens: the oracle holds [n_q, L, L] float64
    matrices); returns TFLOP/s by the backward's convention."""
    import oracle.gqa_oracle as orc
    from transformer_attention_gqa_b200 import workloads as wl

    inp = _cached_inputs(w)
    dout = wl.make_grad_output(inp)
    first = int(inp.cu_seqlens[1])

    def run(L):
        cu = np.array([0, L], dtype=np.int64)
        t0 = time.perf_counter()
        orc.gqa_rope_attention_backward(inp.q[:L], inp.k[:L], inp.v[:L], dout[:L], cu, w.n_q_heads, w.n_kv_heads,
                                        w.rope_theta, causal=w.causal, operand_rounding=True)
        return time.perf_counter() - t0

    L0 = min(first, 128)
    t0 = run(L0)
    L = int(max(L0, min(first, max_len, L0 * np.sqrt(max(budget_s, 0.1) / max(t0, 1e-3)))))
    dt = run(L)
    flops = BWD_FLOP_FACTOR * 4.0 * L * L * w.head_dim * w.n_q_heads / (2.0 if w.causal else 1.0)
    cores = len(os.sched_getaffinity(0))
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"first {L} tokens of {w.name}'s first sequence, all {w.n_q_heads} heads, float64 NumPy, "
                      f"{dt:.1f} s"}


def run_bwd(args, rank, world, local_rank):
    import torch
    import transformer_attention_gqa_b200 as g
    from transformer_attention_gqa_b200 import _abi, replicas, workloads as wl

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = wl.WORKLOADS[BWD_WORKLOADS[args.workload]]
    inp = wl.make_inputs(w, seed=w.seed if rank == 0 else replicas.replica_seed(w.seed, rank))
    bf = torch.bfloat16
    q = torch.from_numpy(inp.q).to(bf).to(dev)
    k = torch.from_numpy(inp.k).to(bf).to(dev)
    v = torch.from_numpy(inp.v).to(bf).to(dev)
    do = torch.from_numpy(wl.make_grad_output(inp)).to(bf).to(dev)
    cu = torch.from_numpy(inp.cu_seqlens).to(dev)
    out, lse = g.gqa_rope_attn_fwd(q, k, v, cu, w.rope_theta, causal=w.causal)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = g.Workspace(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        g.gqa_rope_attn_bwd(q, k, v, out, lse, do, cu, w.rope_theta, causal=w.causal, dq=dq, dk=dk, dv=dv,
                            workspace=ws)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    assert g.get_device_status() == 0
    launches_per_step = _abi.last_launch_count()
    clocks = ClockSampler(local_rank)
    clocks.start()
    total_ms = _timed_steps(step, args.steps, stream, flush)
    prep_ms, bwd_ms = _library_kernel_ms(step, max(3, min(args.steps, 10)), flush)
    clk = clocks.stop()

    # end to end: q, k, v, out, lse, dout and cu_seqlens from pinned host
    # memory every step, dq, dk, dv back
    ins = [(d_, d_.cpu().pin_memory()) for d_ in (q, k, v, out, lse, do, cu)]
    outs = [(torch.empty(d_.shape, dtype=d_.dtype).pin_memory(), d_) for d_ in (dq, dk, dv)]
    h2d, d2h = _nbytes(h_ for _, h_ in ins), _nbytes(h_ for h_, _ in outs)
    e2e_ms = _e2e_serial_ms(step, ins, outs, stream, max(3, min(args.steps, 10)))
    assert g.get_device_status() == 0
    assert torch.equal(outs[0][0], dq.cpu())

    total_ms, e2e_ms, bwd_ms, prep_ms = replicas.max_over_ranks([total_ms, e2e_ms, bwd_ms, prep_ms], device=dev)
    flops = BWD_FLOP_FACTOR * w.flops()
    ms_per_step = total_ms / args.steps
    value = flops * world / (ms_per_step * 1e-3) / 1e12
    peaks, src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    achieved = flops / (bwd_ms * 1e-3) / 1e12
    res = {
        "metric": BWD_METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": bwd_config(args.workload, w, world, flops),
        "pct_of_peak": round(100.0 * value / world / peak, 2),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": None,
                     "peak_source": f"{src} bf16_tflops (burst)",
                     "kernel": "gqa_attn_bwd_kernel + gqa_attn_bwd_q_kernel",
                     "kernel_ms": round(bwd_ms, 4), "prologue_ms": round(prep_ms, 4)},
        "e2e": {"value": round(flops * world / (e2e_ms * 1e-3) / 1e12, 2), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4)},
        "gpu_launches": launches_per_step * args.steps,
    }
    if clk:
        res["clocks"] = clk
    return res


def bwd_config(name, w, world, flops):
    return {"workload": name, "shape": w.description, "total_tokens": w.total_tokens,
            "num_seqs": w.num_seqs, "n_q_heads": w.n_q_heads, "n_kv_heads": w.n_kv_heads,
            "head_dim": w.head_dim, "rope_theta": w.rope_theta, "causal": w.causal,
            "flops_per_step": flops, "parallelism": f"replicas x{world}",
            "l2": "256 MiB written before every timed step, outside the step's events"}


def main_bwd(args, world, rank, local_rank):
    from transformer_attention_gqa_b200 import workloads as wl
    w = wl.WORKLOADS[BWD_WORKLOADS[args.workload]]
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(_reference_line(args, world, BWD_METRIC, UNIT,
                                             bwd_config(args.workload, w, world, BWD_FLOP_FACTOR * w.flops()),
                                             lambda budget, _: cpu_baseline_bwd(w, budget_s=budget))))
        return 0
    from transformer_attention_gqa_b200 import replicas
    replicas.init("nccl", timeout_s=120)
    res = run_bwd(args, rank, world, local_rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline_bwd(w, budget_s=args.cpu_budget)
    replicas.shutdown()
    if rank == 0:
        print(json.dumps(res))
    return 0


# ------------------------------------------------------------------ QKV projection
# The projection with its RoPE epilogue for a forward workload's tokens and
# heads, hidden = n_q * d (the model width): one gqa_rope_attn_qkv_proj call
# per step, 2 * N * hidden * (n_q + 2 n_kv) * d FLOPs.
PROJ_WORKLOADS = {"qkv_llama8b": "llama8b", "qkv_nano": "nano"}
PROJ_METRIC = "GQA QKV projection + RoPE epilogue TFLOP/s on 1 B200; % of dense-BF16 tensor peak"


def _proj_shape(w):
    return w.n_q_heads * w.head_dim, (w.n_q_heads + 2 * w.n_kv_heads) * w.head_dim


def cpu_baseline_proj(w, inp, budget_s: float = 15.0):
    """Times the float64 oracle's projection, as it stands, on the first n
    tokens (n sized by a probe to about budget_s); returns TFLOP/s."""
    import oracle.gqa_oracle as orc

    C, F = _proj_shape(w)
    f, fk = w.n_q_heads * w.head_dim, w.n_kv_heads * w.head_dim
    W = inp.w_qkv

    def run(n):
        t0 = time.perf_counter()
        orc.qkv_rope_projection(inp.x[:n], W[:f], W[f:f + fk], W[f + fk:], w.n_q_heads, w.n_kv_heads, w.rope_theta,
                                positions=inp.positions[:n])
        return time.perf_counter() - t0

    n0 = min(w.total_tokens, 64)
    t0 = run(n0)
    n = int(max(n0, min(w.total_tokens, n0 * budget_s / max(t0, 1e-3))))
    dt = run(n)
    return {"value": 2.0 * n * C * F / dt / 1e12, "unit": UNIT, "cores": len(os.sched_getaffinity(0)),
            "kind": "oracle", "sample": f"first {n} tokens of {w.name} (hidden {C}, {F} output features), "
                                        f"float64 NumPy, {dt:.1f} s"}


def run_proj(args, rank, world, local_rank, inp):
    import torch
    import transformer_attention_gqa_b200 as g
    from transformer_attention_gqa_b200 import _abi, replicas, workloads as wl

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = wl.WORKLOADS[PROJ_WORKLOADS[args.workload]]
    C, F = _proj_shape(w)
    bf = torch.bfloat16
    x = torch.from_numpy(inp.x).to(bf).to(dev)
    wq = torch.from_numpy(inp.w_qkv).to(bf).to(dev)
    cu = torch.from_numpy(inp.cu_seqlens).to(dev)
    N = w.total_tokens
    q = torch.empty((N, w.n_q_heads, w.head_dim), dtype=bf, device=dev)
    k = torch.empty((N, w.n_kv_heads, w.head_dim), dtype=bf, device=dev)
    v = torch.empty_like(k)
    ws = g.Workspace(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        g.gqa_rope_attn_qkv_proj(x, wq, w.n_q_heads, w.n_kv_heads, w.rope_theta, cu_seqlens=cu, q=q, k=k, v=v,
                                 workspace=ws)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    assert g.get_device_status() == 0
    launches_per_step = _abi.last_launch_count()
    clocks = ClockSampler(local_rank)
    clocks.start()
    total_ms = _timed_steps(step, args.steps, stream, flush)
    table_ms, proj_ms = _library_kernel_ms(step, max(3, min(args.steps, 10)), flush)
    clk = clocks.stop()

    # end to end: x and cu_seqlens from pinned host memory every step (the
    # weights stay resident), q, k, v back
    ins = [(d_, d_.cpu().pin_memory()) for d_ in (x, cu)]
    outs = [(torch.empty(d_.shape, dtype=d_.dtype).pin_memory(), d_) for d_ in (q, k, v)]
    h2d, d2h = _nbytes(h_ for _, h_ in ins), _nbytes(h_ for h_, _ in outs)
    e2e_ms = _e2e_serial_ms(step, ins, outs, stream, max(3, min(args.steps, 10)))
    assert g.get_device_status() == 0
    assert torch.equal(outs[0][0], q.cpu())

    total_ms, e2e_ms, proj_ms, table_ms = replicas.max_over_ranks([total_ms, e2e_ms, proj_ms, table_ms], device=dev)
    flops = 2.0 * N * C * F
    ms_per_step = total_ms / args.steps
    value = flops * world / (ms_per_step * 1e-3) / 1e12
    peaks, src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    achieved = flops / (proj_ms * 1e-3) / 1e12
    res = {
        "metric": PROJ_METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": proj_config(args.workload, w, world),
        "pct_of_peak": round(100.0 * value / world / peak, 2),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": None,
                     "peak_source": f"{src} bf16_tflops (burst)", "kernel": "gqa_qkv_proj_kernel",
                     "kernel_ms": round(proj_ms, 4), "table_ms": round(table_ms, 4)},
        "e2e": {"value": round(flops * world / (e2e_ms * 1e-3) / 1e12, 2), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4)},
        "gpu_launches": launches_per_step * args.steps,
    }
    if clk:
        res["clocks"] = clk
    return res


def proj_config(name, w, world):
    C, F = _proj_shape(w)
    N = w.total_tokens
    return {"workload": name, "shape": w.description, "total_tokens": N, "hidden": C,
            "out_features": F, "n_q_heads": w.n_q_heads, "n_kv_heads": w.n_kv_heads,
            "head_dim": w.head_dim, "rope_theta": w.rope_theta, "flops_per_step": 2.0 * N * C * F,
            "parallelism": f"replicas x{world}",
            "l2": "256 MiB written before every timed step, outside the step's events"}


def main_proj(args, world, rank, local_rank):
    from transformer_attention_gqa_b200 import replicas, workloads as wl
    w = wl.WORKLOADS[PROJ_WORKLOADS[args.workload]]
    C, _ = _proj_shape(w)
    seed = w.seed if rank == 0 else replicas.replica_seed(w.seed, rank)
    inp = wl.make_projection_inputs(w.seq_lens, C, w.n_q_heads, w.n_kv_heads, w.head_dim, w.rope_theta, seed=seed)
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(_reference_line(args, world, PROJ_METRIC, UNIT, proj_config(args.workload, w, world),
                                             lambda budget, _: cpu_baseline_proj(w, inp, budget_s=budget))))
        return 0
    replicas.init("nccl", timeout_s=120)
    res = run_proj(args, rank, world, local_rank, inp)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline_proj(w, inp, budget_s=args.cpu_budget)
    replicas.shutdown()
    if rank == 0:
        print(json.dumps(res))
    return 0


# ------------------------------------------------------------------ masked forward
# The forward with an additive mask: a forward workload's shape, causal, with
# a seeded bf16 bias over every in-sequence (query, key) pair (N(0, 1) values,
# no hidden keys beyond the causal ones); one gqa_rope_attn_fwd_masked call
# per step, the forward's FLOP convention.
MASKED_WORKLOADS = {"masked_llama8b": "llama8b", "masked_nano": "nano"}
MASKED_METRIC = "causal GQA+RoPE attention fwd with an additive mask TFLOP/s on 1 B200; % of dense-BF16 tensor peak"


def _bench_mask(w, seed):
    from transformer_attention_gqa_b200 import workloads as wl

    Lm = max(w.seq_lens)
    Lp = (Lm + 7) // 8 * 8
    rng = np.random.default_rng(seed)
    return wl.to_bf16_values(rng.standard_normal((Lp, Lp), dtype=np.float32))


def cpu_baseline_masked(w, inp, mask, budget_s: float = 15.0, max_len: int = 2048):
    """Times the float64 oracle's masked forward, as it stands, on a prefix of
    the workload's first sequence (length sized by a probe to about
    budget_s); returns TFLOP/s by the forward's convention."""
    import oracle.gqa_oracle as orc

    first = int(inp.cu_seqlens[1])

    def run(L):
        t0 = time.perf_counter()
        orc.gqa_rope_attention_masked(inp.q[:L], inp.k[:L], inp.v[:L], [0, L], w.n_q_heads, w.n_kv_heads,
                                      w.rope_theta, mask, causal=True)
        return time.perf_counter() - t0

    L0 = min(first, 128)
    t0 = run(L0)
    L = int(max(L0, min(first, max_len, L0 * np.sqrt(max(budget_s, 0.1) / max(t0, 1e-3)))))
    dt = run(L)
    flops = 4.0 * L * L * w.head_dim * w.n_q_heads / 2.0
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
            "sample": f"first {L} tokens of {w.name}'s first sequence, all {w.n_q_heads} heads, float64 NumPy, "
                      f"{dt:.1f} s"}


def run_masked(args, rank, world, local_rank, inp, mask_np):
    import torch
    import transformer_attention_gqa_b200 as g
    from transformer_attention_gqa_b200 import _abi, replicas, workloads as wl

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = wl.WORKLOADS[MASKED_WORKLOADS[args.workload]]
    bf = torch.bfloat16
    q = torch.from_numpy(inp.q).to(bf).to(dev)
    k = torch.from_numpy(inp.k).to(bf).to(dev)
    v = torch.from_numpy(inp.v).to(bf).to(dev)
    cu = torch.from_numpy(inp.cu_seqlens).to(dev)
    mask = torch.from_numpy(mask_np).to(bf).to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((w.n_q_heads, w.total_tokens), dtype=torch.float32, device=dev)
    ws = g.Workspace(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        g.gqa_rope_attn_fwd_masked(q, k, v, cu, w.rope_theta, mask, causal=True, out=out, lse=lse, workspace=ws)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    assert g.get_device_status() == 0
    launches_per_step = _abi.last_launch_count()
    clocks = ClockSampler(local_rank)
    clocks.start()
    total_ms = _timed_steps(step, args.steps, stream, flush)
    prep_ms, attn_ms = _library_kernel_ms(step, max(3, min(args.steps, 10)), flush)
    clk = clocks.stop()

    # end to end: q, k, v and cu_seqlens from pinned host memory every step
    # (the mask stays resident), out and lse back
    ins = [(d_, d_.cpu().pin_memory()) for d_ in (q, k, v, cu)]
    outs = [(torch.empty(d_.shape, dtype=d_.dtype).pin_memory(), d_) for d_ in (out, lse)]
    h2d, d2h = _nbytes(h_ for _, h_ in ins), _nbytes(h_ for h_, _ in outs)
    e2e_ms = _e2e_serial_ms(step, ins, outs, stream, max(3, min(args.steps, 10)))
    assert g.get_device_status() == 0
    assert torch.equal(outs[0][0], out.cpu())

    total_ms, e2e_ms, attn_ms, prep_ms = replicas.max_over_ranks([total_ms, e2e_ms, attn_ms, prep_ms], device=dev)
    flops = w.flops()
    ms_per_step = total_ms / args.steps
    value = flops * world / (ms_per_step * 1e-3) / 1e12
    peaks, src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    achieved = flops / (attn_ms * 1e-3) / 1e12
    res = {
        "metric": MASKED_METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": masked_config(args.workload, w, world, mask_np.shape),
        "pct_of_peak": round(100.0 * value / world / peak, 2),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": None,
                     "peak_source": f"{src} bf16_tflops (burst)", "kernel": "gqa_attn_fwd_kernel (masked form)",
                     "kernel_ms": round(attn_ms, 4), "prologue_ms": round(prep_ms, 4)},
        "e2e": {"value": round(flops * world / (e2e_ms * 1e-3) / 1e12, 2), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4)},
        "gpu_launches": launches_per_step * args.steps,
    }
    if clk:
        res["clocks"] = clk
    return res


def masked_config(name, w, world, mask_shape):
    return {"workload": name, "shape": w.description, "total_tokens": w.total_tokens,
            "num_seqs": w.num_seqs, "n_q_heads": w.n_q_heads, "n_kv_heads": w.n_kv_heads,
            "head_dim": w.head_dim, "rope_theta": w.rope_theta, "causal": True,
            "mask": f"bf16 [{mask_shape[0]}, {mask_shape[1]}] seeded N(0, 1) bias",
            "flops_per_step": w.flops(), "parallelism": f"replicas x{world}",
            "l2": "256 MiB written before every timed step, outside the step's events"}


def main_masked(args, world, rank, local_rank):
    from transformer_attention_gqa_b200 import replicas, workloads as wl
    w = wl.WORKLOADS[MASKED_WORKLOADS[args.workload]]
    seed = w.seed if rank == 0 else replicas.replica_seed(w.seed, rank)
    inp = wl.make_inputs(w, seed=seed)
    mask = _bench_mask(w, seed + 1)
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(_reference_line(args, world, MASKED_METRIC, UNIT,
                                             masked_config(args.workload, w, world, mask.shape),
                                             lambda budget, _: cpu_baseline_masked(w, inp, mask, budget_s=budget))))
        return 0
    replicas.init("nccl", timeout_s=120)
    res = run_masked(args, rank, world, local_rank, inp, mask)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline_masked(w, inp, mask, budget_s=args.cpu_budget)
    replicas.shutdown()
    if rank == 0:
        print(json.dumps(res))
    return 0


# ------------------------------------------------------------------ GPU arm
SFU_EXP_PER_CLK_PER_SM = 16  # ex2 lanes per clock per SM (special-function unit)


def fwd_roofline(w, kernel_ms, peaks, src, clk, sm_count):
    """The attention kernel's binding roofline among three: dense bf16 tensor
    throughput (the metric's FLOPs), the special-function unit's exponentials
    (one per visible (query, key, head); 16 per clock per SM at the sampled
    SM clock) and HBM (q, k, v read, out and lse written once). The binding
    one is the slowest at its peak; frac = achieved / peak for it."""
    mhz = float((clk or {}).get("sm_mhz") or (clk or {}).get("sm_max_mhz") or 1965.0)
    t = kernel_ms * 1e-3
    cands = {
        "tensor": (w.flops() / 1e12, float(peaks["bf16_tflops"]), "TFLOP/s", f"{src} bf16_tflops (burst)"),
        "alu": (w.exps() / 1e9, SFU_EXP_PER_CLK_PER_SM * sm_count * mhz * 1e-3, "Gexp/s",
                f"SFU ex2 {SFU_EXP_PER_CLK_PER_SM}/clk/SM x {sm_count} SMs x {mhz:.0f} MHz"),
        "hbm": (w.io_bytes() / 1e9, float(peaks["hbm_gbs"]), "GB/s", f"{src} hbm_gbs"),
    }
    bound = max(cands, key=lambda k: cands[k][0] / cands[k][1])
    work, pk, unit, psrc = cands[bound]
    return {"bound": bound, "achieved": round(work / t, 2), "peak": round(pk, 1), "unit": unit,
            "frac": round(work / t / pk, 4), "peak_source": psrc,
            "others": {k: {"achieved": round(v[0] / t, 2), "peak": round(v[1], 1), "unit": v[2],
                           "frac": round(v[0] / t / v[1], 4)} for k, v in cands.items() if k != bound}}


# The forward on already rotated q and k (gqa_rope_attn_fwd_rotated): a
# forward workload's shape, its seeded N(0, 1) q and k taken as the rotated
# operands (a rotation keeps that distribution), the forward's FLOP count.
ROT_WORKLOADS = {"rot_llama8b": "llama8b", "rot_varlen": "varlen", "rot_qwen05b": "qwen05b", "rot_nano": "nano"}
ROT_METRIC = "causal GQA attention fwd on pre-rotated q/k TFLOP/s on 1 B200; % of dense-BF16 tensor peak"


def fwd_config(w, world, name=None):
    cfg = _fwd_config(w, world)
    if name is not None:
        cfg["workload"] = name
        cfg["inputs"] = "q and k taken as already rotated"
    return cfg


def _fwd_config(w, world):
    return {"workload": w.name, "shape": w.description, "total_tokens": w.total_tokens,
            "num_seqs": w.num_seqs, "n_q_heads": w.n_q_heads, "n_kv_heads": w.n_kv_heads,
            "head_dim": w.head_dim, "rope_theta": w.rope_theta, "causal": w.causal,
            "flops_per_step": w.flops(), "parallelism": f"replicas x{world}",
            "l2": "256 MiB written before every timed step, outside the step's events"}


def run_ours(args, rank, world, local_rank, rotated=False):
    import torch
    import transformer_attention_gqa_b200 as g
    from transformer_attention_gqa_b200 import _abi, replicas, workloads as wl

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = wl.WORKLOADS[ROT_WORKLOADS[args.workload] if rotated else args.workload]
    # every rank runs its own batch of the same shape (weak scaling)
    inp = wl.make_inputs(w, seed=w.seed if rank == 0 else replicas.replica_seed(w.seed, rank))
    dt = torch.float32 if w.io_dtype == "fp32" else torch.bfloat16
    q = torch.from_numpy(inp.q).to(dt).to(dev)
    k = torch.from_numpy(inp.k).to(dt).to(dev)
    v = torch.from_numpy(inp.v).to(dt).to(dev)
    cu = torch.from_numpy(inp.cu_seqlens).to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((w.n_q_heads, w.total_tokens), dtype=torch.float32, device=dev)
    ws = g.Workspace(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        if rotated:
            g.gqa_rope_attn_fwd_rotated(q, k, v, cu, causal=w.causal, out=out, lse=lse, workspace=ws)
        else:
            g.gqa_rope_attn_fwd(q, k, v, cu, w.rope_theta, causal=w.causal, out=out, lse=lse, workspace=ws)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    assert g.get_device_status() == 0
    launches_per_step = _abi.last_launch_count()

    barrier = replicas.barrier

    clocks = ClockSampler(local_rank)
    clocks.start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    t_wall = time.perf_counter()
    for i in range(args.steps):
        flush.zero_()  # L2 flush, outside the per-step events
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    wall = time.perf_counter() - t_wall
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = sum(step_ms)

    # per-kernel durations (second pass, same stream, events recorded by the library)
    from cuda.bindings import runtime as rt

    def _ev():
        err, e = rt.cudaEventCreate()
        assert int(err) == 0
        return e

    kern = []
    for i in range(max(3, min(args.steps, 10))):
        e = [_ev() for _ in range(3)]
        flush.zero_()
        _abi.set_profile_events(int(e[0]), int(e[1]), int(e[2]))
        step()
        kern.append(e)
    torch.cuda.synchronize()

    def _ms(a, b):
        err, ms = rt.cudaEventElapsedTime(a, b)
        assert int(err) == 0
        return float(ms)

    prep_ms = statistics.median(_ms(a, b) for a, b, _ in kern)
    attn_ms = statistics.median(_ms(b, c) for _, b, c in kern)
    for e in kern:
        for x in e:
            rt.cudaEventDestroy(x)
    clk = clocks.stop()

    # end to end through the public API with host buffers: every step copies
    # its q, k, v and cu_seqlens from pinned host memory, runs the call and
    # copies out and lse back. Prefill batches are independent, so steps
    # alternate between two streams with their own device buffers and
    # workspaces, as a serving loop would: one step's host-to-device copies
    # overlap the previous step's kernels and device-to-host copies.
    qh = torch.from_numpy(inp.q).to(dt).pin_memory()
    kh = torch.from_numpy(inp.k).to(dt).pin_memory()
    vh = torch.from_numpy(inp.v).to(dt).pin_memory()
    cuh = torch.from_numpy(inp.cu_seqlens).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh, cuh))
    d2h = out.numel() * out.element_size() + lse.numel() * lse.element_size()
    slots = []
    for _ in range(2):
        slots.append(dict(stream=torch.cuda.Stream(dev), q=torch.empty_like(q), k=torch.empty_like(k),
                          v=torch.empty_like(v), cu=torch.empty_like(cu), out=torch.empty_like(out),
                          lse=torch.empty_like(lse), ws=g.Workspace(dev),
                          outh=torch.empty(out.shape, dtype=out.dtype).pin_memory(),
                          lseh=torch.empty(lse.shape, dtype=lse.dtype).pin_memory()))

    def e2e_step(i):
        sl = slots[i % 2]
        with torch.cuda.stream(sl["stream"]):
            sl["q"].copy_(qh, non_blocking=True)
            sl["k"].copy_(kh, non_blocking=True)
            sl["v"].copy_(vh, non_blocking=True)
            sl["cu"].copy_(cuh, non_blocking=True)
            if rotated:
                g.gqa_rope_attn_fwd_rotated(sl["q"], sl["k"], sl["v"], sl["cu"], causal=w.causal, out=sl["out"],
                                            lse=sl["lse"], workspace=sl["ws"], stream=sl["stream"].cuda_stream)
            else:
                g.gqa_rope_attn_fwd(sl["q"], sl["k"], sl["v"], sl["cu"], w.rope_theta, causal=w.causal,
                                    out=sl["out"], lse=sl["lse"], workspace=sl["ws"],
                                    stream=sl["stream"].cuda_stream)
            sl["outh"].copy_(sl["out"], non_blocking=True)
            sl["lseh"].copy_(sl["lse"], non_blocking=True)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    e_steps = max(4, min(args.steps, 10))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    e0.record(stream)
    for sl in slots:
        sl["stream"].wait_event(e0)
    for i in range(e_steps):
        e2e_step(i)
    for sl in slots:
        done = torch.cuda.Event()
        done.record(sl["stream"])
        stream.wait_event(done)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e_steps
    assert g.get_device_status() == 0
    # the copied-back results of the last step match the device-timed path's
    assert torch.equal(slots[(e_steps - 1) % 2]["outh"], out.cpu())

    total_ms, e2e_ms, attn_ms, prep_ms = replicas.max_over_ranks([total_ms, e2e_ms, attn_ms, prep_ms], device=dev)

    flops = w.flops()
    ms_per_step = total_ms / args.steps
    value = flops * world / (ms_per_step * 1e-3) / 1e12
    peaks, src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    roof = fwd_roofline(w, attn_ms, peaks, src, clk, torch.cuda.get_device_properties(dev).multi_processor_count)
    res = {
        "metric": ROT_METRIC if rotated else METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": fwd_config(w, world, args.workload if rotated else None),
        "pct_of_peak": round(100.0 * value / world / peak, 2),
        "roofline": dict(roof, traffic=None if rotated or roof["bound"] != "tensor" else recorded_traffic(w.name),
                         kernel="gqa_attn_fwd_kernel", kernel_ms=round(attn_ms, 4), prologue_ms=round(prep_ms, 4)),
        "e2e": {"value": round(flops * world / (e2e_ms * 1e-3) / 1e12, 2), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4),
                "streams": 2, "note": "independent batches on two alternating streams: a step's host-to-device "
                                      "copies overlap the previous step's kernels and device-to-host copies"},
        "gpu_launches": launches_per_step * args.steps,
        "wall_s": round(wall, 4),
    }
    if clk:
        res["clocks"] = clk
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama8b")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    from transformer_attention_gqa_b200 import workloads as wl
    if args.workload in wl.DECODE_WORKLOADS:
        return main_decode(args, world, rank, local_rank)
    if args.workload in BWD_WORKLOADS:
        return main_bwd(args, world, rank, local_rank)
    if args.workload in PROJ_WORKLOADS:
        return main_proj(args, world, rank, local_rank)
    if args.workload in MASKED_WORKLOADS:
        return main_masked(args, world, rank, local_rank)
    rotated = args.workload in ROT_WORKLOADS
    w = wl.WORKLOADS[ROT_WORKLOADS[args.workload] if rotated else args.workload]
    metric = ROT_METRIC if rotated else METRIC
    cfg_name = args.workload if rotated else None

    if args.impl == "reference":
        if rank != 0:
            return 0
        per_step = []
        # every step: one oracle call on a random sample of rows, with 1-5 s
        # of per-row work beyond the call's fixed part (so the rate is not
        # that fixed part's), about a minute of per-row work in all
        for i in range(args.warmup):
            cpu_baseline(w, budget_s=0.5, seed_rows=1000 + i, beyond_fixed=True)
        info = None
        for i in range(args.steps):
            info = cpu_baseline(w, budget_s=max(1.0, min(5.0, 60.0 / max(args.steps, 1))), seed_rows=i,
                                beyond_fixed=True)
            per_step.append(info["value"])
        val = statistics.median(per_step)
        res = {"impl": "reference", "metric": metric, "value": round(val, 6), "unit": UNIT, "n_gpus": world,
               "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
               "vs_baseline": None, "dtype": "f64", "data": "synthetic",
               "config": fwd_config(w, world, cfg_name),
               "cpu_baseline": {"value": round(val, 6), "unit": UNIT, "cores": info["cores"], "kind": "oracle",
                                "sample": info["sample"]},
               "e2e": {"value": round(val, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(res))
        return 0

    from transformer_attention_gqa_b200 import replicas
    replicas.init("nccl", timeout_s=120)
    res = run_ours(args, rank, world, local_rank, rotated=rotated)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_budget)
    replicas.shutdown()
    if rank == 0:
        print(json.dumps(res))
    return 0


def main_decode(args, world, rank, local_rank):
    from transformer_attention_gqa_b200 import workloads as wl
    w = wl.DECODE_WORKLOADS[args.workload]
    if args.impl == "reference":
        if rank == 0:
            inp = wl.make_decode_inputs(w, nan_tail=False)
            print(json.dumps(_reference_line(args, world, DECODE_METRIC, DECODE_UNIT, decode_config(w, world),
                                             lambda budget, i: cpu_baseline_decode(w, inp, budget_s=budget, seed=i),
                                             digits=4)))
        return 0
    from transformer_attention_gqa_b200 import replicas
    replicas.init("nccl", timeout_s=120)
    res = run_decode(args, rank, world, local_rank)
    inp = res.pop("_inputs")
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline_decode(w, inp, budget_s=args.cpu_budget)
    replicas.shutdown()
    if rank == 0:
        print(json.dumps(res))
    return 0


if __name__ == "__main__":
    sys.exit(main())
