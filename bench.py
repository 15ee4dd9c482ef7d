"""Benchmark of the exact attention forward on B200: prefill TFLOP/s and decode HBM GB/s.

One step = one pass of the hot path over one batch of synthetic input.  The headline
("value", "roofline") times the long causal prefill (B=1, H=32, N=8192, d=128, bf16, bf16
O), one fa_fwd call per step.  The "configs" object, last in the line, gives every other
configuration one compact record (value, unit, ms_per_step, roofline fraction of the
measured burst peak "frac" and of the sustained peak "frac_sus", median SM clock); each is
timed for the line's own "steps":
  mha_d64       B=2 H=8 N=2048 d=64 fp16 causal (fa_fwd)
  noncausal_8k  B=1 H=32 N=8192 d=128 bf16 non-causal
  peaky_8k      the headline shape with Q drawn with std 4
  causal_16k    B=1 H=16 N=16384 d=128 bf16 causal
  causal_32k    B=1 H=16 N=32768 d=128 bf16 causal
  decode        B=16 H=32 Nq=1 Nkv=32768 d=128 bf16, split-KV decode (HBM GB/s)
  decode_paged  the decode shape in a paged cache of 64-key pages (fa_fwd_decode_paged)
  fp8_8k        the headline shape with E4M3 Q and K given (fa_fwd_fp8; peak: 4/3 of bf16)
  fp8q_8k       the same, Q and K quantised on the fly inside the step (fa_fwd_fp8_quant)
  bwd_8k        dQ, dK, dV of the headline shape (fa_bwd; 10*d FLOP per visible pair)
  varlen        a packed causal batch of 16 sequences, lengths log-uniform in [512, 8192]
  bwd_varlen    the backward of that packed batch (fa_bwd_varlen), 10*d FLOP per visible pair
Every configuration is timed for the same --steps.  Inputs are resident in HBM when the
timed region starts; a configuration whose inputs fit in L2 (126 MB) cycles through enough
copies of them that consecutive steps never find them there.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--skip-extra] [--detail out.json]

Multi-GPU (N > 1, one process per GPU via torch.distributed.run): every rank runs the
same independent problem (heads are independent; no collective on the data path);
timings are max over ranks, value = all ranks' FLOPs / that time (weak scaling).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_io_aware_59_b200 import binding  # noqa: E402
from exact_io_aware_59_b200.inputs import (WORKLOADS, Workload, make_grad_out,  # noqa: E402
                                           paged_decode_inputs, varlen_inputs, varlen_lengths,
                                           workload_qkv)

METRIC = "attention fwd TFLOP/s at 1 B200 (% of dense bf16 peak); decode HBM GB/s"
PREFILL = "long_prefill_causal"
DECODE = "decode"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------- accounting
def causal_pairs(Nq: int, Nkv: int) -> int:
    """Visible (query, key) pairs under the bottom-right causal mask."""
    off = Nkv - Nq
    total = 0
    # sum_i min(Nkv, max(0, i + off + 1)) in closed form by segments
    lo = max(0, -off)                       # first row that sees a key
    hi = min(Nq, Nkv - off)                 # rows [lo, hi) see i + off + 1 keys
    if hi > lo:
        total += (hi - lo) * (off + 1) + (hi - 1 + lo) * (hi - lo) // 2
    if Nq > max(hi, lo):
        total += (Nq - max(hi, lo)) * Nkv
    return total


def attention_flops(w: Workload) -> int:
    """4 * d per visible (query, key) pair: 2d for q.k and 2d for p*v; causal counts the
    visible lower triangle only."""
    pairs = causal_pairs(w.Nq, w.Nkv) if w.causal else w.Nq * w.Nkv
    return 4 * w.d * w.B * w.H * pairs


def backward_flops(w: Workload) -> int:
    """10 * d per visible (query, key) pair: five products (S, dP, dV, dK, dQ) of 2d each,
    2.5 times the forward's count."""
    pairs = causal_pairs(w.Nq, w.Nkv) if w.causal else w.Nq * w.Nkv
    return 10 * w.d * w.B * w.H * pairs


def algorithmic_bytes(w: Workload, o_bytes: int) -> int:
    """Read Q, K, V once; write O and LSE once."""
    BH = w.B * w.H
    return BH * (w.Nq * w.d * 2 + 2 * w.Nkv * w.d * 2 + w.Nq * w.d * o_bytes + w.Nq * 4)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            ident = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", ident, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.reader.join(timeout=2)

    def summary(self):
        rows = []
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 7:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), float(parts[2]), parts[3:]))
            except ValueError:
                continue
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, flag in enumerate(r[3])
                          if flag.lower() == "active"})
        busy = [r for r in rows if r[2] > 300.0] or rows
        return {"sm_mhz": statistics.median(r[0] for r in busy),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows), "samples_under_load": len(busy),
                "power_w_max": max(r[2] for r in rows)}


# ---------------------------------------------------------------- timing helpers
def dist_info():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, ws: int) -> float:
    """The largest of the ranks' x (a step time): NCCL on the GPUs, gloo on the host."""
    if ws == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, ms_max: float, ws: int) -> float:
    """Units all ranks processed per second: every rank runs the same independent
    problem, and the job takes as long as its slowest rank."""
    return units_per_rank * ws / (ms_max * 1e-3)


def time_steps(fn, steps: int, warmup: int, ws: int, stream) -> float:
    """Milliseconds per step over `steps` calls, CUDA events on the launch stream."""
    # The inputs were made on torch's default stream; the launch stream does not wait for
    # it by itself.
    torch.cuda.synchronize()
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        fn()
    end.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    return max_over_ranks(start.elapsed_time(end) / steps, ws)


def check(rc, where):
    if rc != binding.FA_OK:
        raise binding.FaError(rc, where)


def make_call(w: Workload, q, k, v, o, lse, stream):
    ic = binding.FA_BF16 if w.dtype == torch.bfloat16 else binding.FA_F16
    oc = binding._dtype_code(o.dtype)
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
            w.B, w.H, w.Nq, w.Nkv, w.d, float(w.softmax_scale), int(w.causal),
            stream.cuda_stream, ic, oc)

    def call():
        check(binding.fa_fwd(*args), "fa_fwd")

    return call


def run_e2e(w: Workload, tensors, steps, warmup, ws, stream):
    """The same call with pinned HOST inputs and results, pipelined as a serving loop runs
    it: step i uploads its Q/K/V on one copy stream, runs fa_fwd on the launch stream once
    they have landed, and downloads O and LSE on a second copy stream.  Two device buffer
    sets let step i+1's upload and step i-1's download overlap step i's kernel (the upload
    into a set waits for the kernel that last read it, the kernel for the download that
    last read its outputs).  Every step's copies are inside the timed region: the clock
    starts before step 0's upload and stops after the last step's download."""
    q, k, v, o, lse = tensors
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    hl = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    sets = [(q, k, v, o, lse), tuple(torch.empty_like(t) for t in (q, k, v, o, lse))]
    calls = [make_call(w, *sets[j], stream) for j in (0, 1)]
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in (0, 1)]    # set j's inputs have landed
    ev_done = [torch.cuda.Event() for _ in (0, 1)]  # the kernel on set j has finished
    ev_out = [torch.cuda.Event() for _ in (0, 1)]   # set j's results are on the host
    state = {"i": 0}

    def step():
        i = state["i"]
        j = i % 2
        sq, sk, sv, so, sl = sets[j]
        if i >= 2:
            up.wait_event(ev_done[j])
        with torch.cuda.stream(up):
            sq.copy_(hq, non_blocking=True)
            sk.copy_(hk, non_blocking=True)
            sv.copy_(hv, non_blocking=True)
        ev_in[j].record(up)
        stream.wait_event(ev_in[j])
        if i >= 2:
            stream.wait_event(ev_out[j])
        calls[j]()
        ev_done[j].record(stream)
        down.wait_event(ev_done[j])
        with torch.cuda.stream(down):
            ho.copy_(so, non_blocking=True)
            hl.copy_(sl, non_blocking=True)
        ev_out[j].record(down)
        state["i"] = i + 1

    torch.cuda.synchronize()
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(up)
    for _ in range(steps):
        step()
    end.record(down)
    torch.cuda.synchronize()
    barrier(ws)
    ms = max_over_ranks(start.elapsed_time(end) / steps, ws)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    d2h = ho.numel() * ho.element_size() + hl.numel() * hl.element_size()
    return ms, h2d, d2h


_HOST_INPUTS = {}


def cpu_baseline(w: Workload, budget_s: float, seed: int = 0):
    """The fp64 oracle, as it stands, on a bounded row sample of the workload; returns
    (TFLOP/s, threads, description, seconds).  Rows are drawn uniformly over heads and
    positions, so the causal FLOPs per row average those of the whole workload."""
    import numpy as np

    import oracle

    g = np.random.default_rng(seed)
    if w.name not in _HOST_INPUTS:
        _HOST_INPUTS[w.name] = workload_qkv(w, device="cpu")
    q, k, v = _HOST_INPUTS[w.name]
    threads = oracle.default_threads()
    n_total = w.B * w.H * w.Nq

    def row_flops(rows):
        i = rows % w.Nq
        vis = np.minimum(w.Nkv, np.maximum(0, i + (w.Nkv - w.Nq) + 1)) if w.causal else w.Nkv
        return int(4 * w.d * np.sum(vis))

    n = max(threads * 2, 16)
    while True:
        rows = np.sort(g.choice(n_total, size=min(n, n_total), replace=False))
        t0 = time.perf_counter()
        oracle.attention(q, k, v, w.softmax_scale, w.causal, rows=rows, nthreads=threads)
        dt = time.perf_counter() - t0
        if dt >= budget_s or len(rows) == n_total:
            break
        n = int(min(n_total, max(n * 2, n * budget_s / max(dt, 1e-3) * 1.1)))
    tflops = row_flops(rows) / dt / 1e12
    desc = (f"{len(rows)} of {n_total} query rows of {w.name}, drawn uniformly at random "
            f"(seed {seed}); {dt:.1f} s of CPU work")
    return tflops, threads, desc, dt


# ---------------------------------------------------------------- arms
def arm_reference(args, ws, rank):
    """The oracle, as it stands, on the host cores: each step a bounded row sample."""
    if rank != 0:
        return
    w = WORKLOADS[PREFILL]
    # Bounded sample per step so that the whole run stays within a few minutes.
    per_step = min(2.0, max(0.05, 90.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_baseline(w, per_step, seed=99)
    vals = []
    threads, desc, secs = 0, "", 0.0
    for s in range(args.steps):
        v, threads, desc, dt = cpu_baseline(w, per_step, seed=s)
        vals.append(v)
        secs += dt
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs * 1e3 / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, "fp64 oracle"),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads,
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(w: Workload, o_dtype: str):
    return {"workload": w.name, "B": w.B, "H": w.H, "Nq": w.Nq, "Nkv": w.Nkv, "d": w.d,
            "causal": w.causal, "in_dtype": str(w.dtype).replace("torch.", ""),
            "o_dtype": o_dtype, "parallelism": "independent problem per GPU",
            "l2": "inputs larger than L2 (no flush)"}


L2_BYTES = 126 * 1024 * 1024


def r4(x):
    """x to 4 significant digits (keeps the JSON line short)."""
    if x is None:
        return None
    return float(f"{x:.4g}")


def timed(calls, steps, warmup, ws, stream, local):
    """Times `steps` steps that cycle through `calls` (one call per step); returns
    (ms per step, clock summary).  Every call's kernel waits are checked afterwards."""
    state = {"i": 0}

    def step():
        calls[state["i"] % len(calls)]()
        state["i"] += 1

    with ClockSampler(local) as clk, torch.cuda.stream(stream):
        ms = time_steps(step, steps, warmup, ws, stream)
    assert binding.fa_device_status(clear=True) == 0, "a kernel wait timed out"
    return ms, clk.summary()


def compact(value, unit, ms, steps, frac, frac_sus, clk):
    """One record of the per-config object: the rate, its time, its roofline fractions."""
    del steps  # every configuration is timed for the line's own "steps"
    d = {"value": r4(value), "unit": unit, "ms_per_step": r4(ms), "frac": r4(frac)}
    if frac_sus is not None:
        d["frac_sus"] = r4(frac_sus)
    if clk:
        d["sm_mhz"] = int(round(clk["sm_mhz"]))
        # sw_power_cap is the normal state of a long dense run on a 1 kW part; any other
        # throttle reason is named
        other = [r for r in clk["reasons"] if r != "sw_power_cap"]
        if other:
            d["reasons"] = other
    return d


def input_sets(w: Workload, out_dtype):
    """Enough copies of the workload's inputs and outputs that one pass over them is larger
    than L2 (one copy when a single one already is): consecutive steps then never find
    their operands in L2.  Returns (list of (q, k, v, o, lse), bytes per copy)."""
    per = (w.B * w.H * (w.Nq + 2 * w.Nkv) * w.d * 2
           + w.B * w.H * w.Nq * (w.d * torch.empty((), dtype=out_dtype).element_size() + 4))
    n = 1 if per > L2_BYTES else min(64, -(-2 * L2_BYTES // per))
    sets = []
    for _ in range(n):
        q, k, v = workload_qkv(w, device="cuda")
        o = torch.empty((w.B, w.H, w.Nq, w.d), dtype=out_dtype, device="cuda")
        lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device="cuda")
        sets.append((q, k, v, o, lse))
    return sets, per


def prefill_record(w: Workload, args, ws, stream, local, peaks):
    """Times one fa_fwd per step on workload w (16-bit O); returns (compact record, ms,
    TFLOP/s of one GPU, clocks, the first input set)."""
    sets, _ = input_sets(w, w.dtype)
    calls = [make_call(w, *t, stream) for t in sets]
    ms, clk = timed(calls, args.steps, args.warmup, ws, stream, local)
    flops = attention_flops(w)
    tf = flops / (ms * 1e-3) / 1e12
    rec = compact(whole_job_rate(flops, ms, ws) / 1e12, "TFLOP/s", ms, args.steps,
                  tf / peaks["bf16_tflops"],
                  tf / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]), clk)
    return rec, ms, tf, clk, sets[0]


def arm_ours(args, ws, rank, local):
    torch.cuda.set_device(local)
    stream = torch.cuda.Stream()
    peaks, peak_src = load_peaks()
    peak_t = peaks["bf16_tflops"]
    peak_sus = peaks.get("bf16_tflops_sustained", peak_t)
    configs = {}
    detail = {}

    # prefill (headline): long causal, 16-bit O
    wp = WORKLOADS[args.prefill_workload]
    _, ms_p, tflops, clk, tensors = prefill_record(wp, args, ws, stream, local, peaks)
    flops = attention_flops(wp)
    value = whole_job_rate(flops, ms_p, ws) / 1e12
    traffic = DRAM_TRAFFIC.get((KERNEL_REV, wp.name))

    only = set(args.only.split(",")) if args.only else None

    def want(key):
        return not args.skip_extra and (only is None or key in only)

    # the other prefill configurations of the same kernel
    for key, name in (("mha_d64", "prefill_mha"), ("noncausal_8k", "long_prefill"),
                      ("peaky_8k", "long_prefill_peaky"), ("causal_16k", "long_ctx_16k"),
                      ("causal_32k", "long_ctx_32k")):
        if name == wp.name or not want(key):
            continue
        rec, ms, _, _, first = prefill_record(WORKLOADS[name], args, ws, stream, local,
                                              peaks)
        configs[key] = rec
        del first
        torch.cuda.empty_cache()

    # split-KV decode (HBM bound): one fa_fwd (split + combine kernels) per step
    wd = WORKLOADS[args.decode_workload]
    bytes_d = algorithmic_bytes(wd, 2)
    if want("decode"):
        sets, _ = input_sets(wd, wd.dtype)
        ms_d, clk_d = timed([make_call(wd, *t, stream) for t in sets], args.steps, args.warmup,
                            ws, stream, local)
        del sets
        gbs = bytes_d / (ms_d * 1e-3) / 1e9
        configs["decode"] = compact(whole_job_rate(bytes_d, ms_d, ws) / 1e9, "GB/s", ms_d,
                                    args.steps, gbs / peaks["hbm_gbs"], None, clk_d)
        detail["decode"] = {"algorithmic_bytes_per_launch": bytes_d, "gpu_launches": 2 * args.steps,
                            "traffic": DECODE_TRAFFIC.get((DECODE_REV, wd.name))}
        torch.cuda.empty_cache()

    if want("decode_paged"):
        # decode against a paged KV cache (same shape): 64-key pages, seeded random table
        ps = 64
        pq, kc, vc, table, sl = paged_decode_inputs(wd.B, wd.H, wd.Nkv, wd.d, ps, wd.dtype,
                                                    1000 * wd.index + 500, device="cuda")
        po = torch.empty((wd.B, wd.H, wd.d), dtype=wd.dtype, device="cuda")
        pl = torch.empty((wd.B, wd.H), dtype=torch.float32, device="cuda")
        pargs = (pq.data_ptr(), kc.data_ptr(), vc.data_ptr(), table.data_ptr(), sl.data_ptr(),
                 po.data_ptr(), pl.data_ptr(), wd.B, wd.H, wd.d, ps, table.shape[1], kc.shape[0],
                 float(wd.softmax_scale), stream.cuda_stream, binding._dtype_code(wd.dtype),
                 binding._dtype_code(wd.dtype), 0)
        ms_pd, clk_pd = timed([lambda: check(binding.fa_fwd_decode_paged(*pargs),
                                             "fa_fwd_decode_paged")],
                              args.steps, args.warmup, ws, stream, local)
        gbs_pd = bytes_d / (ms_pd * 1e-3) / 1e9
        configs["decode_paged"] = compact(whole_job_rate(bytes_d, ms_pd, ws) / 1e9, "GB/s", ms_pd,
                                          args.steps, gbs_pd / peaks["hbm_gbs"], None, clk_pd)
        del pq, kc, vc, table, sl, po, pl
        torch.cuda.empty_cache()

    q, k, v = tensors[0], tensors[1], tensors[2]
    if want("fp8_8k") and wp.d == 128:  # the FP8 path takes d = 128
        # headline shape with E4M3 queries and keys given as codes (quantised by torch with
        # per-tensor scales before the timed region); fp8q_8k below times the on-the-fly path
        q_s = float(q.abs().amax()) / 448.0
        k_s = float(k.abs().amax()) / 448.0
        q8 = (q.float() / q_s).to(torch.float8_e4m3fn).view(torch.uint8)
        k8 = (k.float() / k_s).to(torch.float8_e4m3fn).view(torch.uint8)
        o8 = torch.empty_like(tensors[3])
        l8 = torch.empty_like(tensors[4])
        fargs = (q8.data_ptr(), k8.data_ptr(), v.data_ptr(), o8.data_ptr(), l8.data_ptr(),
                 wp.B, wp.H, wp.Nq, wp.Nkv, wp.d, float(wp.softmax_scale), int(wp.causal),
                 stream.cuda_stream, q_s, k_s, binding._dtype_code(wp.dtype),
                 binding._dtype_code(o8.dtype))
        ms_f, clk_f = timed([lambda: check(binding.fa_fwd_fp8(*fargs), "fa_fwd_fp8")],
                            args.steps, args.warmup, ws, stream, local)
        tf_f = flops / (ms_f * 1e-3) / 1e12
        # Half the FLOPs (Q K^T) run at the E4M3 rate, nominally twice bf16; half (P V) at bf16.
        configs["fp8_8k"] = compact(whole_job_rate(flops, ms_f, ws) / 1e12, "TFLOP/s", ms_f,
                                    args.steps, tf_f / (peak_t * 4 / 3), tf_f / (peak_sus * 4 / 3),
                                    clk_f)
        del q8, k8, o8, l8
        torch.cuda.empty_cache()

    if want("fp8q_8k") and wp.d == 128:  # the FP8 path takes d = 128
        # the same with the quantisation inside the timed region: fa_fwd_fp8_quant takes the
        # bf16 Q and K and quantises them on the fly (one scale per 128-row tile)
        o8 = torch.empty_like(tensors[3])
        l8 = torch.empty_like(tensors[4])
        qargs = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o8.data_ptr(), l8.data_ptr(), wp.B,
                 wp.H, wp.Nq, wp.Nkv, wp.d, float(wp.softmax_scale), int(wp.causal),
                 stream.cuda_stream, binding._dtype_code(wp.dtype), binding._dtype_code(o8.dtype))
        ms_fq, clk_fq = timed([lambda: check(binding.fa_fwd_fp8_quant(*qargs), "fa_fwd_fp8_quant")],
                              args.steps, args.warmup, ws, stream, local)
        tf_fq = flops / (ms_fq * 1e-3) / 1e12
        configs["fp8q_8k"] = compact(whole_job_rate(flops, ms_fq, ws) / 1e12, "TFLOP/s", ms_fq,
                                     args.steps, tf_fq / (peak_t * 4 / 3),
                                     tf_fq / (peak_sus * 4 / 3), clk_fq)
        del o8, l8
        torch.cuda.empty_cache()

    if want("bwd_8k"):
        # backward (dQ, dK, dV) of the headline shape from its O and LSE and a seeded dO
        q, k, v, o, lse = tensors
        g = make_grad_out(wp.B, wp.H, wp.Nq, wp.d, wp.dtype, 1000 * wp.index + 3, device="cuda")
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        nws = binding.fa_bwd_workspace_bytes(wp.B, wp.H, wp.Nq, wp.d)
        bws = torch.empty(nws, dtype=torch.uint8, device="cuda")
        bargs = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                 g.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), bws.data_ptr(), nws,
                 wp.B, wp.H, wp.Nq, wp.Nkv, wp.d, float(wp.softmax_scale), int(wp.causal),
                 stream.cuda_stream, binding._dtype_code(wp.dtype))
        ms_b, clk_b = timed([lambda: check(binding.fa_bwd(*bargs), "fa_bwd")], args.steps,
                            args.warmup, ws, stream, local)
        flops_b = backward_flops(wp)
        tf_b = flops_b / (ms_b * 1e-3) / 1e12
        configs["bwd_8k"] = compact(whole_job_rate(flops_b, ms_b, ws) / 1e12, "TFLOP/s", ms_b,
                                    args.steps, tf_b / peak_t, tf_b / peak_sus, clk_b)
        detail["bwd_8k"] = {"traffic": BWD_TRAFFIC.get((BWD_REV, wp.name)),
                            "gpu_launches": 3 * args.steps, "flops_per_launch": flops_b}
        del g, dq, dk, dv, bws
        torch.cuda.empty_cache()

    if want("varlen") or want("bwd_varlen"):
        # packed variable-length prefill: a ragged causal batch
        lens = varlen_lengths(16, 512, 8192, 4242)
        Hv, dv_ = 32, 128
        vq, vk, vv, vcu = varlen_inputs(lens, Hv, dv_, torch.bfloat16, 8000, device="cuda")
        vo = torch.empty_like(vq)
        vlse = torch.empty((vq.shape[0], Hv), dtype=torch.float32, device="cuda")
        vargs = (vq.data_ptr(), vk.data_ptr(), vv.data_ptr(), vo.data_ptr(), vlse.data_ptr(),
                 vcu.data_ptr(), vcu.data_ptr(), len(lens), Hv, vq.shape[0], vk.shape[0],
                 max(lens), max(lens), dv_, float(dv_ ** -0.5), 1, stream.cuda_stream,
                 binding.FA_BF16, binding.FA_BF16)
        if want("varlen"):
            ms_v, clk_v = timed([lambda: check(binding.fa_fwd_varlen(*vargs), "fa_fwd_varlen")],
                                args.steps, args.warmup, ws, stream, local)
            flops_v = sum(4 * dv_ * Hv * causal_pairs(n, n) for n in lens)
            tf_v = flops_v / (ms_v * 1e-3) / 1e12
            configs["varlen"] = compact(whole_job_rate(flops_v, ms_v, ws) / 1e12, "TFLOP/s", ms_v,
                                        args.steps, tf_v / peak_t, tf_v / peak_sus, clk_v)
        if want("bwd_varlen"):
            # the backward of the same packed batch (fa_bwd_varlen), from the forward's O, LSE
            check(binding.fa_fwd_varlen(*vargs), "fa_fwd_varlen")
            vg = make_grad_out(1, vq.shape[0], Hv, dv_, torch.bfloat16, 8003, device="cuda")
            vg = vg.reshape(vq.shape)
            vdq, vdk, vdv = torch.empty_like(vq), torch.empty_like(vk), torch.empty_like(vv)
            nvw = binding.fa_bwd_varlen_workspace_bytes(len(lens), Hv, vq.shape[0], max(lens), dv_)
            vws = torch.empty(nvw, dtype=torch.uint8, device="cuda")
            bvargs = (vq.data_ptr(), vk.data_ptr(), vv.data_ptr(), vo.data_ptr(), vlse.data_ptr(),
                      vg.data_ptr(), vdq.data_ptr(), vdk.data_ptr(), vdv.data_ptr(), vws.data_ptr(),
                      nvw, vcu.data_ptr(), vcu.data_ptr(), len(lens), Hv, vq.shape[0],
                      vk.shape[0], max(lens), max(lens), dv_, float(dv_ ** -0.5), 1,
                      stream.cuda_stream, binding.FA_BF16)
            ms_bv, clk_bv = timed([lambda: check(binding.fa_bwd_varlen(*bvargs), "fa_bwd_varlen")],
                                  args.steps, args.warmup, ws, stream, local)
            flops_bv = sum(10 * dv_ * Hv * causal_pairs(n, n) for n in lens)
            tf_bv = flops_bv / (ms_bv * 1e-3) / 1e12
            configs["bwd_varlen"] = compact(whole_job_rate(flops_bv, ms_bv, ws) / 1e12, "TFLOP/s",
                                            ms_bv, args.steps, tf_bv / peak_t, tf_bv / peak_sus,
                                            clk_bv)
            del vg, vdq, vdk, vdv, vws
        del vq, vk, vv, vcu, vo, vlse
        torch.cuda.empty_cache()

    # end to end through the C ABI with host buffers
    e2e = None
    if not args.skip_e2e:
        ms_e, h2d, d2h = run_e2e(wp, tensors, args.steps, args.warmup, ws, stream)
        e2e = {"value": r4(whole_job_rate(flops, ms_e, ws) / 1e12), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": r4(ms_e),
               "steps": args.steps, "copies": "pipelined: 2 buffer sets, upload and download streams"}
    del tensors

    cpu = None
    if rank == 0 and ws == 1 and not args.skip_cpu:
        v, threads, desc, _ = cpu_baseline(wp, args.cpu_seconds)
        cpu = {"value": r4(v), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_p,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": workload_config(wp, "bf16"),
            "gpu_launches": args.steps,
            "roofline": {"bound": "tensor", "achieved": r4(tflops), "peak": peak_t,
                         "unit": "TFLOP/s", "frac": r4(tflops / peak_t), "traffic": traffic,
                         "peak_source": f"{peak_src} bf16 burst",
                         "flops_per_launch": flops, "frac_sus": r4(tflops / peak_sus)},
            "clocks": clk,
            "e2e": e2e,
            "cpu_baseline": cpu,
            # every other configuration, last, so that the end of the line holds all of it
            "configs": configs,
        }
        if args.detail:
            with open(args.detail, "w") as f:
                json.dump({"line": line, "detail": detail, "peaks": peaks}, f, indent=1)
        print(json.dumps(line, separators=(",", ":")), flush=True)


# Bumped whenever the backward main kernel changes, so stale ncu traffic is not reported.
BWD_REV = "backward-v6"
# dram__bytes_read.sum + dram__bytes_write.sum of one fa_bwd_sm100 launch at full size
# (ncu; profiles/fa_bwd_sm100_long_prefill_causal.md).
BWD_TRAFFIC = {("backward-v6", "long_prefill_causal"): 629.2e6}

# Bumped whenever the prefill kernel changes, so stale ncu traffic is not reported.
KERNEL_REV = "prefill-v24"
# dram__bytes_read.sum + dram__bytes_write.sum per launch from one ncu capture of the
# kernel at this revision (profiles/fa_prefill_sm100_<workload>.md).
DRAM_TRAFFIC = {("prefill-v24", "long_prefill_causal"): 583.9e6}
# The decode kernel's traffic per launch, taken on decode_4k (B16 H32 Nkv4096: 1.0816 GB)
# and scaled by the keys streamed (x8 for Nkv 32768): the kernel reads each key once.
DECODE_REV = "decode-v2"
DECODE_TRAFFIC = {("decode-v2", "decode"): 8 * 1.0799e9}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--prefill-workload", default=PREFILL, choices=sorted(WORKLOADS))
    ap.add_argument("--decode-workload", default=DECODE, choices=sorted(WORKLOADS))
    ap.add_argument("--skip-extra", action="store_true",
                    help="time the headline prefill only")
    ap.add_argument("--detail", default=None, help="also write a detailed JSON record here")
    ap.add_argument("--only", default=None,
                    help="comma-separated configs to time besides the headline (default: all)")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    ws, rank, local = dist_info()
    if ws > 1:
        import datetime

        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if args.impl == "reference":
            arm_reference(args, ws, rank)
        else:
            arm_ours(args, ws, rank, local)
    finally:
        if ws > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
