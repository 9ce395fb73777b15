#!/usr/bin/env python
"""Benchmark of the attention-with-KV-cache hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--sub LIST]
                    [--impl ours|reference]

One step = one library call over one batch of seeded synthetic input resident
in HBM.  The default line is the headline prefill workload, MLA-like causal
attention (bf16, batch 4, 16 heads, 4096 query and key rows, d_qk 192,
d_v 128; flash-attention PR #1604's head dims), in TFLOP/s of algorithmic
FLOPs against the dense bf16 tensor peak.  Beside it, under "decode", the
line carries one sub-record per decode workload (the MLA decode over a
16384-row cache and the GQA decode with RoPE, bf16, 32 query / 8 kv heads,
cache_seqlens ~ U{1024..8000}), each in HBM GB/s of algorithmic bytes
against the copy bandwidth.  --config picks another headline workload (then
no sub-records unless --sub names some); --sub none drops them.

Timing: W untimed warm-up steps, then K steps, each timed with CUDA events on
the launching stream around a CUDA-graph replay of the call; L2 is flushed
before every timed step, outside the events.  The roofline object divides the
algorithmic amount by the attention kernel's own event-timed duration, and
takes the burst peak of MEASURED_PEAKS.json for a tensor-bound kernel (each
launch is timed alone, after an idle L2 flush); power-cap throttling seen on
the clocks is reported beside it.  Multi-GPU runs (torchrun, one rank per
GPU) give every rank its own full copy of the workload (weak scaling, no
collective on the data path) and report the max over ranks.

--impl reference times the float64 CPU oracle (the correctness reference of
the tests, not tuned for speed) on a bounded sample of the headline
workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "prefill attention TFLOP/s and decode KV-cache GB/s on 1 B200, % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Nominal B200 figures (HGX HBM3e bandwidth; dense bf16/fp16 tensor rate, no sparsity), reported beside
# the measured peaks as a second ceiling.
SPEC_PEAKS = {"hbm": (7700.0, "GB/s"), "tensor": (2250.0, "TFLOP/s")}
DEFAULT_CONFIG = "mla-prefill"
# decode workloads reported beside the default headline
DEFAULT_SUBS = ("mla-decode", "gqa-decode")


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(W.CONFIGS))
    ap.add_argument("--sub", default=None,
                    help="comma-separated workloads reported as 'decode' sub-records ('none' for none; "
                         "default: mla-decode,gqa-decode beside the default headline, none otherwise)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="CPU time budget of the oracle sample (cpu_baseline / reference arm)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg (profiling runs)")
    return ap.parse_args(argv)


def is_decode(w: W.Workload) -> bool:
    return w.mode == "kvcache" and w.s_q <= 8


def work_units(w: W.Workload, seqlens):
    """(algorithmic amount per step, unit, bound) for the workload."""
    if w.mode == "rotary":
        return W.rotary_bytes(w) / 1e9, "GB/s", "hbm"
    if is_decode(w):
        return W.kvcache_bytes(w, seqlens) / 1e9, "GB/s", "hbm"
    return W.flops(w, seqlens) / 1e12, "TFLOP/s", "tensor"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- traffic record
def traffic_record(config_key: str, kernel_tag: str):
    """DRAM traffic per launch of the attention kernel on this workload, from
    the committed ncu summary profiles/traffic_<workload>.md, if it was taken
    on the current kernel source (its sha256 prefix must match)."""
    src = {"decode": "decode.cu", "prefill": "prefill_sm100.cu", "rotary": "rotary.cu",
           "backward": "backward.cu"}.get(kernel_tag)
    summ = os.path.join(ROOT, "profiles", f"traffic_{config_key}.md")
    if not src or not os.path.exists(summ):
        return None
    path = os.path.join(ROOT, "rotary_embedding_b200", "csrc", src)
    if not os.path.exists(path):
        return None
    sha = hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]
    text = open(summ).read()
    m = re.search(r"source_file:\s*(\S+).*?source_sha256_16:\s*([0-9a-f]{16}).*?"
                  r"traffic_bytes_per_launch_full_size:\s*([0-9.eE+]+)", text, re.S)
    if not m or m.group(1) != src or m.group(2) != sha:
        return None
    return float(m.group(3))


# ----------------------------------------------------------------------------- our arm
def make_step(w, inp_dev, fa):
    """(step, plan, outputs): `step` enqueues one library call on the current
    stream; `outputs` are the tensors it writes (None entries are skipped)."""
    if w.mode == "bwd":
        q, k, v, dout = (inp_dev[n] for n in ("q", "k", "v", "dout"))
        if "out" not in inp_dev:
            # the forward's out and lse, made once outside every timed region
            inp_dev["out"], inp_dev["lse"] = fa.fa_fwd(q, k, v, causal=w.causal, softmax_scale=w.scale or None,
                                                       window=w.window)
        out, lse = inp_dev["out"], inp_dev["lse"]
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(max(fa.fa_bwd_workspace_size(q), 1), dtype=torch.uint8, device=q.device)

        def step():
            fa.fa_bwd(q, k, v, out, dout, lse, causal=w.causal, softmax_scale=w.scale or None, window=w.window,
                      dq=dq, dk=dk, dv=dv, workspace=ws)
        plan = {"path": 0, "launches": 3, "n_splits": 1, "chunk": 0, "workspace_bytes": ws.numel()}
        return step, plan, (dq, dk, dv)
    if w.mode == "varlen":
        q, k, v, cu = inp_dev["q"], inp_dev["k"], inp_dev["v"], inp_dev["cu_seqlens"]
        out = torch.empty((q.shape[0], q.shape[1], v.shape[2]), dtype=q.dtype, device=q.device)
        lse = torch.empty((q.shape[1], q.shape[0]), dtype=torch.float32, device=q.device)

        def step():
            fa.fa_fwd_varlen(q, k, v, cu, cu, w.s_q, causal=w.causal, softmax_scale=w.scale or None,
                             window=w.window, out=out, lse=lse)
        plan = {"path": fa.FA_PATH_DENSE, "launches": 1, "n_splits": 1, "chunk": 0, "workspace_bytes": 0}
        return step, plan, (out, lse)
    if w.mode == "rotary":
        x, offs = inp_dev["q"], inp_dev["cache_seqlens"]
        out = torch.empty_like(x)

        def step():
            fa.fa_rotary(x, inp_dev["cos"], inp_dev["sin"], offs, w.rotary_dim, w.interleaved, w.conjugate,
                         out=out)
        plan = {"path": 0, "launches": 1, "n_splits": 1, "chunk": 0, "workspace_bytes": 0}
        return step, plan, (out, None)
    if w.mode == "dense":
        q, k, v = inp_dev["q"], inp_dev["k"], inp_dev["v"]
        out = torch.empty(q.shape[:3] + (w.d_v,), dtype=q.dtype, device=q.device)
        lse = torch.empty((w.batch, w.h_q, w.s_q), dtype=torch.float32, device=q.device)

        def step():
            fa.fa_fwd(q, k, v, causal=w.causal, softmax_scale=w.scale or None, out=out, lse=lse, window=w.window)
        plan = fa.fa_fwd_plan(q, k, v)
        return step, plan, (out, lse)
    d = inp_dev
    out = torch.empty((w.batch, w.s_q, w.h_q, w.d_v), dtype=d["q"].dtype, device=d["q"].device)
    lse = torch.empty((w.batch, w.h_q, w.s_q), dtype=torch.float32, device=d["q"].device)
    ws_bytes = fa.fa_kvcache_workspace_size(d["q"], d["k_cache"], d["v_cache"], d["k_new"], w.rotary_dim)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=d["q"].device)
    seq = d["cache_seqlens"] if not w.seqlens_scalar else int(d["cache_seqlens"][0].item())

    def step():
        fa.fa_kvcache_fwd(d["q"], d["k_cache"], d["v_cache"], d["k_new"], d["v_new"], d.get("cos"),
                          d.get("sin"), cache_seqlens=seq, rotary_dim=w.rotary_dim or None,
                          rotary_interleaved=w.interleaved, causal=w.causal,
                          softmax_scale=w.scale or None, out=out, lse=lse, workspace=ws)
    plan = fa.fa_kvcache_plan(d["q"], d["k_cache"], d["v_cache"], d["k_new"], w.rotary_dim)
    return step, plan, (out, lse)


class L2Flush:
    """Evicts L2 between timed steps (untimed): a 512 MiB write, then a
    256 MiB read of another buffer, so that L2 holds neither the step's data
    nor dirty lines whose write-back would land inside the next step."""

    def __init__(self, device):
        self.wbuf = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=device)
        self.rbuf = torch.zeros(64 * 1024 * 1024, dtype=torch.float32, device=device)
        self.out = torch.empty((), dtype=torch.float32, device=device)

    def zero_(self):
        self.wbuf.zero_()
        torch.sum(self.rbuf, dim=None, out=self.out)


def time_steps(step, steps, warmup, stream, flush_buf, barrier):
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    barrier()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for i in range(steps):
        flush_buf.zero_()
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    barrier()
    return [s.elapsed_time(e) for s, e in zip(starts, ends)]


def time_e2e(w, inp_host, inp_dev, step_fn_factory, steps, warmup, stream, flush_buf, barrier):
    """End-to-end through the public API: per step, copy the step's inputs from
    pinned host memory, run the call, read out + lse back to pinned host memory."""
    names = {"dense": ["q", "k", "v"], "rotary": ["q", "cache_seqlens"],
             "varlen": ["q", "k", "v", "cu_seqlens"], "bwd": ["q", "k", "v", "out", "dout", "lse"]}.get(
        w.mode, ["q", "k_new", "v_new", "cache_seqlens"])
    pinned = {n: inp_host[n].pin_memory() for n in names}
    step, _, outs = step_fn_factory()
    outs = [t for t in outs if t is not None]
    outs_h = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs]
    h2d = sum(t.numel() * t.element_size() for t in pinned.values())
    d2h = sum(t.numel() * t.element_size() for t in outs_h)

    def e2e_step():
        for n in names:
            inp_dev[n].copy_(pinned[n], non_blocking=True)
        step()
        for t, th in zip(outs, outs_h):
            th.copy_(t, non_blocking=True)
    times = time_steps(e2e_step, steps, warmup, stream, flush_buf, barrier)
    return times, h2d, d2h


def cpu_sample(w, inp, budget_s):
    """Time the float64 oracle on successive batch entries of the workload until
    the budget is spent; returns (amount processed in the metric's unit numerator,
    seconds, description)."""
    import oracle
    t_total, amount, done = 0.0, 0.0, []
    b = 0
    while not done or (t_total < budget_s and len(done) < 4 * w.batch):
        bi = b % w.batch
        if w.mode == "varlen":
            # one (sequence, head) pair, every query row
            cu = inp["cu_seqlens"]
            h = (b // w.batch) % w.h_q
            q0, q1 = int(cu[bi]), int(cu[bi + 1])
            hk = h // (w.h_q // w.h_kv)
            q = inp["q"][None, q0:q1, h:h + 1].double().numpy()
            k = inp["k"][None, q0:q1, hk:hk + 1].double().numpy()
            v = inp["v"][None, q0:q1, hk:hk + 1].double().numpy()
            t0 = time.perf_counter()
            oracle.fwd(q, k, v, causal=w.causal, scale=w.softmax_scale(), window=w.window)
            dt = time.perf_counter() - t0
            amount += W.flops(w.scaled(mode="dense", batch=1, h_q=1, h_kv=1, s_q=q1 - q0, s_k=q1 - q0)) / 1e12
            done.append(f"s{bi}h{h}")
        elif w.mode == "rotary":
            # 64 rows of one batch entry, every head
            i0 = (b // w.batch) * 64 % w.s_q
            x = inp["q"][bi:bi + 1, i0:i0 + 64].double().numpy()
            cs, sn = inp["cos"].double().numpy(), inp["sin"].double().numpy()
            t0 = time.perf_counter()
            oracle.rotary(x, cs, sn, int(inp["cache_seqlens"][bi]) + i0, w.rotary_dim, w.interleaved,
                          w.conjugate, fmt=w.dtype)
            dt = time.perf_counter() - t0
            amount += W.rotary_bytes(w.scaled(batch=1, s_q=x.shape[1])) / 1e9
            done.append(f"b{bi}rows{i0}")
        elif w.mode == "bwd":
            # one (batch, head) pair, every query and key row
            h = (b // w.batch) % w.h_q
            hk = h // (w.h_q // w.h_kv)
            q = inp["q"][bi:bi + 1, :, h:h + 1].double().numpy()
            k = inp["k"][bi:bi + 1, :, hk:hk + 1].double().numpy()
            v = inp["v"][bi:bi + 1, :, hk:hk + 1].double().numpy()
            do = inp["dout"][bi:bi + 1, :, h:h + 1].double().numpy()
            t0 = time.perf_counter()
            oracle.bwd(q, k, v, do, causal=w.causal, scale=w.softmax_scale(), window=w.window)
            dt = time.perf_counter() - t0
            amount += W.flops(w.scaled(batch=1, h_q=1, h_kv=1)) / 1e12
            done.append(f"b{bi}h{h}")
        elif w.mode == "dense":
            # one (batch, head) pair, every query row
            h = (b // w.batch) % w.h_q
            q = inp["q"][bi:bi + 1, :, h:h + 1].double().numpy()
            hk = h // (w.h_q // w.h_kv)
            k = inp["k"][bi:bi + 1, :, hk:hk + 1].double().numpy()
            v = inp["v"][bi:bi + 1, :, hk:hk + 1].double().numpy()
            t0 = time.perf_counter()
            oracle.fwd(q, k, v, causal=w.causal, scale=w.softmax_scale(), window=w.window)
            dt = time.perf_counter() - t0
            sub = w.scaled(batch=1, h_q=1, h_kv=1)
            amount += W.flops(sub) / 1e12
            done.append(f"b{bi}h{h}")
        else:
            L = int(inp["cache_seqlens"][bi])
            n = L + w.s_q
            args = [inp["q"][bi:bi + 1], inp["k_cache"][bi:bi + 1, :n], inp["v_cache"][bi:bi + 1, :n],
                    inp["k_new"][bi:bi + 1], inp["v_new"][bi:bi + 1]]
            args = [a.double().numpy() for a in args]
            cs = inp["cos"].double().numpy() if "cos" in inp else None
            sn = inp["sin"].double().numpy() if "sin" in inp else None
            t0 = time.perf_counter()
            oracle.kvcache_fwd(*args, cs, sn, [L], rotary_dim=w.rotary_dim, interleaved=w.interleaved,
                               causal=w.causal, scale=w.softmax_scale(), fmt=w.dtype)
            dt = time.perf_counter() - t0
            sub = w.scaled(batch=1)
            amount += (W.kvcache_bytes(sub, [L]) / 1e9 if is_decode(w) else W.flops(sub, [L]) / 1e12)
            done.append(f"b{bi}")
        t_total += dt
        b += 1
    unit_desc = {"dense": "(batch, head) pairs", "bwd": "(batch, head) pairs", "rotary": "64-row blocks (all heads)",
                 "varlen": "(sequence, head) pairs"}.get(w.mode, "batch entries")
    desc = (f"float64 oracle, single thread, on {len(done)} {unit_desc} of the workload "
            f"({', '.join(done[:8])}{'...' if len(done) > 8 else ''}); inputs converted to float64 "
            f"outside the timed region")
    return amount, t_total, desc


def cpu_model() -> str:
    """The host CPU's model name (for the oracle baseline's record)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def aggregate_over_ranks(ms_local: float, amount: float, world: int, device):
    """Whole-job throughput: every rank processed `amount` units in its own
    device time; the job takes the slowest rank's time (max over ranks)."""
    ms_max = ms_local
    if world > 1:
        import torch.distributed as dist
        t = torch.tensor([ms_local], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_max = float(t.item())
    return ms_max, world * amount / (ms_max / 1e3)


def time_kernel(fa, step, steps, flush_buf):
    """Per-step duration (ms) of the attention kernel alone: CUDA events that
    the library records on the launching stream right before and after that
    kernel (fa_set_kernel_events), replayed from a CUDA graph so that no host
    latency sits between the start event and the launch; L2 flushed before
    every step.  None if the events cannot be timed."""
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    fa.fa_set_kernel_events(start, stop)
    try:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, capture_error_mode="relaxed"):
            step()
    finally:
        fa.fa_set_kernel_events()
    torch.cuda.synchronize()
    try:
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        times = []
        for _ in range(steps):
            flush_buf.zero_()
            graph.replay()
            torch.cuda.synchronize()
            times.append(start.elapsed_time(stop))
    except RuntimeError:
        return None
    return times


def sub_names(args):
    """Workloads reported as sub-records beside the headline."""
    if args.sub is None:
        return list(DEFAULT_SUBS) if args.config == DEFAULT_CONFIG else []
    if args.sub.strip().lower() in ("", "none"):
        return []
    names = [n.strip() for n in args.sub.split(",") if n.strip()]
    for n in names:
        if n not in W.CONFIGS:
            raise SystemExit(f"--sub: unknown workload {n!r}")
    return names


def measure(name, args, fa, device, world, barrier, peaks, peaks_src):
    """Time one workload: the whole call (graph replay, L2 flushed per step),
    the attention kernel alone (library events) and the end-to-end API leg.
    Every rank runs the same steps and the same collectives in the same order.
    Returns (record, clocks, w, inp, amount, unit)."""
    w = W.CONFIGS[name]
    inp = W.make_inputs(w, seed=0)
    inp_dev = {k: v.to(device) for k, v in inp.items()}
    seqlens = (inp["cache_seqlens"].tolist() if w.mode == "kvcache"
               else (inp["cu_seqlens"].diff().tolist() if w.mode == "varlen" else None))
    amount, unit, bound = work_units(w, seqlens)
    stream = torch.cuda.current_stream(device)
    flush_buf = L2Flush(device)

    step, plan, _ = make_step(w, inp_dev, fa)
    if w.mode == "bwd":
        # the end-to-end leg copies the forward's results in from the host too
        inp["out"], inp["lse"] = inp_dev["out"].cpu(), inp_dev["lse"].cpu()
    # The timed step replays a CUDA graph of the library call, so the host's
    # Python/ctypes overhead is not inside the device-timed region.
    step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="relaxed"):
        step()
    torch.cuda.synchronize()
    with ClockSampler(device.index) as clk:
        # untimed soak so the clock sampler sees the GPU under this load
        t_end = time.perf_counter() + 1.5
        while time.perf_counter() < t_end:
            for _ in range(20):
                graph.replay()
            torch.cuda.synchronize()
        times = time_steps(graph.replay, args.steps, max(args.warmup, 3), stream, flush_buf, barrier)
        k_times = time_kernel(fa, step, args.steps, flush_buf)
    ms = sum(times) / len(times)
    kernel_ms = sum(k_times) / len(k_times) if k_times else None
    ms_max, value = aggregate_over_ranks(ms, amount, world, device)
    # every rank takes part in the reduction, with -1 where its kernel events could not be timed
    kms_max = aggregate_over_ranks(kernel_ms if kernel_ms else -1.0, amount, world, device)[0]
    kms_max = kms_max if kms_max > 0 else None

    e2e_value, h2d, d2h = None, 0, 0
    if not args.no_e2e:
        e2e_times, h2d, d2h = time_e2e(w, inp, inp_dev, lambda: make_step(w, inp_dev, fa), args.steps,
                                       max(args.warmup, 3), stream, flush_buf, barrier)
        e_ms = sum(e2e_times) / len(e2e_times)
        _, e2e_value = aggregate_over_ranks(e_ms, amount, world, device)
        e2e_value = round(e2e_value, 3)

    clocks = clk.summary()
    # A tensor-bound kernel takes the burst cuBLAS figure: each launch is
    # timed alone, after an idle L2 flush, like the burst measurement.  The
    # power cap, when the sampled clocks show it, is reported as a note.
    peak_key = "hbm_gbs" if bound == "hbm" else "bf16_tflops"
    peak = float(peaks.get(peak_key, FALLBACK_PEAKS[peak_key]))
    # algorithmic amount of one call / the attention kernel's own duration
    # (the whole call's duration if the kernel events could not be timed)
    achieved = amount / ((kms_max if kms_max else ms_max) / 1e3)
    kernel_tag = "rotary" if w.mode == "rotary" else ("decode" if plan["path"] == fa.FA_PATH_DECODE else "prefill")
    kernel_name = {fa.FA_PATH_DECODE: "decode_kernel", fa.FA_PATH_PREFILL: "prefill2_kernel / prefill_kernel",
                   fa.FA_PATH_DENSE: "prefill2_kernel / prefill_kernel"}.get(plan["path"], "rotary_kernel")
    if w.mode == "bwd":
        kernel_tag, kernel_name = "backward", "bwd_dkdv_kernel + bwd_dq_kernel"
    capped = bool(clocks) and "sw_power_cap" in clocks.get("reasons", [])
    rec = {
        "workload": w.name,
        "value": round(value, 3),
        "unit": unit,
        "ms_per_step": round(ms_max, 5),
        "dtype": w.dtype,
        "config": {"workload": w.name, "batch": w.batch, "h_q": w.h_q, "h_kv": w.h_kv,
                   "d_qk": w.d_qk, "d_v": w.d_v, "s_q": w.s_q,
                   "cap_or_s_k": w.cap if w.mode == "kvcache" else w.s_k, "causal": w.causal,
                   "rotary_dim": w.rotary_dim, "interleaved": w.interleaved,
                   "l2": "flushed before every timed step (untimed 512 MiB write, then 256 MiB read of "
                         "another buffer: no step data and no dirty lines left in L2)",
                   "parallelism": f"{world} independent replicas" if world > 1 else "1 GPU",
                   "plan": plan},
        "roofline": {"bound": bound, "achieved": round(achieved, 3), "peak": peak,
                     "unit": unit, "frac": round(achieved / peak, 4),
                     "traffic": traffic_record(name, kernel_tag),
                     "peak_source": f"{peaks_src} ({peak_key})" + (
                         "; sw_power_cap active on the sampled clocks" if capped and bound != "hbm" else ""),
                     "kernel": kernel_name,
                     "kernel_ms": round(kms_max, 5) if kms_max else None,
                     "timing": ("CUDA events around the kernel's launch on its stream, graph replay, "
                                "L2 flushed per step" if kms_max else "whole call (kernel events unavailable)"),
                     "call_ms": round(ms_max, 5),
                     "spec_peak": SPEC_PEAKS[bound][0] if bound in SPEC_PEAKS else None,
                     "frac_of_spec": (round(achieved / SPEC_PEAKS[bound][0], 4) if bound in SPEC_PEAKS else None),
                     "amount_per_launch": amount},
        "e2e": {"value": e2e_value, "unit": unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": int(plan["launches"]) * args.steps,
    }
    if clocks:
        rec["clocks"] = clocks
    del graph
    return rec, clocks, w, inp, amount, unit


def run_ours(args):
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        print(json.dumps({"metric": METRIC, "error": "no CUDA device"}))
        return 1
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    barrier = (lambda: dist.barrier()) if world > 1 else (lambda: None)

    import rotary_embedding_b200 as fa
    peaks, peaks_src = load_peaks()
    subs = sub_names(args)
    head, clocks, w, inp, _, unit = measure(args.config, args, fa, device, world, barrier, peaks, peaks_src)
    sub_recs = {}
    for name in subs:
        rec = measure(name, args, fa, device, world, barrier, peaks, peaks_src)[0]
        sub_recs[name] = rec

    result = {
        "metric": METRIC,
        "value": head["value"],
        "unit": head["unit"],
        "n_gpus": world,
        "steps": args.steps,
        "warmup": max(args.warmup, 3),
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic (seeded, N(0,1)/U[0,1) as the workload states)",
        "config": head["config"],
        "roofline": head["roofline"],
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"] + sum(r["gpu_launches"] for r in sub_recs.values()),
    }
    if clocks:
        result["clocks"] = clocks
    if sub_recs:
        # each decode workload with its own value, roofline (HBM) and end-to-end leg
        result["decode"] = sub_recs
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        amt, secs, desc = cpu_sample(w, inp, args.cpu_seconds)
        result["cpu_baseline"] = {"value": round(amt / secs, 6), "unit": unit, "cores": 1,
                                  "kind": "oracle", "sample": desc, "seconds": round(secs, 2),
                                  "cpu": cpu_model(), "host_cores": os.cpu_count()}
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = W.CONFIGS[args.config]
    inp = W.make_inputs(w, seed=0)
    seqlens = (inp["cache_seqlens"].tolist() if w.mode == "kvcache"
               else (inp["cu_seqlens"].diff().tolist() if w.mode == "varlen" else None))
    _, unit, _ = work_units(w, seqlens)
    # each step is one bounded sample; the whole run stays within a few minutes
    per_step = max(0.2, min(5.0, 60.0 / max(args.steps, 1)))
    for _ in range(max(args.warmup, 0)):
        cpu_sample(w, inp, 0.0)
    vals, tot_amt, tot_s, desc = [], 0.0, 0.0, ""
    for _ in range(args.steps):
        amt, secs, desc = cpu_sample(w, inp, per_step)
        vals.append(amt / secs)
        tot_amt += amt
        tot_s += secs
    value = tot_amt / tot_s
    result = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": unit,
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 * tot_s / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)", "config": {"workload": w.name},
        "cpu_baseline": {"value": round(value, 6), "unit": unit, "cores": 1, "kind": "oracle",
                         "sample": desc, "cpu": cpu_model(), "host_cores": os.cpu_count()},
        "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(result), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
