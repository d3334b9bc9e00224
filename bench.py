#!/usr/bin/env python
"""Benchmark of the Liger Attention forward pass on B200.

Workload (Llama-3-8B attention shape, synthetic seeded N(0,1) data):
  prefill: B=2, T=8192, Hq=32, Hkv=8, d=128, bf16, w=64, alpha=0.5, fp32 final state
  decode:  B=64, Hq=32, Hkv=8, d=128 after a 1024-token prefill; 1000 steps captured in a CUDA graph
  shared-state decode (one state per kv head): B=256, same shape
The Llama-3.2-1B prefill (B=4, T=2048, d=64) and the long packed prefill (4 sequences,
32768 tokens, d=128) are timed the same way and reported under "llama1b_prefill" and
"long_varlen".

One step = one prefill call over the whole batch (the headline `value`,
tokens/s); the decode loops are timed in the same run and reported under
"decode" and "decode_kvshared".  The 8B and long prefill inputs and the decode
states are larger than L2 (q, k, v 201 MB; decode states 268 MB per head at
B=64 and 134 MB per kv head at B=256), so no L2 flush is needed between their
iterations; the 1B prefill's 86 MB would fit, so an L2-sized buffer is written
between its timed calls (outside the events that time the chunk pass).
Multi-GPU: one process per GPU, every rank runs the same per-GPU workload (weak
scaling, no collective on the data path); times are the max over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_linear_attention_liger_b200 import inputs  # noqa: E402

METRIC = "prefill tokens/s & decode tokens/s (8B attn shape), % of roofline"
PREFILL = inputs.WORKLOADS["llama8b_prefill"]
PREFILL_1B = inputs.WORKLOADS["llama1b_prefill"]
PREFILL_LONG = inputs.WORKLOADS["long_varlen"]
DECODE = inputs.WORKLOADS["llama8b_decode"]
DECODE_KV = inputs.WORKLOADS["llama8b_decode_kvshared"]
L2_BYTES = 126 * 2 ** 20


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


def measured_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu capture, or None when the
    kernel's sources have changed since the capture was taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)[kernel]
    except (OSError, KeyError, ValueError):
        return None
    m = hashlib.sha256()
    for name in rec["source_files"]:
        with open(os.path.join(ROOT, "gated_linear_attention_liger_b200", "csrc", name), "rb") as f:
            m.update(f.read())
    return float(rec["bytes"]) if m.hexdigest()[:16] == rec["source_sha"] else None


def prefill_algorithmic(wl=PREFILL):
    """Algorithmic bytes and flops of one prefill call (read q, k, v once, write out and the
    final state once; flops of readout, causal intra-chunk, state update and window)."""
    tok = wl.B * wl.T
    esz = 2 if wl.dtype == torch.bfloat16 else 4
    bytes_ = tok * (2 * wl.Hq + 2 * wl.Hkv) * wl.d * esz + wl.n_seqs * wl.Hq * wl.d * wl.d * 4
    C = 64
    flops = tok * (wl.Hq * 2 * wl.d ** 2 + wl.Hq * 4 * wl.d * (C + 1) / 2 + wl.Hkv * 2 * wl.d ** 2
                   + wl.Hq * 4 * wl.w * wl.d)
    return bytes_, flops


def exact_decay_chunks(wl, k, threshold=-60.0):
    """(chunk, kv head) pairs whose total log gate lies below `threshold`: the prefill's chunk
    pass evaluates their decay without factoring it at the chunk end (a slower mode).  Chunks
    are 64-token blocks counted from each sequence start.  A statistic of the input for the
    report, computed here in numpy from the gate's definition (sigmoid of the key's mean)."""
    kk = k.float().numpy().astype(np.float64)   # [B, T, Hkv, d]
    cu = wl.cu_seqlens
    seqs = [kk[0, a:b] for a, b in zip(cu[:-1], cu[1:])] if cu else [kk[b] for b in range(wl.B)]
    total = exact = 0
    for ks in seqs:
        m = ks.mean(-1)                                                   # [len, Hkv]
        lg = np.minimum(m, 0.0) - np.log1p(np.exp(-np.abs(m)))            # log sigmoid(m)
        for c0 in range(0, ks.shape[0], 64):
            bc = lg[c0:c0 + 64].sum(0)
            total += bc.size
            exact += int((bc < threshold).sum())
    return exact, total


def decode_algorithmic(wl=DECODE, kvshared=False):
    """Bytes of one decode step: state read + write, window ring read, the new key and value
    written into the ring, q/k/v read, out write."""
    esz = 2
    state = wl.B * (wl.Hkv if kvshared else wl.Hq) * wl.d * wl.d * 4 * 2
    ring = wl.B * wl.Hkv * 2 * wl.w * wl.d * esz + wl.B * wl.Hkv * 2 * wl.d * esz
    io = wl.B * (2 * wl.Hq + 2 * wl.Hkv) * wl.d * esz
    return state + ring + io


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML in a background thread."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples = []
        self.ok = False
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.sm_max = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - depends on the box
            self.err = repr(e)
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                clk = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                except AttributeError:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                self.samples.append((time.perf_counter(), clk, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t.start()
        return self

    def stop(self):
        self._stop.set()
        if self.ok:
            self._t.join(timeout=2)

    def summary(self, windows):
        if not self.ok:
            return {"error": getattr(self, "err", "nvml unavailable")}
        sel = [s for s in self.samples if any(a <= s[0] <= b for a, b in windows)]
        if not sel:  # regions shorter than the sampling period: take the nearest samples
            mids = [(a + b) / 2 for a, b in windows]
            sel = [min(self.samples, key=lambda s: abs(s[0] - m)) for m in mids] if self.samples else []
        reasons = set()
        for _, _, rs in sel:
            for name, bit in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median([s[1] for s in sel]) if sel else None,
                "sm_max_mhz": self.sm_max, "reasons": sorted(reasons), "samples": len(sel)}


# ----------------------------------------------------------------- dist

def timing_events(n, stream):
    """n timing events whose CUDA handles exist (torch creates them at first record), so the
    library can record them by handle."""
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for e in evs:
        e.record(stream)
    return evs


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def weak_scaling_value(tokens_per_rank: int, world: int, max_ms_per_step: float) -> float:
    """Whole-job throughput: every rank processes its own copy of the workload, the step time
    is the slowest rank's."""
    return world * tokens_per_rank / (max_ms_per_step * 1e-3)


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------- CPU oracle

def cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_model() -> str:
    """The host CPU's model name (first entry of /proc/cpuinfo), or "unknown"."""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_prefill_sample(target_s: float):
    """Times the fp64 oracle on a bounded sample of the prefill workload and returns
    (workload tokens/s, seconds, sample description, threads).  The sample is the first T_s
    tokens of every sequence, all q heads, with T_s sized by a short calibration so the run
    takes about target_s; if the whole workload fits in that time it is run whole, repeated
    until target_s has passed."""
    from oracle import oracle
    wl = PREFILL
    q, k, v = inputs.prefill_inputs(wl)
    q, k, v = (t.float().numpy().astype(np.float64) for t in (q, k, v))
    nthr = min(cpu_threads(), wl.B * wl.Hq)
    t_cal = 128
    t0 = time.perf_counter()
    oracle.prefill(q[:, :t_cal], k[:, :t_cal], v[:, :t_cal], w=wl.w, alpha=wl.alpha, nthreads=nthr)
    dt = time.perf_counter() - t0
    T_s = int(min(wl.T, max(t_cal, t_cal * target_s / max(dt, 1e-6))))
    reps, secs = 0, 0.0
    while reps == 0 or secs < target_s:
        t0 = time.perf_counter()
        oracle.prefill(q[:, :T_s], k[:, :T_s], v[:, :T_s], w=wl.w, alpha=wl.alpha, nthreads=nthr)
        secs += time.perf_counter() - t0
        reps += 1
    tokens = wl.B * T_s * reps
    desc = (f"fp64 oracle, all {wl.B} sequences x {wl.Hq} q heads, first {T_s} of {wl.T} tokens, "
            f"run {reps}x ({tokens} workload tokens in {secs:.1f} s), {nthr} threads")
    return tokens / secs, secs, desc, nthr


def run_reference(args, world, rank):
    """The reference arm: the fp64 CPU oracle as it stands, on host cores, rank 0 only."""
    if rank != 0:
        return
    per_step = max(2.0, 150.0 / max(1, args.steps + args.warmup))
    vals = []
    desc = ""
    nthr = cpu_threads()
    for i in range(args.warmup + args.steps):
        tps, secs, desc, nthr = oracle_prefill_sample(per_step)
        if i >= args.warmup:
            vals.append(tps)
    value = float(statistics.median(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": PREFILL.tokens / value * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1))", "config": workload_config(),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": nthr, "kind": "oracle",
                         "sample": desc, "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config():
    p, d, dk = PREFILL, DECODE, DECODE_KV
    return {"workload": "llama8b_prefill (+ llama8b_decode)",
            "prefill": {"B": p.B, "T": p.T, "Hq": p.Hq, "Hkv": p.Hkv, "d": p.d, "w": p.w,
                        "alpha": p.alpha},
            "decode": {"B": d.B, "prefix": d.T, "Hq": d.Hq, "Hkv": d.Hkv, "d": d.d, "w": d.w,
                       "alpha": d.alpha},
            "decode_kvshared": {"B": dk.B, "prefix": dk.T},
            "l2": "inputs larger than L2 (prefill q+k+v 201 MB; decode states 268 MB per head at B=64, "
                  "134 MB per kv head at B=256; L2 126 MB)"}


# ----------------------------------------------------------------- GPU arm

def run_ours(args, world, rank, local):
    from gated_linear_attention_liger_b200 import ops
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    ops.load()
    pk = peaks()
    stream = torch.cuda.Stream(device=dev)
    sampler = ClockSampler(local).start()
    windows = []

    if args.only == "decode":
        dec = run_decode(args, world, dev, stream, pk, windows)
        dec_kv = run_decode(args, world, dev, stream, pk, windows, kvshared=True)
        sampler.stop()
        if rank == 0:
            print(json.dumps({"metric": METRIC, "partial": "decode only", "decode": dec,
                              "decode_kvshared": dec_kv, "clocks": sampler.summary(windows)}), flush=True)
        return

    # ---------------- prefill
    wl = PREFILL
    res8 = time_prefill(wl, args, world, dev, stream, pk, windows)
    q, k, v, out, fs, ws = res8.pop("_tensors")
    value = weak_scaling_value(wl.tokens, world, res8["ms_per_step"])
    ms_step = res8["ms_per_step"]
    prefill_launches = res8["gpu_launches"]
    roofline = res8["roofline"]
    roofline["traffic"] = measured_traffic("chunk_kernel<128>")

    # ---------------- e2e: host buffers, copies inside the timed region
    # Consecutive batches as a serving loop runs them: two device buffer sets, the next
    # batch's inputs copied in on one stream while the current batch computes, and the
    # results copied out on a third (PCIe moves both directions at once).  Every step's
    # copies in and out are inside the timed region.
    e2e = None
    if not args.no_e2e and args.only is None:
        hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
        ho = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        hfs = torch.empty(fs.shape, dtype=fs.dtype).pin_memory()
        n_e2e = max(2, min(args.steps, 10))
        bufs = [(q, k, v, out, fs), tuple(torch.empty_like(t) for t in (q, k, v, out, fs))]
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev = {(n, i): torch.cuda.Event() for n in ("in", "comp", "out") for i in (0, 1)}
        used = [False, False]

        def e2e_step(i):
            bq, bk, bv, bo, bfs = bufs[i % 2]
            j = i % 2
            with torch.cuda.stream(s_in):
                if used[j]:
                    s_in.wait_event(ev[("comp", j)])   # this buffer's previous batch is computed
                bq.copy_(hq, non_blocking=True)
                bk.copy_(hk, non_blocking=True)
                bv.copy_(hv, non_blocking=True)
                ev[("in", j)].record(s_in)
            stream.wait_event(ev[("in", j)])
            if used[j]:
                stream.wait_event(ev[("out", j)])      # and its results are copied out
            ops.prefill(bq, bk, bv, alpha=wl.alpha, w=wl.w, out=bo, final_state=bfs, workspace=ws,
                        stream=stream)
            ev[("comp", j)].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev[("comp", j)])
                ho.copy_(bo, non_blocking=True)
                hfs.copy_(bfs, non_blocking=True)
                ev[("out", j)].record(s_out)
            used[j] = True

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s_in)
        for i in range(n_e2e):
            e2e_step(i)
        s_out.wait_event(ev[("out", (n_e2e - 1) % 2)])
        b.record(s_out)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(b) / n_e2e, world, dev)
        e2e = {"value": world * wl.tokens / (e_ms * 1e-3), "unit": "tokens/s",
               "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in (hq, hk, hv)),
               "d2h_bytes_per_step": ho.numel() * ho.element_size() + hfs.numel() * hfs.element_size(),
               "ms_per_step": e_ms, "steps": n_e2e,
               "pipeline": "two device buffer sets; copy-in, compute and copy-out on three streams"}
        del hq, hk, hv, ho, hfs, bufs
    del q, k, v, out, ws

    # ---------------- the other prefill workloads (1B shape, long packed sequences)
    others = {}
    if args.only is None or args.only == "prefill":
        for owl, flush in ((PREFILL_1B, True), (PREFILL_LONG, False)):
            r = time_prefill(owl, args, world, dev, stream, pk, windows, flush_l2=flush)
            r.pop("_tensors")
            r["roofline"]["traffic"] = measured_traffic(f"chunk_kernel<{owl.d}>@{owl.name}")
            others[owl.name] = r

    # ---------------- the prefill's gradient (the fine-tune's backward pass)
    bwd = None
    if args.only is None or args.only == "backward":
        bwd = time_backward(PREFILL, args, world, dev, stream, pk, windows)

    # ---------------- the per-dimension (vector) gate prefill
    vgate = None
    if args.only is None or args.only == "vgate":
        vgate = time_vector_gate(PREFILL, args, world, dev, stream, pk, windows)

    # ---------------- the hybrid's standard attention layer (causal softmax attention)
    full = None
    if args.only is None or args.only == "full":
        full = time_full_attention(PREFILL, args, world, dev, stream, pk, windows)

    # ---------------- decode
    dec = (None if args.only in ("prefill", "full", "backward", "vgate")
           else run_decode(args, world, dev, stream, pk, windows))
    dec_kv = (None if args.only in ("prefill", "full", "backward", "vgate")
              else run_decode(args, world, dev, stream, pk, windows, kvshared=True))

    sampler.stop()
    clocks = sampler.summary(windows)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.only is None:
        tps, secs, desc, nthr = oracle_prefill_sample(args.cpu_seconds)
        cpu = {"value": tps, "unit": "tokens/s", "cores": nthr, "kind": "oracle", "sample": desc,
               "seconds": secs, "cpu_model": cpu_model()}
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1), Llama-3-8B attention shapes)",
            "config": workload_config(), "roofline": roofline, "prefill_call": res8["call"],
            "llama1b_prefill": others.get("llama1b_prefill"), "long_varlen": others.get("long_varlen"),
            "full_attention": full, "backward": bwd, "vector_gate": vgate,
            "decode": dec, "decode_kvshared": dec_kv, "e2e": e2e,
            "gpu_launches": prefill_launches, "clocks": clocks, "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)


def time_prefill(wl, args, world, dev, stream, pk, windows, flush_l2=False):
    """Times `args.steps` prefill calls of workload `wl` (after `args.warmup` untimed ones) and,
    in a second pass, the chunk kernel alone with CUDA events the library records around it on
    the call's stream.  With flush_l2, a buffer larger than L2 is written before every call
    (between the step events, so the step time then includes it: the kernel time does not)."""
    from gated_linear_attention_liger_b200 import ops
    q, k, v = (t.to(dev) for t in inputs.prefill_inputs(wl))
    cu = None if wl.cu_seqlens is None else torch.tensor(wl.cu_seqlens, dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    fs = torch.empty(wl.n_seqs, wl.Hq, wl.d, wl.d, device=dev, dtype=torch.float32)
    ws_n = ops.prefill_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.T, wl.d, wl.n_seqs)
    ws = torch.empty(max(ws_n, 1), device=dev, dtype=torch.uint8)
    flush = torch.empty(2 * L2_BYTES // 4, device=dev, dtype=torch.float32) if flush_l2 else None

    def call():
        if flush is not None:
            with torch.cuda.stream(stream):
                flush.fill_(1.0)
        ops.prefill(q, k, v, alpha=wl.alpha, w=wl.w, cu_seqlens=cu, out=out, final_state=fs, workspace=ws,
                    stream=stream)

    torch.cuda.synchronize()
    for _ in range(args.warmup):
        call()
    ks = timing_events(args.steps, stream)
    ke = timing_events(args.steps, stream)
    cs = timing_events(args.steps, stream)
    ce = timing_events(args.steps, stream)
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stream.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    launches0 = ops.kernel_launches()
    w0 = time.perf_counter()
    t_start.record(stream)
    for i in range(args.steps):
        if flush is not None:   # time each call alone, without the flush in front of it
            with torch.cuda.stream(stream):
                flush.fill_(1.0)
            cs[i].record(stream)
            ops.prefill(q, k, v, alpha=wl.alpha, w=wl.w, cu_seqlens=cu, out=out, final_state=fs, workspace=ws,
                        stream=stream)
            ce[i].record(stream)
        else:
            call()
    t_end.record(stream)
    torch.cuda.synchronize()
    windows.append((w0, time.perf_counter()))
    barrier(world)
    launches = ops.kernel_launches() - launches0
    if flush is not None:
        ms_step = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in zip(cs, ce)), world, dev)
    else:
        ms_step = max_over_ranks(t_start.elapsed_time(t_end) / args.steps, world, dev)
    # the chunk kernel's own time, from events around it in a second pass (the events
    # serialise its launch, so the step time above is taken without them)
    w1 = time.perf_counter()
    for i in range(args.steps):
        ops.set_timing_events(ks[i], ke[i])
        call()
    ops.set_timing_events(None, None)
    torch.cuda.synchronize()
    windows.append((w1, time.perf_counter()))
    barrier(world)
    k_ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in zip(ks, ke)), world, dev)
    alg_bytes, alg_flops = prefill_algorithmic(wl)
    achieved = alg_bytes / (k_ms * 1e-3) / 1e9
    res = {
        "metric": f"prefill tokens/s ({wl.name})", "value": weak_scaling_value(wl.tokens, world, ms_step),
        "unit": "tokens/s", "ms_per_step": ms_step, "gpu_launches": launches,
        "workload": {"B": wl.B, "T": wl.T, "Hq": wl.Hq, "Hkv": wl.Hkv, "d": wl.d, "w": wl.w,
                     "alpha": wl.alpha, "seqlens": list(wl.seqlens) or None,
                     "l2": "L2-sized buffer written before each timed call" if flush_l2 else
                           "inputs larger than L2"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / pk["hbm_gbs"], "traffic": None,
                     "kernel": "prefill chunk pass", "kernel_ms": k_ms,
                     "algorithmic_bytes": alg_bytes, "algorithmic_flops": alg_flops,
                     "tensor_frac": alg_flops / (k_ms * 1e-3) / (pk["bf16_tflops"] * 1e12),
                     "peak_source": pk["source"], "frac_of": f"{pk['source']} HBM copy bandwidth"},
        # the whole call (every kernel of it) against the same roofline
        "call": {"ms": ms_step, "achieved": alg_bytes / (ms_step * 1e-3) / 1e9,
                 "frac": alg_bytes / (ms_step * 1e-3) / 1e9 / pk["hbm_gbs"]},
    }
    if wl.key_bias_std or wl.cu_seqlens:
        ex, tot = exact_decay_chunks(wl, k.cpu())
        res["exact_decay_chunks"] = {"count": ex, "of": tot,
                                     "note": "(chunk, kv head) pairs with total log gate < -60"}
    res["_tensors"] = (q, k, v, out, fs, ws)
    return res


def backward_algorithmic(wl):
    """Algorithmic bytes and flops of one backward call: read q, k, v and d_out, write dq, dk, dv
    once; flops per token of the window branch (10 w d per q head: scores, dO.v, and the three
    gradient products over the band), the recurrent branch's causal intra-chunk products
    (5 d (C+1) per q head) and its state products (4 d^2 per q head, 6 d^2 per kv head)."""
    tok = wl.B * wl.T
    esz = 2
    bytes_ = tok * (3 * wl.Hq + 4 * wl.Hkv) * wl.d * esz
    C = 64
    flops = tok * (wl.Hq * (10 * wl.w * wl.d + 5 * wl.d * (C + 1) + 4 * wl.d ** 2) + wl.Hkv * 6 * wl.d ** 2)
    return bytes_, flops


def time_backward(wl, args, world, dev, stream, pk, windows):
    """Times the gradient of the prefill (bf16, d_out given, no final-state gradient) with the
    library's events around its two per-chunk gradient kernels, and the whole call."""
    from gated_linear_attention_liger_b200 import ops
    q, k, v = (t.to(dev) for t in inputs.prefill_inputs(wl))
    gen = torch.Generator().manual_seed(23)
    dout = torch.randn(q.shape, generator=gen).to(q.dtype).to(dev)
    ws = torch.empty(ops.prefill_backward_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.T, wl.d, wl.n_seqs), device=dev,
                     dtype=torch.uint8)

    def call():
        ops.prefill_backward(q, k, v, dout, alpha=wl.alpha, workspace=ws, stream=stream)

    torch.cuda.synchronize()
    for _ in range(args.warmup):
        call()
    n = max(3, min(args.steps, 10))
    ks, ke = timing_events(n, stream), timing_events(n, stream)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stream.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    w0 = time.perf_counter()
    a.record(stream)
    for i in range(n):
        call()
    b.record(stream)
    torch.cuda.synchronize()
    for i in range(n):
        ops.set_timing_events(ks[i], ke[i])
        call()
    ops.set_timing_events(None, None)
    torch.cuda.synchronize()
    windows.append((w0, time.perf_counter()))
    barrier(world)
    status = ops.prefill_status(ws)
    ms = max_over_ranks(a.elapsed_time(b) / n, world, dev)
    k_ms = max_over_ranks(statistics.mean(x.elapsed_time(y) for x, y in zip(ks, ke)), world, dev)
    alg_bytes, alg_flops = backward_algorithmic(wl)
    t_bw, t_tc = alg_bytes / (pk["hbm_gbs"] * 1e9), alg_flops / (pk["bf16_tflops"] * 1e12)
    bound = "hbm" if t_bw >= t_tc else "tensor"
    achieved = alg_bytes / (ms * 1e-3) / 1e9 if bound == "hbm" else alg_flops / (ms * 1e-3) / 1e12
    peak = pk["hbm_gbs"] if bound == "hbm" else pk["bf16_tflops"]
    del q, k, v, dout, ws
    return {"metric": "prefill backward tokens/s (8B attn shape)", "value": world * wl.tokens / (ms * 1e-3),
            "unit": "tokens/s", "ms_per_step": ms, "steps": n, "status": ops.STATUS_NAMES.get(status, status),
            "gradient_kernels_ms": k_ms,
            "roofline": {"bound": bound, "achieved": achieved, "peak": peak,
                         "unit": "GB/s" if bound == "hbm" else "TFLOP/s", "frac": achieved / peak, "traffic": None,
                         "kernel": "whole backward call", "algorithmic_bytes": alg_bytes,
                         "algorithmic_flops": alg_flops,
                         "tensor_frac": alg_flops / (ms * 1e-3) / (pk["bf16_tflops"] * 1e12),
                         "peak_source": pk["source"]}}


def time_vector_gate(wl, args, world, dev, stream, pk, windows):
    """Times the prefill with one gate per key dimension (general CUDA-core kernel) on the
    workload; the same algorithmic bytes as the scalar-gate prefill."""
    from gated_linear_attention_liger_b200 import ops
    q, k, v = (t.to(dev) for t in inputs.prefill_inputs(wl))
    ws = torch.empty(ops.prefill_vector_gate_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.T, wl.d, wl.n_seqs), device=dev,
                     dtype=torch.uint8)
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        ops.prefill_vector_gate(q, k, v, alpha=wl.alpha, w=wl.w, workspace=ws, stream=stream)
    n = max(3, min(args.steps, 10))
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stream.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    w0 = time.perf_counter()
    a.record(stream)
    for _ in range(n):
        ops.prefill_vector_gate(q, k, v, alpha=wl.alpha, w=wl.w, workspace=ws, stream=stream)
    b.record(stream)
    torch.cuda.synchronize()
    windows.append((w0, time.perf_counter()))
    barrier(world)
    ms = max_over_ranks(a.elapsed_time(b) / n, world, dev)
    alg_bytes, alg_flops = prefill_algorithmic(wl)
    achieved = alg_bytes / (ms * 1e-3) / 1e9
    del q, k, v, ws
    return {"metric": "vector-gate prefill tokens/s (8B attn shape)", "value": world * wl.tokens / (ms * 1e-3),
            "unit": "tokens/s", "ms_per_step": ms, "steps": n,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / pk["hbm_gbs"], "traffic": None,
                         "kernel": "whole call (segment-parallel general prefill, CUDA cores)",
                         "algorithmic_bytes": alg_bytes, "peak_source": pk["source"]}}


def full_attention_flops(wl):
    """Algorithmic flops of causal softmax attention: Q K^T and P V over the causal half of the
    T x T score matrix (diagonal included), 2 flops per multiply-add."""
    pairs = wl.T * (wl.T + 1) / 2
    return wl.B * wl.Hq * pairs * wl.d * 4


def time_full_attention(wl, args, world, dev, stream, pk, windows):
    """Times the causal attention layer (the inter-layer hybrid's standard attention) on the
    workload's q, k, v: kernel time from the library's events, tensor-bound roofline."""
    from gated_linear_attention_liger_b200 import ops
    q, k, v = (t.to(dev) for t in inputs.prefill_inputs(wl))
    out = torch.empty_like(q)

    def call():
        ops.full_causal_attention(q, k, v, out=out, stream=stream)

    torch.cuda.synchronize()
    for _ in range(args.warmup):
        call()
    n = max(3, min(args.steps, 10))
    ks, ke = timing_events(n, stream), timing_events(n, stream)
    stream.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    w0 = time.perf_counter()
    for i in range(n):
        ops.set_timing_events(ks[i], ke[i])
        call()
    ops.set_timing_events(None, None)
    torch.cuda.synchronize()
    windows.append((w0, time.perf_counter()))
    barrier(world)
    status = ops.full_causal_status()
    k_ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in zip(ks, ke)), world, dev)
    flops = full_attention_flops(wl)
    achieved = flops / (k_ms * 1e-3) / 1e12
    del q, k, v, out
    return {"metric": "causal attention tokens/s (8B attn shape)", "value": world * wl.tokens / (k_ms * 1e-3),
            "unit": "tokens/s", "ms_per_step": k_ms, "steps": n, "status": ops.STATUS_NAMES.get(status, status),
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": achieved / pk["bf16_tflops"], "traffic": measured_traffic("full_attn_kernel<128>"), "kernel": "causal attention",
                         "kernel_ms": k_ms, "algorithmic_flops": flops, "peak_source": pk["source"],
                         "frac_of": f"{pk['source']} cuBLAS bf16 burst"}}


def run_decode(args, world, dev, stream, pk, windows, kvshared=False):
    from gated_linear_attention_liger_b200 import ops
    wl = DECODE_KV if kvshared else DECODE
    n_graph = args.decode_steps
    # state, ring and pos from a seeded 1024-token prefill through the library
    pre = inputs.Workload("decode_prefix", "prefill", wl.B, wl.Hq, wl.Hkv, wl.T, wl.d, wl.dtype,
                          seed=wl.seed)
    pq, pkk, pv = (t.to(dev) for t in inputs.prefill_inputs(pre))
    _, state, ring, pos = ops.prefill(pq, pkk, pv, alpha=wl.alpha, w=wl.w, return_ring=True,
                                      stream=stream)
    stream.synchronize()
    if kvshared:   # one state per (sequence, kv head): the group's copies are equal after prefill
        state = state[:, ::wl.Hq // wl.Hkv].contiguous()
    step_fn = ops.decode_kvshared if kvshared else ops.decode
    del pq, pkk, pv
    steps_in = [inputs.decode_step_inputs(wl, s) for s in range(n_graph)]
    dq = torch.stack([s[0] for s in steps_in]).to(dev)
    dk = torch.stack([s[1] for s in steps_in]).to(dev)
    dv = torch.stack([s[2] for s in steps_in]).to(dev)
    dout = torch.empty_like(dq)
    ks = timing_events(n_graph, stream)
    ke = timing_events(n_graph, stream)

    def steps(timed):
        for s in range(n_graph):
            if timed:
                ops.set_timing_events(ks[s], ke[s])
            step_fn(dq[s], dk[s], dv[s], state, ring, pos, alpha=wl.alpha, out=dout[s], stream=stream)
        ops.set_timing_events(None, None)

    steps(False)  # warm-up outside the graph
    stream.synchronize()
    # two graphs of the same steps: a plain one for the step rate, and one whose kernels are
    # bracketed by timing events (event nodes serialise the launches, so it only gives kernel time)
    graph = torch.cuda.CUDAGraph()
    l0 = ops.kernel_launches()
    with torch.cuda.graph(graph, stream=stream):
        steps(False)
    per_graph_launches = ops.kernel_launches() - l0
    kernel_events = True
    tgraph = torch.cuda.CUDAGraph()
    try:
        with torch.cuda.graph(tgraph, stream=stream):
            steps(True)
    except Exception:
        kernel_events = False

    for _ in range(max(1, min(args.warmup, 3))):
        graph.replay()
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 2
    w0 = time.perf_counter()
    k_ms = []
    with torch.cuda.stream(stream):
        a.record(stream)
        for _ in range(reps):
            graph.replay()
        b.record(stream)
    torch.cuda.synchronize()
    windows.append((w0, time.perf_counter()))
    if kernel_events:
        with torch.cuda.stream(stream):
            for _ in range(max(1, reps // 2)):
                tgraph.replay()
                stream.synchronize()
                try:
                    k_ms.append(statistics.mean(x.elapsed_time(y) for x, y in zip(ks, ke)))
                except (RuntimeError, ValueError):
                    kernel_events = False
                    break
    barrier(world)
    ms_step = max_over_ranks(a.elapsed_time(b) / (reps * n_graph), world, dev)
    kms = max_over_ranks(statistics.mean(k_ms), world, dev) if (kernel_events and k_ms) else ms_step
    alg = decode_algorithmic(wl, kvshared)
    achieved = alg / (kms * 1e-3) / 1e9
    del graph, tgraph

    # end to end through the public call: every step's q, k, v copied in from pinned host
    # memory and its output copied back, on copy streams that overlap the compute stream
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (t.cpu().pin_memory() for t in (dq, dk, dv))
        ho = torch.empty(dout.shape, dtype=dout.dtype).pin_memory()
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(n_graph)]
        ev_c = [torch.cuda.Event() for _ in range(n_graph)]
        torch.cuda.synchronize()
        barrier(world)
        ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ea.record(s_in)
        stream.wait_event(ea)
        with torch.cuda.stream(s_in):
            for s_ in range(n_graph):
                dq[s_].copy_(hq[s_], non_blocking=True)
                dk[s_].copy_(hk[s_], non_blocking=True)
                dv[s_].copy_(hv[s_], non_blocking=True)
                ev_in[s_].record(s_in)
        for s_ in range(n_graph):
            stream.wait_event(ev_in[s_])
            step_fn(dq[s_], dk[s_], dv[s_], state, ring, pos, alpha=wl.alpha, out=dout[s_], stream=stream)
            ev_c[s_].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_c[s_])
                ho[s_].copy_(dout[s_], non_blocking=True)
        s_out.wait_event(ev_c[-1])
        eb.record(s_out)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(ea.elapsed_time(eb) / n_graph, world, dev)
        e2e = {"value": world * wl.B / (e_ms * 1e-3), "unit": "tokens/s", "ms_per_step": e_ms,
               "steps": n_graph,
               "h2d_bytes_per_step": sum(t[0].numel() * t.element_size() for t in (hq, hk, hv)),
               "d2h_bytes_per_step": ho[0].numel() * ho.element_size(),
               "pipeline": "per step: q, k, v copied in, one decode call, out copied back; copies on "
                           "two streams beside the compute stream; states stay on the device"}
        del hq, hk, hv, ho
    name = f"decode tokens/s (8B attn shape, B={wl.B}" + (", one state per kv head)" if kvshared else ")")
    return {"metric": name, "value": world * wl.B / (ms_step * 1e-3), "e2e": e2e,
            "unit": "tokens/s", "ms_per_step": ms_step, "graph_steps": n_graph, "replays": reps,
            "gpu_launches": per_graph_launches * reps,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / pk["hbm_gbs"],
                         "traffic": measured_traffic("decode_stream_kernel<bf16,128,4,kv-shared>" if kvshared
                                                     else "decode_stream_kernel<bf16,128,1,per-head>"),
                         "kernel": "decode state stream" + (" (kv-shared)" if kvshared else ""), "kernel_ms": kms,
                         "kernel_timing": "events in graph" if kernel_events else "graph step average",
                         "algorithmic_bytes": alg, "peak_source": pk["source"]}}


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-steps", type=int, default=1000, help="decode steps per captured graph")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target length of the CPU baseline")
    ap.add_argument("--only", choices=["prefill", "decode", "full", "backward", "vgate"], default=None,
                    help="run one part only (for profiling); the JSON line is then partial")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("note: warm-up raised to 3", file=sys.stderr)
        args.warmup = 3
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
