#!/usr/bin/env python
"""Decode-step benchmark of the RTPurbo sparse attention library on B200.

One step = one rtp_decode_step call over one batch of a synthetic workload
(index scoring, top-p selection, block lists, retrieval and local attention,
combine).  Default workload: 1M context (B=1, 8 KV heads x GQA 4, one
retrieval KV group, 28 local heads, window 4096, sink 4, p=0.9,
needle-peaked), inputs resident in HBM, L2 flushed (256 MB write) before
every timed step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 1..5] [--impl ours|reference]

Multi-GPU: replicas (the step has no cross-GPU exchange); launched by
torch.distributed.run, one process per GPU; time = max over ranks.
Prints ONE JSON line on rank 0.
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

METRIC = "decode context-tokens/s (RTPurbo sparse decode step)"
UNIT = "tokens/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=4)
    ap.add_argument("--scale", type=int, default=1, help="divide the workload's context lengths (profiling runs)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--dense", action="store_true", help="p = 1 for every sequence (dense comparator)")
    ap.add_argument("--topk", type=int, default=0,
                    help="static top-k selection with this k (the fixed-budget variant) instead of top-p")
    ap.add_argument("--no-dense-comparator", action="store_true",
                    help="skip timing the same captured step with p = 1 (the line's dense_comparator)")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="time only the headline workload (skip the 32K, 4 x 128K and ragged lines)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--op", choices=["decode", "append", "kv_append", "prefill"], default="decode",
                    help="append: time the index-cache append instead of the decode step; "
                         "kv_append: the KV-cache write with the index append; "
                         "prefill: the prefill attention of a whole 32K prompt")
    return ap.parse_args()


def hbm_peak():
    try:
        with open(PEAKS_FILE) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ncu summaries whose DRAM traffic the roofline object may quote: kernel ->
# (summary file, workload name).  The figure is used only while the kernel
# sources still hash to the value the summary records and the bench runs the
# summary's workload; otherwise traffic is null.
PROFILED = {"stream": ("profiles/stream_kernel_w4_1m.md", "w4-1m"),
            "retrieve": ("profiles/retrieve_kernel_w3_4x128k.md", "w3-4x128k")}


def kernel_source_hash():
    """Hash of the sources that define the two profiled kernels (the decode
    step's streaming and retrieval kernels and the helpers they include)."""
    import hashlib
    csrc = os.path.join(ROOT, "sparse_attention_decode_rtpurbo_b200", "csrc")
    files = [os.path.join(csrc, f) for f in ("rtp_common.cuh", "rtp_attn.cuh", "rtp_stream.cuh", "rtp_retrieve.cuh")]
    h = hashlib.sha256()
    for p in files:
        h.update(os.path.basename(p).encode())
        with open(p, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel, workload_name):
    entry = PROFILED.get(kernel)
    if entry is None or entry[1] != workload_name:
        return None
    try:
        text = open(os.path.join(ROOT, entry[0])).read()
    except OSError:
        return None
    fields = dict(line.split(":", 1) for line in text.splitlines()
                  if line.startswith(("traffic_bytes_per_launch:", "source_sha256_16:")))
    if fields.get("source_sha256_16", "").strip() != kernel_source_hash():
        return None
    return int(fields["traffic_bytes_per_launch"])


def workload_config(case, wl):
    import synth

    return {"workload": synth.WORKLOADS[wl], "name": case.name, "batch": int(case.B),
            "context": [int(x) for x in case.seq_lens][:16], "context_total": int(case.seq_lens.sum()),
            "q_heads": case.Hq, "kv_heads": case.Hkv, "retrieval_heads": int(case.head_kind.sum()),
            "window": case.window, "sink": case.sink, "p": sorted(set(float(x) for x in case.p)),
            "layout": "paged" if case.paged else "contiguous", "l2": "flushed (256 MB write) before every timed step"}


def algorithmic_bytes(case, kept):
    """Algorithmic byte count of one step (the roofline numerator): index cache of every retrieval KV
    group + the union of kept K/V blocks per retrieval group (rows < L) +
    sink/window rows of every local KV group.  512 B per K+V row, 32 B per
    index row.  "local" counts every sink/window row (the streaming kernel
    reads them all); a KV group with both kinds of heads reads some rows for
    both ("shared": its sink/window rows inside kept blocks), and the step's
    total counts those once."""
    import synth

    G = case.G
    idx = kv = loc = shared = 0
    for b in range(case.B):
        L = int(case.seq_lens[b])
        nblk = (L + 63) // 64
        rows = np.minimum(64, L - 64 * np.arange(nblk))
        for g in range(case.Hkv):
            heads = range(g * G, (g + 1) * G)
            uni = np.zeros(nblk, dtype=bool)
            if any(case.head_kind[h] for h in heads):
                idx += L * 32
                for h in heads:
                    if case.head_kind[h]:
                        uni |= kept[b, h, :nblk].astype(bool)
                kv += int(rows[uni].sum()) * 512
            if any(not case.head_kind[h] for h in heads):
                pos = synth.local_positions(L, case.window, case.sink)
                loc += pos.size * 512
                shared += int(np.count_nonzero(uni[pos // 64])) * 512
    return {"index": idx, "kept_kv": kv, "local": loc, "shared": shared, "total": idx + kv + loc - shared}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def stage_inputs(tensors, host_arrays, device, pin=True):
    """One device buffer for a step's per-step inputs, each at a 256-byte
    aligned offset, and its host twin (pinned): views into the device buffer
    take the place of `tensors` (same shapes and dtypes, same values), so a
    step's inputs cross in one host-to-device copy.  host_arrays: the host
    values of the same tensors (numpy, same element sizes).  Returns
    (device buffer, host buffer, views)."""
    import torch

    offs, off = [], 0
    for t in tensors:
        off = (off + 255) // 256 * 256
        offs.append(off)
        off += t.numel() * t.element_size()
    dbuf = torch.empty(off, dtype=torch.uint8, device=device)
    hbuf = torch.zeros(off, dtype=torch.uint8)
    if pin:
        hbuf = hbuf.pin_memory()
    views = []
    for t, o, a in zip(tensors, offs, host_arrays):
        n = t.numel() * t.element_size()
        v = dbuf[o:o + n].view(t.dtype).view(t.shape)
        v.copy_(t)
        views.append(v)
        raw = np.ascontiguousarray(a).view(np.uint8).reshape(-1)
        assert raw.size == n, "host array and tensor sizes differ"
        hbuf[o:o + n].copy_(torch.from_numpy(raw))
    return dbuf, hbuf, views


def max_over_ranks(values, world, device):
    """Each rank's timings -> the maximum over the ranks, on every rank (the
    replicas' device times; the whole job is as slow as its slowest rank)."""
    import torch

    vals = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist

        dist.all_reduce(vals, op=dist.ReduceOp.MAX)
    return [float(v) for v in vals]


def selection_name(args):
    return f"static top-k, k={args.topk}" if args.topk > 0 else ("top-p, p=1 (dense)" if args.dense else "top-p")


def cpu_model():
    """The host CPU's model name (from /proc/cpuinfo), or None."""
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def oracle_single_thread(case, tokens, topk=0, budget_s=5.0):
    """The oracle on one host thread: whole steps until about budget_s have
    passed (at least one).  Returns a dict for the cpu_baseline entry."""
    import oracle

    reps, t0 = 0, time.perf_counter()
    while reps == 0 or (time.perf_counter() - t0 < budget_s and reps < 20):
        if topk > 0:
            oracle.decode_step_topk(case, topk, nthreads=1)
        else:
            oracle.decode_step(case, nthreads=1)
        reps += 1
    t = (time.perf_counter() - t0) / reps
    return {"value": tokens / t, "s_per_step": t, "sample": f"{reps} whole decode steps, 1 thread"}


def run_reference(args, rank):
    """The oracle (fp64 C, OpenMP over heads) on the host cores, same workload."""
    if rank != 0:
        return
    import oracle
    import synth

    case = synth.workload(args.workload, scale=args.scale)
    if args.dense:
        case.p[:] = 1.0
    cores = os.cpu_count() or 1

    def step():
        if args.topk > 0:
            oracle.decode_step_topk(case, args.topk, nthreads=cores)
        else:
            oracle.decode_step(case, nthreads=cores)

    for _ in range(args.warmup):
        step()
    ts = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        step()
        ts.append(time.perf_counter() - t0)
    t = statistics.mean(ts)
    tokens = float(case.seq_lens.sum())
    v = tokens / t
    single = oracle_single_thread(case, tokens, args.topk)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(workload_config(case, args.workload), selection=selection_name(args)),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "cpu_model": cpu_model(),
                             "sample": f"whole decode step of the workload per timed step ({args.steps} steps)",
                             "single_thread": single},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def bench_append(args):
    """rtp_index_append alone (--op append) or rtp_kv_append (--op kv_append):
    a decode-sized append (one new token for each of 16 sequences x 8 KV
    heads) and a 32K-token chunk of one sequence.  HBM bytes per token and KV
    head: k_pre read (256 B) + k_idx written (32 B); kv_append adds the new
    value read (256 B) and the key and value rows written (512 B), and the
    angle table row (512 B) once per position.  W^K (32 KB) stays in L2.  L2
    flushed before every timed call."""
    kv = args.op == "kv_append"
    import torch

    import sparse_attention_decode_rtpurbo_b200 as rtp

    dev = torch.device("cuda", 0)
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    peak, peak_kind = hbm_peak()
    for name, B, Hkv, T, ncap in [("decode 16x8 heads x 1 token", 16, 8, 1, 65536),
                                  ("chunk 1x8 heads x 32768 tokens", 1, 8, 32768, 65536)]:
        g = torch.Generator(device=dev).manual_seed(1)
        k_pre = torch.randn((B, Hkv, T, 128), generator=g, device=dev).to(torch.bfloat16)
        Wk = (torch.randn((Hkv, 16, 128), generator=g, device=dev) / 11.3).to(torch.bfloat16)
        pos = torch.zeros(B, dtype=torch.int32, device=dev)
        cache = torch.zeros((B, Hkv, ncap, 16), dtype=torch.bfloat16, device=dev)
        if kv:
            v_new = torch.randn((B, Hkv, T, 128), generator=g, device=dev).to(torch.bfloat16)
            ang = torch.rand((ncap, 64), generator=g, device=dev, dtype=torch.float64) * 6.283
            rc, rs = torch.cos(ang).float(), torch.sin(ang).float()
            kc = torch.zeros((B, Hkv, ncap, 128), dtype=torch.bfloat16, device=dev)
            vc = torch.zeros((B, Hkv, ncap, 128), dtype=torch.bfloat16, device=dev)
        dims = rtp.make_dims(B, Hkv, Hkv, ncap)
        stream = torch.cuda.current_stream()
        ts = []
        for i in range(args.warmup + args.steps):
            flush_w.zero_()
            a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            if kv:
                rtp.kv_append(dims, k_pre, v_new, Wk, rc, rs, pos, T, cache, kc, vc, None, stream)
            else:
                rtp.index_append(dims, k_pre, Wk, pos, T, cache, None, stream)
            z.record(stream)
            z.synchronize()
            if i >= args.warmup:
                ts.append(a.elapsed_time(z))
        t_ms = statistics.median(ts)
        nbytes = B * Hkv * T * (256 + 32 + (256 + 512 if kv else 0)) + (T * 512 if kv else 0)
        gbs = nbytes / (t_ms * 1e-3) / 1e9
        metric = "KV-cache write + index append (rtp_kv_append)" if kv else "index-cache append (rtp_index_append)"
        print(json.dumps({"metric": metric, "op": args.op, "case": name,
                          "value": gbs, "unit": "GB/s", "us_per_call": t_ms * 1e3, "bytes": nbytes,
                          "peak": peak, "frac": gbs / peak, "peak_source": peak_kind, "steps": args.steps,
                          "warmup": args.warmup, "l2": "flushed (256 MB write) before every call"}), flush=True)


class StepBench:
    """One workload on the device, ready to time: its inputs staged in one
    device buffer (so the end-to-end leg makes one host-to-device copy), a
    CUDA graph of one rtp_decode_step, and a second graph that records the
    library's phase events between its kernels."""

    def __init__(self, case, args, dev, flush):
        import ctypes

        import torch

        import sparse_attention_decode_rtpurbo_b200 as rtp
        from synth.torch_io import DeviceCase

        self.case, self.dev, self.flush = case, dev, flush
        self.stream = torch.cuda.current_stream(dev)
        dc = DeviceCase(case, device=dev, debug=True)
        dc.topk = max(0, args.topk)
        self.dbuf, self.hbuf, views = stage_inputs(
            [dc.q_pre, dc.q_rope, dc.seq_lens, dc.p],
            [case.q_pre, case.q_rope, case.seq_lens.astype(np.int32), case.p.astype(np.float32)], dev)
        dc.q_pre, dc.q_rope, dc.seq_lens, dc.p = views
        self.dc = dc
        # one debug step: kept blocks for the algorithmic byte count
        dc.run(self.stream)
        res = dc.results()
        if res["status"] != 0:
            raise SystemExit(f"device status {res['status']}")
        self.nbytes = algorithmic_bytes(case, res["kept"])
        ret = np.nonzero(case.head_kind)[0]
        self.kept_tokens = float(np.mean([res["kstar"][b, h] / case.seq_lens[b] for b in range(case.B)
                                          for h in ret])) if ret.size else 0.0
        self.kept_blocks = float(np.mean([res["kept_blocks"][b, h] / ((case.seq_lens[b] + 63) // 64)
                                          for b in range(case.B) for h in ret])) if ret.size else 0.0
        dc.step.dims.debug = ctypes.POINTER(rtp.RtpDebug)()   # timed steps run without diagnostics
        self.inner = [torch.cuda.Event(enable_timing=True) for _ in range(rtp.TIMING_EVENTS)]
        for e in self.inner:
            e.record(self.stream)
        dc.run(self.stream)                                   # eager warm-up (sets kernel attributes)
        torch.cuda.synchronize(dev)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            dc.run(torch.cuda.current_stream(dev))
        dc.step.set_timing_events(self.inner)
        self.graph_ev = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph_ev):
            dc.run(torch.cuda.current_stream(dev))
        dc.step.set_timing_events(None)

    def warm(self, n):
        import torch

        for _ in range(n):
            self.flush()
            self.graph.replay()
            self.flush()
            self.graph_ev.replay()
        torch.cuda.synchronize(self.dev)

    def timed(self, steps, replay=None):
        """Device time (ms) of each of `steps` graph replays, L2 flushed before each."""
        import torch

        replay = replay or self.graph.replay
        out = []
        for _ in range(steps):
            self.flush()
            a = torch.cuda.Event(enable_timing=True)
            z = torch.cuda.Event(enable_timing=True)
            a.record(self.stream)
            replay()
            z.record(self.stream)
            z.synchronize()
            out.append(a.elapsed_time(z))
        return out

    def phases(self, steps):
        import sparse_attention_decode_rtpurbo_b200 as rtp

        acc = [0.0] * len(rtp.PHASES)
        for _ in range(steps):
            self.flush()
            self.graph_ev.replay()
            self.inner[-1].synchronize()
            for k in range(len(rtp.PHASES)):
                acc[k] += self.inner[k].elapsed_time(self.inner[k + 1])
        return {n: acc[k] / steps for k, n in enumerate(rtp.PHASES)}

    def timeline(self, reps=5):
        """Median over `reps` debug-traced steps of the library's timeline (us since the first CTA)."""
        import ctypes

        import torch

        import sparse_attention_decode_rtpurbo_b200 as rtp

        dc = self.dc
        trace_buf = torch.zeros(rtp.TRACE_WORDS, dtype=torch.int64, device=self.dev)
        tdbg = rtp.RtpDebug(trace=trace_buf.data_ptr())
        dc.step.dims.debug = ctypes.pointer(tdbg)
        tl = []
        for _ in range(reps):
            self.flush()
            trace_buf.zero_()
            dc.run(self.stream)
            torch.cuda.synchronize(self.dev)
            t = trace_buf.cpu().numpy().astype(np.float64)
            ev = {n: (t[k] - t[0]) / 1e3 if t[k] > 0 else None for k, n in enumerate(rtp.TRACE_EVENTS) if k}
            for k, n in enumerate(rtp.TRACE_SUMS):
                v = t[16 + k]
                ev[n] = ((v - t[0]) / 1e3 if v > 0 else None) if n in rtp.TRACE_SUM_EVENTS else v
            tl.append(ev)
        dc.step.dims.debug = ctypes.POINTER(rtp.RtpDebug)()
        return {n: (statistics.median([x[n] for x in tl]) if tl[0][n] is not None else None) for n in tl[0]}

    def e2e(self, steps, warmup):
        """End to end through the public call: each step copies the staged
        per-step inputs host -> device (one pinned copy), calls
        rtp_decode_step eagerly through the Python binding (argument
        checks, workspace plan and tensor maps on the host every call), and
        copies the output device -> host.  Also the same with the captured
        graph in place of the eager call."""
        import torch

        dc = self.dc
        hout = torch.empty(dc.out.shape, dtype=torch.bfloat16).pin_memory()

        def leg(call):
            ts = []
            for i in range(warmup + steps):
                self.flush()
                a = torch.cuda.Event(enable_timing=True)
                z = torch.cuda.Event(enable_timing=True)
                a.record(self.stream)
                self.dbuf.copy_(self.hbuf, non_blocking=True)
                call()
                hout.copy_(dc.out, non_blocking=True)
                z.record(self.stream)
                z.synchronize()
                if i >= warmup:
                    ts.append(a.elapsed_time(z))
            return statistics.mean(ts)

        eager = leg(lambda: dc.run(self.stream))
        graph = leg(self.graph.replay)
        return eager, graph, self.hbuf.numel(), hout.numel() * hout.element_size()

    def dense(self, steps, warmup):
        """The same captured step with p = 1 for every sequence (every block
        of every retrieval head): the stand-in for the pages' dense-attention
        baseline.  Returns (mean ms, device status)."""
        import torch

        dc, case = self.dc, self.case
        dc.p.fill_(1.0)
        dts = self.timed(warmup + steps)[warmup:]
        dc.p.copy_(torch.from_numpy(case.p.astype(np.float32)).to(self.dev))
        torch.cuda.synchronize(self.dev)
        return statistics.mean(dts), dc.step.status()

    def status(self):
        return self.dc.step.status()


def step_summary(sb, step_ms, peak, dense_ms=0.0, dense_status=0):
    """us/step (mean, median, p10/p90), context-tokens/s and the step's HBM fraction."""
    t_ms = statistics.mean(step_ms)
    tokens = float(sb.case.seq_lens.sum())
    gbs = sb.nbytes["total"] / (t_ms * 1e-3) / 1e9
    d = {"us_per_step": t_ms * 1e3, "us_per_step_median": statistics.median(step_ms) * 1e3,
         "us_per_step_p10_p90": [float(np.percentile(step_ms, 10)) * 1e3, float(np.percentile(step_ms, 90)) * 1e3],
         "context_tokens_per_s": tokens / (t_ms * 1e-3),
         "step_roofline": {"algorithmic_bytes": sb.nbytes, "achieved": gbs, "peak": peak, "unit": "GB/s",
                           "frac": gbs / peak},
         "sparsity": {"kept_token_frac": sb.kept_tokens, "kept_block_frac": sb.kept_blocks}}
    if dense_ms > 0:
        d["dense_comparator"] = {"us_per_step": dense_ms * 1e3, "value": tokens / (dense_ms * 1e-3), "unit": UNIT,
                                 "speedup_of_sparse": dense_ms / t_ms, "device_status": dense_status,
                                 "what": "the same step with p = 1 (every block of every retrieval head)"}
    return d


# the other workloads of the metric's range (32K to 1M), timed after the
# headline with fewer steps; the 4K workload is a parity case only
OTHER_WORKLOADS = (2, 3, 5)


def prefill_flops(T, pos, head_kind, window, sink):
    """Multiply-add flops of a prefill chunk: 4 x 128 per attended (query,
    key) pair (q.k and p.v), summed over heads; query t attends m + 1 keys
    (retrieval) or its sink and window (local), m = pos + t."""
    m = pos + np.arange(T, dtype=np.int64)
    dense = m + 1
    local = np.minimum(sink, m + 1) + np.maximum(0, (m + 1) - np.maximum(sink, m + 1 - window))
    nret = int(np.sum(head_kind))
    nloc = len(head_kind) - nret
    return 4 * 128 * (nret * int(dense.sum()) + nloc * int(local.sum()))


def bench_prefill(args):
    """rtp_prefill alone: the prefill of a whole 32K prompt (B=1, 8 KV heads x
    GQA 4, KV group 0 retrieval = 4 of 32 heads, the rest local with window
    8192 and sink 4, the pages' prefill setting), and the same prompt with
    every head retrieval (dense causal attention, the stand-in for the pages'
    dense baseline).  Tensor-core bound: flops / time against the measured
    bf16 peak.  L2 flushed before every timed call."""
    import torch

    import sparse_attention_decode_rtpurbo_b200 as rtp

    dev = torch.device("cuda", 0)
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    B, Hkv, G, T = 1, 8, 4, 32768 // max(1, args.scale)
    window, sink = 8192 // max(1, args.scale), 4
    ncap = (T + 63) // 64 * 64
    g = torch.Generator(device=dev).manual_seed(7)
    q = torch.randn((B, Hkv * G, T, 128), generator=g, device=dev).to(torch.bfloat16)
    k = torch.randn((B, Hkv, ncap, 128), generator=g, device=dev).to(torch.bfloat16)
    v = torch.randn((B, Hkv, ncap, 128), generator=g, device=dev).to(torch.bfloat16)
    pos = torch.zeros(B, dtype=torch.int32, device=dev)
    out = torch.empty((B, Hkv * G, T, 128), dtype=torch.bfloat16, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    dims = rtp.make_dims(B, Hkv * G, Hkv, ncap)
    stream = torch.cuda.current_stream()
    try:
        peak = float(json.load(open(PEAKS_FILE))["bf16_tflops"])
        peak_kind = "measured (MEASURED_PEAKS.json bf16_tflops, burst)"
    except Exception:
        peak, peak_kind = 1590.0, "fallback"
    res = {}
    kernel = ("mma.sync m16n8k16 bf16" if os.environ.get("RTP_PREFILL_TC") == "0"
              else "tcgen05, 128-key tiles, two row groups per CTA (tensor memory, TMA)")
    for name, hk in (("sparse", [1] * G + [0] * (Hkv - 1) * G), ("dense", [1] * (Hkv * G))):
        ts = []
        for i in range(args.warmup + args.steps):
            flush_w.zero_()
            a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            rtp.prefill(dims, q, k, v, hk, pos, T, window, sink, out, status, stream)
            z.record(stream)
            z.synchronize()
            if i >= args.warmup:
                ts.append(a.elapsed_time(z))
        if int(status.item()) != 0:
            raise SystemExit(f"prefill device status {int(status.item())}")
        t_ms = statistics.mean(ts)
        fl = prefill_flops(T, 0, np.array(hk), window, sink)
        tf = fl / (t_ms * 1e-3) / 1e12
        res[name] = {"ms_per_call": t_ms, "flops": fl, "tflops": tf, "frac": tf / peak,
                     "tokens_per_s": B * T / (t_ms * 1e-3)}
    print(json.dumps({"metric": "prefill tokens/s (rtp_prefill, whole prompt)", "op": "prefill",
                      "value": res["sparse"]["tokens_per_s"], "unit": "tokens/s",
                      "config": {"batch": B, "prompt": T, "q_heads": Hkv * G, "kv_heads": Hkv, "retrieval_heads": G,
                                 "window": window, "sink": sink, "l2": "flushed (256 MB write) before every call"},
                      "roofline": {"bound": "tensor", "achieved": res["sparse"]["tflops"], "peak": peak,
                                   "unit": "TFLOP/s", "frac": res["sparse"]["frac"], "peak_source": peak_kind,
                                   "kernel": f"rtp_prefill: {kernel}"},
                      "sparse": res["sparse"], "dense_all_heads_retrieval": res["dense"],
                      "speedup_over_dense": res["dense"]["ms_per_call"] / res["sparse"]["ms_per_call"],
                      "steps": args.steps, "warmup": args.warmup}), flush=True)


def main():
    args = parse()
    if args.op in ("append", "kv_append"):
        return bench_append(args)
    if args.op == "prefill":
        return bench_prefill(args)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return

    import torch
    import torch.distributed as dist

    import sparse_attention_decode_rtpurbo_b200 as rtp
    import synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    # L2 flush between timed steps: write 256 MB, then read another 256 MB so
    # the dirty lines of the write are evicted before the step, not during it
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(256 << 20, dtype=torch.uint8, device=dev)

    def flush():
        flush_w.zero_()
        flush_r.sum(dtype=torch.int64)

    case = synth.workload(args.workload, scale=args.scale)
    if args.dense:
        case.p[:] = 1.0
    sb = StepBench(case, args, dev, flush)
    sb.warm(max(3, args.warmup))

    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize(dev)
    t_begin = time.perf_counter()
    step_ms = sb.timed(args.steps)
    torch.cuda.synchronize(dev)
    barrier()
    wall = time.perf_counter() - t_begin
    clocks = sampler.stop()
    phase_ms = sb.phases(args.steps)
    timeline = sb.timeline()
    e2e_t, e2e_graph_t, h2d, d2h = sb.e2e(args.steps, max(3, args.warmup))
    if sb.status() != 0:
        raise SystemExit("device status set during the timed steps")
    dense_ms, dense_status = 0.0, 0
    if not args.no_dense_comparator and not args.dense and args.topk == 0 and case.head_kind.any():
        dense_ms, dense_status = sb.dense(args.steps, max(3, args.warmup))

    # ---- max over ranks ----
    t_ms = statistics.mean(step_ms)
    vals = max_over_ranks([t_ms, e2e_t, e2e_graph_t, dense_ms] + [phase_ms[n] for n in rtp.PHASES], world, dev)
    t_ms, e2e_t, e2e_graph_t, dense_ms = vals[:4]
    phase_ms = {n: vals[4 + k] for k, n in enumerate(rtp.PHASES)}

    tokens = float(case.seq_lens.sum())
    value = world * tokens / (t_ms * 1e-3)
    peak, peak_kind = hbm_peak()
    # two launches per step: rtp::stream_kernel (index cache + local heads'
    # sink/window K/V) and, when there are retrieval heads,
    # rtp::retrieve_kernel (kept K/V blocks; exact select when needed).
    # The roofline is reported for the one that takes longer.
    nbytes = sb.nbytes
    kbytes = {"stream": nbytes["index"] + nbytes["local"], "retrieve": nbytes["kept_kv"]}
    has_ret = bool(case.head_kind.any())
    dom = "retrieve" if has_ret and phase_ms["retrieve"] > phase_ms["stream"] else "stream"
    ach = kbytes[dom] / (phase_ms[dom] * 1e-3) / 1e9
    launches_per_step = 2 if has_ret else 1
    summary = step_summary(sb, step_ms, peak, dense_ms, dense_status)
    del sb
    torch.cuda.empty_cache()

    # ---- the metric's other context lengths (32K, 4 x 128K, ragged paged) ----
    per_workload = {}
    if args.workload == 4 and args.scale == 1 and not args.dense and args.topk == 0 and not args.no_per_workload:
        for wl in OTHER_WORKLOADS:
            c2 = synth.workload(wl)
            s2 = StepBench(c2, args, dev, flush)
            s2.warm(3)
            ms2 = s2.timed(max(5, args.steps // 2))
            dm2, ds2 = s2.dense(max(5, args.steps // 2), 3) if c2.head_kind.any() else (0.0, 0)
            st2 = s2.status()
            ms2_max = max_over_ranks([statistics.mean(ms2), dm2], world, dev)
            entry = step_summary(s2, ms2, peak, dm2, ds2)
            entry["us_per_step_max_over_ranks"] = ms2_max[0] * 1e3
            entry["config"] = workload_config(c2, wl)
            entry["device_status"] = st2
            per_workload[synth.WORKLOADS[wl]] = entry
            del s2
            torch.cuda.empty_cache()

    line = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            import oracle

            cores = os.cpu_count() or 1
            def oracle_step():
                if args.topk > 0:
                    oracle.decode_step_topk(case, args.topk, nthreads=cores)
                else:
                    oracle.decode_step(case, nthreads=cores)

            oracle_step()
            reps, t0 = 0, time.perf_counter()
            while time.perf_counter() - t0 < 10.0 and reps < 50:
                oracle_step()
                reps += 1
            tc = (time.perf_counter() - t0) / reps
            cpu = {"value": tokens / tc, "unit": UNIT, "cores": cores, "kind": "oracle", "cpu_model": cpu_model(),
                   "sample": f"{reps} whole decode steps of this workload (fp64 C oracle, OpenMP over heads)",
                   "single_thread": oracle_single_thread(case, tokens, args.topk)}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t_ms, "us_per_step": t_ms * 1e3,
            "us_per_step_median": summary["us_per_step_median"],
            "us_per_step_p10_p90": summary["us_per_step_p10_p90"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16 in, fp32 accumulate",
            "data": "synthetic (seeded generators in synth/, shaped like the pages' workloads)",
            "config": dict(workload_config(case, args.workload), parallelism=f"replicas x{world}",
                           dense_p1=bool(args.dense), selection=selection_name(args), timing="CUDA-graph replay of one rtp_decode_step (2 kernels, programmatic launch) per step; "
                           "CUDA events on the launching stream; value from the mean step time"),
            "wall_s_timed_loop": wall,
            "roofline": {"bound": "hbm", "kernel": f"rtp::{dom}_kernel", "achieved": ach, "peak": peak, "unit": "GB/s",
                         "frac": ach / peak, "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs, burst)",
                         "traffic": profiled_traffic(dom, case.name) if selection_name(args) == "top-p" else None,
                         "algorithmic_bytes_per_launch": kbytes[dom],
                         "us_per_launch": phase_ms[dom] * 1e3},
            "step_roofline": summary["step_roofline"],
            "phases_us": {n: phase_ms[n] * 1e3 for n in rtp.PHASES},
            "timeline_us": timeline,
            "sparsity": summary["sparsity"],
            "e2e": {"value": world * tokens / (e2e_t * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "us_per_step": e2e_t * 1e3,
                    "what": "eager rtp_decode_step through the Python binding per step (host checks, plan and "
                            "tensor maps included), inputs host->device in one pinned copy, output device->host",
                    "graph_replay": {"value": world * tokens / (e2e_graph_t * 1e-3), "us_per_step": e2e_graph_t * 1e3,
                                     "what": "the same with the captured graph in place of the eager call"}},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
            "cpu_baseline": cpu,
            "dense_comparator": summary.get("dense_comparator"),
            "per_workload": per_workload or None,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
