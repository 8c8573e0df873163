"""Benchmark of the sink-attention hot path on B200.

One step = forward + backward of one sliding-window layer (window 128) and
one full-causal layer of gpt-oss attention shapes (B=4, S=4096, 64 query
heads, 8 key/value heads, head dim 64, scale 1/8), on synthetic seeded bf16
inputs already resident in HBM.  The metric is TFLOP/s on unmasked FLOPs
(forward 4*D per allowed (query, key, head) triple, backward 10*D), counted
exactly from the mask.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched by torchrun) every rank runs its own replica of the
workload on its own GPU (the path has no exchange step: replicas only, weak
scaling); the reported time is the max over ranks.  Rank 0 prints one JSON
line.

--impl reference times the fp64 CPU oracle (the correctness reference) on a
bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from sink_sliding_window_b200 import synth  # noqa: E402

WORKLOAD = "prefill4k"
B, S, HQ, HKV, D = 4, 4096, 64, 8, 64
LAYERS = (128, 0)  # window per layer: sliding window 128, then full causal
# The forward kernels timed one by one next to sink_attn_fwd's own choice.
FWD_KERNEL_NAMES = ("one_tile", "two_tiles", "pair")
METRIC = "sink-attn fwd/bwd TFLOP/s (unmasked FLOPs) and % of B200 bf16 tensor peak"


# ------------------------------------------------------------------ work
def pairs(cu_seqlens, window, Hq):
    """Allowed (query, key, head) triples, counted exactly from the mask."""
    c = np.asarray(cu_seqlens, np.int64)
    tot = 0
    for b in range(len(c) - 1):
        i = np.arange(int(c[b + 1] - c[b]), dtype=np.int64)
        n = i + 1 if window <= 0 else np.minimum(i + 1, window)
        tot += int(n.sum())
    return tot * Hq


def layer_flops(window):
    p = pairs(synth.uniform_cu_seqlens(B, S), window, HQ)
    return 4 * D * p, 10 * D * p


def step_flops():
    return sum(sum(layer_flops(w)) for w in LAYERS)


# ------------------------------------------------------------- CPU sample
_SAMPLE_CACHE = {}


def _sample_inputs(seed):
    if seed not in _SAMPLE_CACHE:
        _SAMPLE_CACHE[seed] = synth.workload(f"{WORKLOAD}:w128", seed=seed).generate(with_dout=True)
    return _SAMPLE_CACHE[seed]


def oracle_sample(len_window=S, len_full=1024, seed=0, nthreads=0):
    """Bounded sample of the workload for the CPU oracle: forward+backward
    (the oracle's backward recomputes the forward rows) restricted to 4 of
    the 8 key/value heads (and their 32 query heads), all 4 documents:
      - the window-128 layer on the first `len_window` tokens of each
        document, and
      - the full-causal layer on the first `len_full` tokens of each document.
    The oracle parallelises over (document, key/value head) tasks: 16 here.
    Returns (seconds, flops, description, threads)."""
    import oracle

    a = _sample_inputs(seed)
    G = HQ // HKV
    groups = [0, 2, 5, 7]
    heads = np.concatenate([np.arange(g * G, (g + 1) * G) for g in groups])
    flops = 0
    secs = 0.0
    for window, length in ((128, len_window), (0, len_full)):
        rows = np.concatenate([np.arange(b * S, b * S + length) for b in range(B)])
        q = np.ascontiguousarray(a["q"][rows][:, heads])
        k = np.ascontiguousarray(a["k"][rows][:, groups])
        v = np.ascontiguousarray(a["v"][rows][:, groups])
        do = np.ascontiguousarray(a["dout"][rows][:, heads])
        cu = synth.uniform_cu_seqlens(B, length)
        t0 = time.perf_counter()
        oracle.bwd(q, k, v, a["sinks"][heads], cu, window, 1.0 / 8.0, do, nthreads=nthreads)
        secs += time.perf_counter() - t0
        flops += (4 + 10) * D * pairs(cu, window, len(heads))
    desc = (f"fp64 oracle fwd+bwd, 4 documents x 4 of 8 KV heads (32 query heads): window-128 layer on the first "
            f"{len_window} tokens and full-causal layer on the first {len_full} tokens of each document")
    return secs, flops, desc, oracle.max_threads() if nthreads <= 0 else nthreads


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_id}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 7:
                continue
            try:
                sm.append(float(f[0]))
                smax.append(float(f[1]))
            except ValueError:
                continue
            for n, v in zip(names, f[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


def gpu_id_for(torch, dev):
    try:
        p = torch.cuda.get_device_properties(dev)
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        return vis.split(",")[dev] if vis else str(dev)


# ---------------------------------------------------------------- helpers
def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return float(pk["bf16_tflops"]), float(pk["hbm_gbs"]), "measured"
    return 1590.0, 6650.0, "fallback"


# Sources the backward main kernel is compiled from (its measured DRAM
# traffic is reported only while their code is unchanged).
BWD_MAIN_SOURCES = ("bwd_kernels.cuh", "common.cuh", "ptx.cuh", "tmem_io.cuh", "tma_host.cuh")


def _code_only(text):
    """C/C++ source without its comments and blank lines (string literals in
    these headers hold no comment markers)."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def kernel_source_hash():
    """Hash of the code (comments excluded) of BWD_MAIN_SOURCES."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sink_sliding_window_b200", "csrc")
    for n in BWD_MAIN_SOURCES:
        with open(os.path.join(csrc, n), encoding="utf-8") as f:
            h.update(n.encode() + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


def measured_traffic():
    """DRAM bytes per launch of the backward main kernel on this workload,
    from the committed ncu summary; None when the kernels changed since."""
    path = os.path.join(ROOT, "profiles", "bwd_main_prefill4k_full.traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    return t.get("dram_bytes_per_launch") if t.get("kernel_source_hash") == kernel_source_hash() else None


# --------------------------------------------------------------- decode
DECODE_CASES = (
    # (name, sequences, cached tokens, new tokens, cache slots, window, e4m3 cache)
    ("decode 64 seqs x 8191 cached + 1 new, full-causal layer, linear 8192-slot cache", 64, 8191, 1, 8192, 0, False),
    ("decode 64 seqs x 8191 cached + 1 new, window-128 layer, 128-slot ring", 64, 8191, 1, 128, 128, False),
    ("decode 64 seqs x 8191 cached + 1 new, full-causal layer, linear 8192-slot e4m3 cache", 64, 8191, 1, 8192, 0,
     True),
    ("decode 64 seqs x 8191 cached + 1 new, full-causal layer, linear 8192-slot e4m3 cache, FP8 PV product", 64, 8191,
     1, 8192, 0, "f8pv"),
)


def measure_decode(torch, ops, stream, iters=20):
    """Times sink_attn_decode (append + attend + combine) on gpt-oss heads with
    CUDA events on the launching stream, writing a 256 MiB buffer between
    iterations so that no K/V tile is served from L2.  Bandwidth counts the
    K and V bytes the new queries must read (every cached key they can see)."""
    _, hbm, kind = read_peaks()
    res = []
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    for name, Bd, L0, Lq, C, W, f8 in DECODE_CASES:
        a = synth.decode_inputs(7, [0], Lq, HQ, HKV)  # sinks and new-token rows
        g = torch.Generator(device="cuda").manual_seed(7)
        mk = lambda *shape: torch.randn(*shape, device="cuda", generator=g).to(torch.bfloat16)  # noqa: E731
        q, kn, vn = mk(Bd, Lq, HQ, D), mk(Bd, Lq, HKV, D), mk(Bd, Lq, HKV, D)
        if f8:
            # The N(0,1) bf16 history quantised to e4m3 with one scale per KV
            # head (amax / 448), as an FP8 cache would hold it (input preparation
            # only; the timed call reads the codes).
            def quantised():
                x = mk(Bd, C, HKV, D).float()
                sc = x.abs().amax(dim=(0, 1, 3)) / 448.0
                return (x / sc[None, None, :, None]).to(torch.float8_e4m3fn).view(torch.uint8), sc
            kc, k_scale = quantised()
            vc, v_scale = quantised()
        else:
            kc, vc = mk(Bd, C, HKV, D), mk(Bd, C, HKV, D)
        sl = torch.full((Bd,), L0, dtype=torch.int32, device="cuda")
        sinks = torch.from_numpy(a["sinks"]).cuda()
        ws = torch.empty((ops.decode_workspace_size(Bd, Lq, C, L0 + Lq, HQ, HKV, W),), dtype=torch.uint8,
                         device="cuda")
        out = torch.empty_like(q)
        lse = torch.empty((HQ, Bd * Lq), dtype=torch.float32, device="cuda")

        def call():
            if f8:
                ops.decode_e4m3(q, kn, vn, kc, vc, sl, k_scale, v_scale, sinks, W, 0.125, max_seqlen=L0 + Lq, out=out,
                                lse=lse, workspace=ws, stream=stream, f8pv=f8 == "f8pv")
            else:
                ops.decode(q, kn, vn, kc, vc, sl, sinks, W, 0.125, max_seqlen=L0 + Lq, out=out, lse=lse,
                           workspace=ws, stream=stream)
        for _ in range(3):
            call()
        torch.cuda.synchronize()
        tot = 0.0
        for _ in range(iters):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            call()
            e1.record(stream)
            torch.cuda.synchronize()
            tot += e0.elapsed_time(e1)
        if ops.device_error() != 0:
            raise RuntimeError("a decode kernel reported an error")
        ms = tot / iters
        keys = min(L0 + Lq, C) if W <= 0 else min(L0 + Lq, W + Lq - 1, C)
        kv = Bd * keys * HKV * D * 2 * (1 if f8 else 2)  # K and V bytes as stored
        res.append({"workload": name, "us": ms * 1e3, "kv_bytes": kv, "achieved_GBps": kv / ms / 1e6,
                    "peak_GBps": hbm, "frac": kv / ms / 1e6 / hbm, "peak_source": f"{kind} hbm_gbs",
                    "launches": ops.decode_launches(Bd, Lq, C, L0 + Lq, HQ, HKV, W)})
    return res


def time_calls(torch, stream, fns, iters, rounds=4, warm=2):
    """ms per call of each function in `fns`: CUDA events on the launching
    stream around `iters` calls, in `rounds` rounds that take the functions in
    turn (in reverse order every other round), so that clock changes under the
    power cap fall on all of them alike; the median over the rounds."""
    for fn in fns.values():
        for _ in range(warm):
            fn()
    torch.cuda.synchronize()
    keys = list(fns)
    times = {k: [] for k in keys}
    for r in range(rounds):
        for k in (keys if r % 2 == 0 else keys[::-1]):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(iters):
                fns[k]()
            e1.record(stream)
            torch.cuda.synchronize()
            times[k].append(e0.elapsed_time(e1) / iters)
    return {k: statistics.median(v) for k, v in times.items()}


def measure_layers(torch, ops, stream, q, k, v, sinks, dout, outs, grads, ws, iters=10):
    """Forward and backward of each layer alone (time_calls: CUDA events on
    the launching stream, the forward kernels taken in turn): TFLOP/s on the
    counted pairs, and GB/s of the layer's minimum DRAM bytes (every input
    read once, every output written once) against the measured HBM peak; the
    window-128 layers are rated by the latter.  "fwd" is sink_attn_fwd (the
    kernel it picks is named), "fwd_kernels" each forward kernel through
    sink_attn_fwd_with.  q, dout, out and dq (134 MB each) exceed the 126 MB
    L2, so no flush between calls."""
    _, hbm, kind = read_peaks()
    nb = lambda *ts: sum(t.numel() * t.element_size() for t in ts)  # noqa: E731
    res = []
    for W in LAYERS:
        o, l = outs[W]
        dq, dk, dv, ds = grads[W]
        kw = dict(batch=B, max_seqlen=S, stream=stream)
        fwd_bytes = nb(q, k, v, sinks) + nb(o, l)
        bwd_bytes = nb(q, k, v, sinks, o, l, dout) + nb(dq, dk, dv, ds)
        fwd = {"fwd": lambda: ops.fwd(q, k, v, sinks, None, W, 0.125, out=o, lse=l, **kw)}
        for kn in FWD_KERNEL_NAMES:
            fwd["fwd:" + kn] = (lambda kn=kn: ops.fwd(q, k, v, sinks, None, W, 0.125, out=o, lse=l, kernel=kn,
                                                      **kw))
        ms = time_calls(torch, stream, fwd, iters)
        # the backward reads the saved out / lse of the last forward call
        ops.fwd(q, k, v, sinks, None, W, 0.125, out=o, lse=l, **kw)
        ms.update(time_calls(torch, stream, {"bwd": lambda: ops.bwd(q, k, v, sinks, o, l, dout, None, W, 0.125, dq=dq,
                                                                      dk=dk, dv=dv, dsinks=ds, workspace=ws, **kw)},
                             iters, rounds=2))
        fl = dict(zip(("fwd", "bwd"), layer_flops(W)))
        entry = {"window": W, "workload": f"{WORKLOAD} ({'window %d' % W if W > 0 else 'full causal'})"}
        for name, t in ms.items():
            base = name.split(":")[0]
            mb = fwd_bytes if base == "fwd" else bwd_bytes
            r = {"ms": t, "tflops": fl[base] / t / 1e9, "min_bytes": mb, "GBps": mb / t / 1e6,
                 "hbm_frac": mb / t / 1e6 / hbm}
            if ":" in name:
                entry.setdefault("fwd_kernels", {})[name.split(":")[1]] = r
            else:
                entry[name] = r
        entry["fwd"]["kernel"] = ops.fwd_kernel_for(B * S, HQ, HKV, D, B, S, W)
        entry["peak_GBps"] = hbm
        entry["peak_source"] = f"{kind} hbm_gbs"
        res.append(entry)
    if ops.device_error() != 0:
        raise RuntimeError("a kernel reported a timed-out wait")
    return res


# ------------------------------------------------- long and packed shapes
EXTRA_WORKLOADS = ("long60k", "varlen64k")


def device_inputs(torch, w, seed=11, with_dout=True):
    """Device-resident N(0,1) bf16 q, k, v (and dout) of a workload's shapes,
    drawn on the GPU from a seeded generator (the timing does not depend on
    the exact values, and drawing 0.5 G values on the host would dominate
    the run), and the workload's own sinks."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    mk = lambda *shape: torch.randn(*shape, generator=g, device="cuda").to(torch.bfloat16)  # noqa: E731
    t = {"q": mk(w.T, w.Hq, w.D), "k": mk(w.T, w.Hkv, w.D), "v": mk(w.T, w.Hkv, w.D),
         "sinks": torch.from_numpy(w.sinks_only()).cuda()}
    if with_dout:
        t["dout"] = mk(w.T, w.Hq, w.D)
    t["cu"] = None if w.uniform_seqlen is not None else torch.from_numpy(w.cu_seqlens).cuda()
    return t


def layer_calls(ops, w, t, stream, window, bufs):
    """(forward call, backward call) of one layer of workload w on the
    device tensors t, writing into bufs = (out, lse, dq, dk, dv, dsinks, ws)."""
    o, l, dq, dk, dv, ds, ws = bufs
    if w.uniform_seqlen is not None:
        kw = dict(batch=w.batch, max_seqlen=w.uniform_seqlen, stream=stream)
    else:
        kw = dict(max_seqlen=w.max_seqlen, stream=stream)
    f = lambda kernel="auto": ops.fwd(t["q"], t["k"], t["v"], t["sinks"], t["cu"], window, w.scale,  # noqa
                                      out=o, lse=l, kernel=kernel, **kw)
    b = lambda: ops.bwd(t["q"], t["k"], t["v"], t["sinks"], o, l, t["dout"], t["cu"], window, w.scale, dq=dq,  # noqa
                        dk=dk, dv=dv, dsinks=ds, workspace=ws, **kw)
    return f, b


def layer_buffers(torch, ops, w, t):
    q, k = t["q"], t["k"]
    ws = torch.empty((ops.bwd_workspace_size(w.T, w.Hq, w.Hkv, w.D, w.batch, w.max_seqlen),), dtype=torch.uint8,
                     device="cuda")
    return (torch.empty_like(q), torch.empty((w.Hq, w.T), dtype=torch.float32, device="cuda"), torch.empty_like(q),
            torch.empty_like(k), torch.empty_like(k), torch.empty((w.Hq,), dtype=torch.float32, device="cuda"), ws)


def measure_extra(torch, ops, stream, iters=5):
    """Forward and backward of the long-context (one 61,440-token document,
    sinks ~N(0, 2^2)) and packed-document (65,536 tokens in documents of
    ~U[256, 8192] tokens) workloads, window 128 and full causal, timed with
    time_calls (CUDA events on the launching stream, the forward kernels in
    turn; every input exceeds the L2, so no flush).  Full causal: TFLOP/s on
    the counted pairs and % of the measured bf16 peak; window 128: GB/s of
    the layer's minimum bytes against the HBM peak."""
    peak, hbm, kind = read_peaks()
    nb = lambda *ts: sum(x.numel() * x.element_size() for x in ts if x is not None)  # noqa: E731
    res = {}
    for base in EXTRA_WORKLOADS:
        w = synth.workload(f"{base}:full")
        t = device_inputs(torch, w)
        bufs = layer_buffers(torch, ops, w, t)
        o, l, dq, dk, dv, ds, _ = bufs
        entry = {"workload": f"{base}: T={w.T} in {w.batch} document(s) (max {w.max_seqlen}), Hq=64 Hkv=8 D=64, "
                             f"sinks ~N(0, {w.sink_std:g}^2); inputs drawn on the GPU",
                 "layers": []}
        for window in (128, 0):
            f, b = layer_calls(ops, w, t, stream, window, bufs)
            p = pairs(w.cu_seqlens, window, w.Hq)
            lay = {"window": window}
            fwd_mb = nb(t["q"], t["k"], t["v"], t["sinks"], o, l)
            bwd_mb = nb(t["q"], t["k"], t["v"], t["sinks"], o, l, t["dout"], dq, dk, dv, ds)
            # full-causal 60k calls take ~40 ms (forward) and ~100 ms (backward)
            n = 1 if (window == 0 and w.T > 60000) else iters
            fns = {"fwd": f}
            fns.update({"fwd:" + kn: (lambda kn=kn: f(kn)) for kn in FWD_KERNEL_NAMES})
            ms = time_calls(torch, stream, fns, n, rounds=4, warm=1)
            f()  # the backward reads the saved out / lse of sink_attn_fwd
            ms.update(time_calls(torch, stream, {"bwd": b}, n, rounds=2, warm=1))
            for name, tm in ms.items():
                pas = name.split(":")[0]  # "fwd" or "bwd"
                flops = (4 if pas == "fwd" else 10) * D * p
                mb = fwd_mb if pas == "fwd" else bwd_mb
                r = {"ms": tm, "tflops": flops / tm / 1e9, "pct_of_peak": 100.0 * flops / tm / 1e9 / peak,
                     "min_bytes": mb, "GBps": mb / tm / 1e6, "hbm_frac": mb / tm / 1e6 / hbm}
                if ":" in name:
                    lay.setdefault("fwd_kernels", {})[name.split(":")[1]] = r
                else:
                    lay[name] = r
            lay["fwd"]["kernel"] = ops.fwd_kernel_for(w.T, w.Hq, w.Hkv, w.D, w.batch, w.max_seqlen, window)
            entry["layers"].append(lay)
        entry["peak_TFLOPs"], entry["peak_GBps"], entry["peak_source"] = peak, hbm, f"{kind} bf16_tflops / hbm_gbs"
        res[base] = entry
        del t, bufs
        torch.cuda.empty_cache()
    if ops.device_error() != 0:
        raise RuntimeError("a kernel reported a timed-out wait")
    return res


def run_profile_case(args):
    """--profile-case KIND:WORKLOAD:LAYER (e.g. fwd:long60k:full, fwd.pair:long60k:full,
    fwd.two_tiles:prefill4k:w128, bwd:prefill4k:w128; fwd.<kernel> runs one of
    the forward kernels explicitly): two calls of one entry point on one workload, for an
    ncu capture of its kernels (capture the second: -s <launches of one
    call>).  Prints nothing but a done line."""
    import torch
    from sink_sliding_window_b200 import build, ops
    kind, name = args.profile_case.split(":", 1)
    kind, _, fwd_kernel = kind.partition(".")
    fwd_kernel = fwd_kernel or "auto"
    torch.cuda.set_device(0)
    build.build()
    ops.load()
    w = synth.workload(name)
    t = device_inputs(torch, w, with_dout=kind == "bwd")
    stream = torch.cuda.current_stream()
    bufs = layer_buffers(torch, ops, w, t)
    f, b = layer_calls(ops, w, t, stream, w.window, bufs)
    if kind == "bwd":
        f()
    for _ in range(2):
        if kind == "fwd":
            f(fwd_kernel)
        else:
            b()
    torch.cuda.synchronize()
    if ops.device_error() != 0:
        raise RuntimeError("a kernel reported a timed-out wait")
    print(f"profile case {args.profile_case} done", flush=True)


# ----------------------------------------------------------- aggregation
def max_over_ranks(x, dist, device):
    """Largest value of x over all ranks (the slowest rank's time); x itself
    when running alone."""
    if dist is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, flops_per_step, steps, ms):
    """Whole-job TFLOP/s: every rank runs its own replica of the step, so the
    job does world x steps steps in the slowest rank's time."""
    return world * flops_per_step * steps / (ms / 1e3) / 1e12


# ------------------------------------------------------------------- arms
def run_reference(args, rank):
    if rank != 0:
        return
    # Size each step so that all warmup + timed steps take about two minutes:
    # the sample's work grows ~linearly with the window-layer prefix and
    # quadratically with the full-causal prefix.
    budget = args.budget_s / (args.warmup + args.steps)
    secs1, _, _, _ = oracle_sample(256, 256)  # calibration, untimed
    lw, lf = 256, 256
    while lw < S and secs1 * (2 * lw / 256 + (lf / 256) ** 2) / 3 * 2 < budget:
        lw, lf = 2 * lw, min(1024, 2 * lf)
    steps = []
    for i in range(args.warmup + args.steps):
        secs, flops, desc, threads = oracle_sample(lw, lf)
        if i >= args.warmup:
            steps.append((secs, flops))
    secs = sum(s for s, _ in steps)
    flops = sum(f for _, f in steps)
    value = flops / secs / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / len(steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_dict():
    return {"workload": f"{WORKLOAD}: B=4 S=4096 Hq=64 Hkv=8 D=64 scale=1/8, one window-128 layer + one "
                        f"full-causal layer, forward+backward",
            "batch": B, "seq_len": S, "num_q_heads": HQ, "num_kv_heads": HKV, "head_dim": D,
            "windows": list(LAYERS), "parallelism": "replicas (one independent workload per GPU)",
            "l2": "no flush; per-step working set (q,k,v,dout,out,lse,dq accumulator ~ 1 GB) exceeds the 126 MB L2"}


def run_ours(args, rank, world, torch, dist):
    from sink_sliding_window_b200 import build, ops

    dev = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(dev)
    build.build()
    ops.load()
    w = synth.workload(f"{WORKLOAD}:w128", seed=rank)
    a = w.generate(with_dout=True)

    def to_dev(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()

    q, k, v, dout = to_dev(a["q"]), to_dev(a["k"]), to_dev(a["v"]), to_dev(a["dout"])
    sinks = torch.from_numpy(a["sinks"]).cuda()
    T = B * S
    def out_buffers():
        outs = {W: (torch.empty_like(q), torch.empty((HQ, T), dtype=torch.float32, device="cuda")) for W in LAYERS}
        grads = {W: (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
                     torch.empty((HQ,), dtype=torch.float32, device="cuda")) for W in LAYERS}
        return outs, grads

    outs, grads = out_buffers()
    ws = torch.empty((ops.bwd_workspace_size(T, HQ, HKV, D, B, S),), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step(q, k, v, sinks, dout, prof=None, bufs=None, st=None):
        o_set, g_set = bufs if bufs is not None else (outs, grads)
        kw = dict(batch=B, max_seqlen=S, stream=st if st is not None else stream)
        for W in LAYERS:
            o, l = o_set[W]
            ops.fwd(q, k, v, sinks, None, W, 0.125, out=o, lse=l, **kw)
        for W in LAYERS:
            o, l = o_set[W]
            dq, dk, dv, ds = g_set[W]
            if prof is not None and W == 0:
                ops.profile_events(ops.PROFILE_BWD_MAIN, *prof)
            ops.bwd(q, k, v, sinks, o, l, dout, None, W, 0.125, dq=dq, dk=dk, dv=dv, dsinks=ds, workspace=ws, **kw)
            if prof is not None and W == 0:
                ops.profile_events(ops.PROFILE_BWD_MAIN)

    def barrier():
        if dist is not None:
            dist.barrier()

    # ---- device-resident timing
    for _ in range(args.warmup):
        step(q, k, v, sinks, dout)
    torch.cuda.synchronize()
    assert ops.device_error() == 0
    prof = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for b_, e_ in prof:  # torch creates the CUDA event on its first record
        b_.record(stream)
        e_.record(stream)
    clocks = ClockSampler(gpu_id_for(torch, dev))
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        step(q, k, v, sinks, dout, prof=prof[i])
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    kern_ms = float(np.mean([b.elapsed_time(e) for b, e in prof]))
    if ops.device_error() != 0:
        raise RuntimeError("a kernel reported a timed-out wait")
    ms = max_over_ranks(ms, dist, "cuda")

    flops = step_flops()
    value = job_throughput(world, flops, args.steps, ms)
    launches = args.steps * len(LAYERS) * (ops.fwd_launches(T, HQ, HKV, D, B, S) + ops.bwd_launches(T, HQ, HKV, D, B, S))

    # ---- end to end through host buffers (pinned), copies inside the region.
    # Every step copies its inputs in from pinned host memory and all of its
    # results (outputs, lse, dq, dk, dv, dsinks of both layers) back out.  The
    # loop is pipelined the way a caller streaming batches would write it:
    # host-to-device copies, the step and device-to-host copies run on three
    # streams over two sets of device buffers, so step i+1's inputs and step
    # i-1's results cross PCIe (both directions at once) while step i runs.
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    names = ("q", "k", "v", "sinks", "dout")
    h_in = {n: t.cpu().pin_memory() for n, t in zip(names, (q, k, v, sinks, dout))}
    d_in = [dict(zip(names, (q, k, v, sinks, dout)))]
    d_in.append({n: torch.empty_like(t) for n, t in d_in[0].items()})  # device copies of the device tensors
    d_sets = [(outs, grads), out_buffers()]
    flat = lambda bs: [t for W in LAYERS for t in (*bs[0][W], *bs[1][W])]  # noqa: E731
    h_out = [t.cpu().pin_memory() for t in flat(d_sets[0])]
    h2d = sum(t.numel() * t.element_size() for t in h_in.values())
    d2h = sum(t.numel() * t.element_size() for t in h_out)
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_ready, in_free = [ev(), ev()], [ev(), ev()]
    done, out_free = [ev(), ev()], [ev(), ev()]
    barrier()
    torch.cuda.synchronize()
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record(stream)
    s_in.wait_event(x0)
    s_out.wait_event(x0)
    for i in range(e2e_steps):
        j = i & 1
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(in_free[j])  # step i-2 has finished reading these inputs
            for n in names:
                d_in[j][n].copy_(h_in[n], non_blocking=True)
            in_ready[j].record(s_in)
        stream.wait_event(in_ready[j])
        if i >= 2:
            stream.wait_event(out_free[j])  # step i-2's results have been copied out
        dj = d_in[j]
        step(dj["q"], dj["k"], dj["v"], dj["sinks"], dj["dout"], bufs=d_sets[j], st=stream)
        in_free[j].record(stream)
        done[j].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done[j])
            for h, d in zip(h_out, flat(d_sets[j])):
                h.copy_(d, non_blocking=True)
            out_free[j].record(s_out)
    stream.wait_event(out_free[(e2e_steps - 1) & 1])
    stream.wait_event(in_ready[(e2e_steps - 1) & 1])
    x1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(x0.elapsed_time(x1), dist, "cuda")
    e2e_value = job_throughput(world, flops, e2e_steps, e2e_ms)

    layers = measure_layers(torch, ops, stream, q, k, v, sinks, dout, outs, grads, ws)
    decode = measure_decode(torch, ops, stream) if not args.skip_decode else None
    extra = measure_extra(torch, ops, stream) if not args.skip_extra else None

    if rank != 0:
        return
    peak, _, peak_kind = read_peaks()
    fwd_full, bwd_full = layer_flops(0)
    achieved = bwd_full / (kern_ms / 1e3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16 q/k/v/dout, N(0,1) sinks)",
        "config": config_dict(),
        "pct_of_peak": 100.0 * value / world / peak,
        "roofline": {"bound": "tensor", "kernel": "sink_attn_bwd_main (full-causal layer)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": f"{peak_kind} bf16_tflops (burst)", "traffic": measured_traffic(),
                     "flops_per_launch": bwd_full, "avg_launch_ms": kern_ms},
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps},
        "gpu_launches": launches,
        "clocks": clk,
    }
    line["layers"] = layers
    if decode is not None:
        line["decode"] = decode
    if extra is not None:
        line.update(extra)
    if world == 1 and not args.skip_cpu_baseline:
        secs, cflops, desc, threads = oracle_sample(S, 2048)
        line["cpu_baseline"] = {"value": cflops / secs / 1e12, "unit": "TFLOP/s", "cores": threads,
                                "kind": "oracle", "sample": desc, "seconds": secs}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--skip-decode", action="store_true", help="do not time sink_attn_decode after the step")
    ap.add_argument("--skip-extra", action="store_true",
                    help="do not time the long-context and packed-document layers after the step")
    ap.add_argument("--profile-case", default=None,
                    help="KIND:WORKLOAD:LAYER, e.g. fwd:long60k:full: only run two calls of one entry point (for ncu)")
    ap.add_argument("--budget-s", type=float, default=120.0,
                    help="--impl reference: seconds all warmup + timed oracle steps should take")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return 0
    if args.profile_case:
        run_profile_case(args)
        return 0
    import torch

    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist_
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist_.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = dist_
    try:
        run_ours(args, rank, world, torch, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
