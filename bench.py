"""Benchmark of the attention-sink kernels on B200.

Headline workload (one "step"): prefill of one MiMo SWA layer, batch 1,
n = 32768, 64 Q / 8 KV heads, window 128, partial RoPE on 64 dims (theta 1e4),
per-head sink; inputs synthetic N(0,1) bf16, resident in HBM and larger than L2.
``value`` is algorithmic TFLOP/s (2 * (192 + 128) * scored pairs * Hq / time).
The same JSON line also carries, under ``workloads``, the GA-layer prefill
(n = 32768 causal, 64/4), one hybrid decode step over the 48-layer pattern
(B = 64) and the token-level sparse decode (B = 8, L = 262144, 128 + 1024), each
with its roofline.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
Under torchrun each rank runs its own copy of the workload (weak scaling); the
job time is the max over ranks.
"""

from __future__ import annotations

import argparse
import ctypes
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from hybrid_sliding_window_sink_b200 import dist as D  # noqa: E402
from hybrid_sliding_window_sink_b200 import workloads as wl  # noqa: E402

METRIC = "prefill attn TFLOP/s & decode HBM GB/s, % of B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- peaks / clocks
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled through NVML every millisecond by a
    thread while the timed loop runs (the headline's timed region is only milliseconds long,
    too short for nvidia-smi's sampling interval). Read-only queries."""

    # NVML clock-event reason bits
    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40}

    def __init__(self, device_index: int, period_s: float = 0.001):
        import threading
        self.samples, self.reasons, self.smax, self.err = [], set(), None, None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.smax = float(pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM))
        except Exception as e:  # no NVML: report it in the line
            self.err = repr(e)[:80]
            return
        self._thread = threading.Thread(target=self._run, args=(period_s,), daemon=True)
        self._thread.start()

    def _run(self, period_s):
        nv, h = self._nv, self._h
        while not self._stop.is_set():
            try:
                self.samples.append(float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                for name, bit in self.REASONS.items():
                    if bits & bit:
                        self.reasons.add(name)
            except Exception as e:
                self.err = repr(e)[:80]
                return
            time.sleep(period_s)

    def stop(self):
        if self.err is not None and not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [f"NVML unavailable: {self.err}"]}
        self._stop.set()
        self._thread.join(timeout=2)
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.smax,
                "samples": len(self.samples), "reasons": sorted(self.reasons)}


# ----------------------------------------------------------------------------- measured traffic
def traffic_for(key, units):
    """DRAM bytes of one launch from the ncu-measured bytes per unit (profiles/traffic.json),
    or None when the kernel sources changed since the counters were taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)[key]
        h = hashlib.sha256()
        for name in rec["sources"]:
            with open(os.path.join(ROOT, "hybrid_sliding_window_sink_b200", "csrc", name), "rb") as f:
                h.update(f.read())
        if h.hexdigest()[:16] != rec["sha"]:
            return None
        return round(rec["bytes_per_unit"] * units)
    except (OSError, KeyError, ValueError):
        return None


# ----------------------------------------------------------------------------- algorithmic work
def swa_pairs(n, window):
    if window <= 0 or window >= n:
        return n * (n + 1) // 2
    return n * window - window * (window - 1) // 2


def prefill_work(case: wl.PrefillCase):
    pairs = swa_pairs(case.seqlen, case.window) * case.batch
    flops = 2.0 * (wl.DQK + wl.DV) * pairs * case.hq
    n, B = case.seqlen, case.batch
    bytes_ = (B * n * case.hq * wl.DQK * 2 + B * n * case.hkv * (wl.DQK + wl.DV) * 2
              + B * n * case.hq * wl.DV * 2 + B * case.hq * n * 4 + case.hq * 4)
    return flops, float(bytes_)


def decode_layer_bytes(lengths, hq, hkv, kind, cap):
    L = np.asarray(lengths, dtype=np.int64)
    keys = np.minimum(L, cap) if kind == "ring" else L
    kv = int(keys.sum()) * hkv * (wl.DQK + wl.DV) * 2
    B = len(L)
    return float(kv + B * hq * wl.DQK * 2 + B * hq * wl.DV * 2 + B * hq * 4 + hq * 4 + B * 4)


# ----------------------------------------------------------------------------- timing
class DeviceError(RuntimeError):
    pass


def timed(fn, steps, warmup, stream, flush=None, clocks=None):
    """Run ``warmup`` untimed steps, then time exactly ``steps`` with CUDA events on
    ``stream``, bracketed by barrier + synchronize. Returns elapsed ms of this rank.
    Raises DeviceError (before timing) if a warm-up step set the library's device error
    word, so that a broken kernel is not timed. ``clocks``: a list that receives a
    ClockSampler's record of the timed region."""
    from hybrid_sliding_window_sink_b200 import _lib
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    err = _lib.last_device_error()
    if err:
        raise DeviceError(f"device error word {err} set during warm-up")
    D.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device()) if clocks is not None else None
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        if flush is not None:
            flush()
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    if sampler is not None:
        clocks.append(sampler.stop())
    D.barrier()
    return e0.elapsed_time(e1)


def timed_stream(fn, steps, warmup, stream):
    """``timed`` with the events recorded on ``stream`` (the stream the work runs on)."""
    with torch.cuda.stream(stream):
        return timed(fn, steps, warmup, stream)


def timed_graph(fn, steps, warmup, dev):
    """Captures ``fn(stream)`` (launches on ``stream`` only) in a CUDA graph on a side stream and
    times ``steps`` replays after ``warmup`` with CUDA events on that stream (``timed``). Short
    kernels launched one by one from Python would otherwise be timed at the host's launch rate;
    a serving loop replays its decode step as a graph, too."""
    s = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        fn(s)                        # outside capture first: library loaded, attributes set
        s.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            fn(s)
    torch.cuda.synchronize()
    ms = timed_stream(graph.replay, steps, warmup, s)
    del graph
    return ms


def roofline_hbm(bytes_per_launch, ms_per_launch, peaks, tag, traffic=None):
    ach = bytes_per_launch / (ms_per_launch * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(ach / peaks["hbm_gbs"], 4), "traffic": traffic, "peak_source": tag}


def roofline_tensor(flops_per_launch, ms_per_launch, peak, tag, traffic=None):
    ach = flops_per_launch / (ms_per_launch * 1e-3) / 1e12
    return {"bound": "tensor", "achieved": round(ach, 2), "peak": peak, "unit": "TFLOP/s",
            "frac": round(ach / peak, 4), "traffic": traffic, "peak_source": tag}


# ----------------------------------------------------------------------------- CPU oracle baseline
def run_oracle_harness(*extra, timeout=900):
    """Runs the float64 oracle's timing harness (``python -m oracle.baseline``) as a separate
    process that never touches a GPU, on all host cores; returns its JSON object."""
    cmd = [sys.executable, "-m", "oracle.baseline", *[str(x) for x in extra]]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=timeout)
    if res.returncode != 0:
        raise RuntimeError(f"oracle harness failed: {res.stderr[-500:]}")
    return json.loads(res.stdout.strip().splitlines()[-1])


def cpu_baseline_line(budget=3.0):
    """The oracle on every configuration (full where it finishes in seconds, a row sample
    extrapolated by work otherwise); ``value`` is the headline SWA-prefill throughput."""
    h = run_oracle_harness("--budget", budget)
    w = h["workloads"]
    per = {k: [v["s"], v["how"][:5]] for k, v in w.items()}
    return {"value": w["swa_prefill"]["rate"], "unit": "TFLOP/s", "cores": h["cores"], "kind": "oracle",
            "sample": (f"float64 oracle, {h['cores']} processes x 1 BLAS thread: SWA n=32768 random rows x heads "
                       f"({budget:g} s per process), extrapolated by pairs; per_config = est. seconds per call "
                       "(full|extra[polated])"),
            "per_config": per}


# ----------------------------------------------------------------------------- workloads
def bench_prefill(case, steps, warmup, peaks, tag, dev, stream, clocks=None):
    from hybrid_sliding_window_sink_b200 import _lib
    inp = wl.case_prefill_inputs(case, device=dev)
    out = torch.empty(case.batch, case.seqlen, case.hq, wl.DV, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(case.batch, case.hq, case.seqlen, dtype=torch.float32, device=dev)

    def step():
        _lib.prefill(inp["q"], inp["k"], inp["v"], inp["sink"], window=case.window,
                     rope_theta=case.theta, rot_dims=wl.ROT_DIMS, out=out, lse=lse, stream=stream)

    ms = timed(step, steps, warmup, stream, clocks=clocks)
    flops, bytes_ = prefill_work(case)
    err = _lib.last_device_error()
    res = {"inp": inp, "ms_total": ms, "flops": flops, "bytes": bytes_, "device_error": err}
    return res


def bench_tiny_prefill(steps, peaks, tag, dev, stream):
    """Tiny SWA+sink prefill (n=1024, 8 Q / 1 KV, W=128): 5.9 MB of inputs and outputs, below
    L2, so every launch follows a 256 MB write that flushes L2; the time is that of a CUDA
    graph of (flush, prefill) minus that of a graph of the flush alone."""
    from hybrid_sliding_window_sink_b200 import _lib
    case = wl.TINY_SWA_PREFILL
    inp = wl.case_prefill_inputs(case, device=dev)
    out = torch.empty(case.batch, case.seqlen, case.hq, wl.DV, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(case.batch, case.hq, case.seqlen, dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step(st):
        _lib.prefill(inp["q"], inp["k"], inp["v"], inp["sink"], window=case.window,
                     rope_theta=case.theta, rot_dims=wl.ROT_DIMS, out=out, lse=lse, stream=st)

    # graph(flush, prefill) minus graph(flush): the kernel's time after an L2 flush, without the
    # host's launch latency
    ms_both = timed_graph(lambda st: (flush.fill_(1), step(st)), steps, 3, dev) / steps
    ms_flush = timed_graph(lambda st: flush.fill_(1), steps, 3, dev) / steps
    ms = ms_both - ms_flush
    flops, bytes_ = prefill_work(case)
    del inp, out, lse, flush
    return {"ms": round(ms, 5), "tflops": round(flops / (ms * 1e-3) / 1e12, 2),
            "frac": round(bytes_ / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
            "device_error": _lib.last_device_error()}


def bench_chunk_prefill(steps, warmup, peaks, tag, dev, stream, chunk=16384, prefix=16384):
    """Chunked prefill (16K chunk after a 16K prefix held rotated, as a cache holds it), B=1,
    on an SWA layer (64Q/8KV, W=128, HBM-bound) and a GA layer (64Q/4KV, tensor-bound)."""
    from hybrid_sliding_window_sink_b200 import _lib
    res = {}
    nk = prefix + chunk
    for name, hq, hkv, window, theta in (("swa", 64, 8, wl.SWA_WINDOW, wl.SWA_THETA),
                                         ("ga", 64, 4, 0, wl.GA_THETA)):
        inp = wl.prefill_inputs(1, nk, hq, hkv, seed=1700, device=dev, k_scale=0.5 if window == 0 else 1.0)
        q = inp["q"][:, prefix:].contiguous()
        out = torch.empty(1, chunk, hq, wl.DV, dtype=torch.bfloat16, device=dev)
        lse = torch.empty(1, hq, chunk, dtype=torch.float32, device=dev)

        def step():
            _lib.prefill_chunk(q, inp["k"], inp["v"], inp["sink"], pos_offset=prefix, k_prefix_rotated=True,
                               window=window, rope_theta=theta, rot_dims=wl.ROT_DIMS, out=out, lse=lse,
                               stream=stream)

        n_steps = steps if window > 0 else max(3, steps // 20)
        ms = timed(step, n_steps, warmup, stream) / n_steps
        if window > 0:
            pairs = sum(min(window, prefix + i + 1) for i in range(chunk))
            bytes_ = (chunk * hq * wl.DQK * 2 + (chunk + window - 1) * hkv * (wl.DQK + wl.DV) * 2
                      + chunk * hq * wl.DV * 2 + hq * chunk * 4)
        else:
            pairs = chunk * prefix + chunk * (chunk + 1) // 2
            bytes_ = chunk * hq * wl.DQK * 2 + nk * hkv * (wl.DQK + wl.DV) * 2 + chunk * hq * (wl.DV * 2 + 4)
        flops = 2.0 * (wl.DQK + wl.DV) * pairs * hq
        res[name] = {"ms": round(ms, 4), "tflops": round(flops / (ms * 1e-3) / 1e12, 2),
                     "roofline": (roofline_hbm(bytes_, ms, peaks, tag) if window > 0 else
                                  roofline_tensor(flops, ms, peaks["bf16_tflops"], tag)),
                     "device_error": _lib.last_device_error()}
        del inp, q, out, lse
        torch.cuda.empty_cache()
    res["workload"] = f"chunked prefill, {chunk}-token chunk after a {prefix}-token prefix (rotated), B=1"
    res["kernel"] = {"swa": "prefill_swa_kernel (K/V ring)", "ga": "prefill_ga_kernel (row-block pairs)"}
    return res


def e2e_prefill(case, steps, dev, stream):
    """Same metric through the public call with host buffers: every step copies its inputs from
    pinned host memory to the device, runs the call and copies out and lse back, all inside the
    timed region. Steps are pipelined the way a serving loop would run them: the host-to-device
    copies of step i + 1 and the device-to-host copies of step i - 1 overlap the call of step i
    (three streams, two device buffer sets; PCIe carries both directions at once)."""
    from hybrid_sliding_window_sink_b200 import _lib
    host = wl.case_prefill_inputs(case, device="cpu")
    host = {k: v.pin_memory() for k, v in host.items()}
    sets = []
    for _ in range(2):
        sets.append({
            "q": torch.empty_like(host["q"], device=dev), "k": torch.empty_like(host["k"], device=dev),
            "v": torch.empty_like(host["v"], device=dev), "sink": torch.empty_like(host["sink"], device=dev),
            "out": torch.empty(case.batch, case.seqlen, case.hq, wl.DV, dtype=torch.bfloat16, device=dev),
            "lse": torch.empty(case.batch, case.hq, case.seqlen, dtype=torch.float32, device=dev)})
    h_out = torch.empty(sets[0]["out"].shape, dtype=torch.bfloat16).pin_memory()
    h_lse = torch.empty(sets[0]["lse"].shape, dtype=torch.float32).pin_memory()
    s_in, s_cmp, s_out = torch.cuda.Stream(device=dev), stream, torch.cuda.Stream(device=dev)
    ev = {name: [torch.cuda.Event() for _ in range(2)] for name in ("in", "cmp", "out")}
    started = [False, False]

    def step(i):
        b, d = i % 2, sets[i % 2]
        with torch.cuda.stream(s_in):
            if started[b]:
                s_in.wait_event(ev["cmp"][b])          # step i - 2 has read this input set
            for name in ("q", "k", "v", "sink"):
                d[name].copy_(host[name], non_blocking=True)
            ev["in"][b].record(s_in)
        s_cmp.wait_event(ev["in"][b])
        if started[b]:
            s_cmp.wait_event(ev["out"][b])             # step i - 2's outputs have left this set
        _lib.prefill(d["q"], d["k"], d["v"], d["sink"], window=case.window, rope_theta=case.theta,
                     rot_dims=wl.ROT_DIMS, out=d["out"], lse=d["lse"], stream=s_cmp)
        ev["cmp"][b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["cmp"][b])
            h_out.copy_(d["out"], non_blocking=True)
            h_lse.copy_(d["lse"], non_blocking=True)
            ev["out"][b].record(s_out)
        started[b] = True

    for i in range(3):                                 # warm-up: both buffer sets, then one more
        step(i)
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    for i in range(steps):
        step(i)
    t1.record(s_out)                                   # after the last step's copies out
    torch.cuda.synchronize(dev)
    ms = t0.elapsed_time(t1)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = h_out.numel() * h_out.element_size() + h_lse.numel() * h_lse.element_size()
    return ms / steps, h2d, d2h


def bench_decode_step(steps, warmup, peaks, tag, dev, stream, batch_range=None):
    """One decode step over the 48-layer hybrid pattern (B=64): 39 SWA ring layers with
    distinct caches and 9 GA layers reading one padded linear cache (131072 slots). With
    ``batch_range`` = (lo, hi) only sequences [lo, hi) of the batch (their lengths, caches,
    queries and outputs): this rank's share when the step is partitioned across ranks."""
    from hybrid_sliding_window_sink_b200 import _lib
    cs, cg = wl.HYBRID_DECODE_SWA, wl.HYBRID_DECODE_GA
    L = wl.lengths_uniform(cs.batch, cs.min_len, cs.max_len, seed=cs.seed)
    lo, hi = batch_range if batch_range is not None else (0, cs.batch)
    L = L[lo:hi]
    B = hi - lo
    Ld = L.to(dev)
    g = torch.Generator(device=dev)
    g.manual_seed(cs.seed + 1000 * lo)
    pattern = wl.layer_pattern()
    layers = []
    ga_k = torch.randn(B, cg.capacity, cg.hkv, wl.DQK, generator=g, device=dev,
                       dtype=torch.float32).to(torch.bfloat16)
    ga_v = torch.randn(B, cg.capacity, cg.hkv, wl.DV, generator=g, device=dev,
                       dtype=torch.float32).to(torch.bfloat16)
    for li, kind in enumerate(pattern):
        hkv = cs.hkv if kind == 1 else cg.hkv
        q = torch.randn(B, cs.hq, wl.DQK, generator=g, device=dev).to(torch.bfloat16)
        sink = torch.randn(cs.hq, generator=g, device=dev)
        if kind == 1:
            kc = torch.randn(B, cs.capacity, hkv, wl.DQK, generator=g, device=dev).to(torch.bfloat16)
            vc = torch.randn(B, cs.capacity, hkv, wl.DV, generator=g, device=dev).to(torch.bfloat16)
        else:
            kc, vc = ga_k, ga_v
        out = torch.empty(B, cs.hq, wl.DV, dtype=torch.bfloat16, device=dev)
        lse = torch.empty(B, cs.hq, dtype=torch.float32, device=dev)
        layers.append((kind, q, kc, vc, sink, out, lse))
    nws = _lib.workspace_size(B, cg.hq, cg.hkv, op=_lib.MIMO_OP_DECODE,
                              kind=_lib.MIMO_CACHE_LINEAR, capacity=cg.capacity)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev)

    def run_layer(lay, st):
        kind, q, kc, vc, sink, out, lse = lay
        _lib.decode(q, kc, vc, Ld, sink, kind="ring" if kind == 1 else "linear",
                    out=out, lse=lse, workspace=ws, stream=st)

    ms = timed_graph(lambda st: [run_layer(l, st) for l in layers], steps, warmup, dev)
    Ls = L.tolist()
    b_swa = decode_layer_bytes(Ls, cs.hq, cs.hkv, "ring", cs.capacity)
    b_ga = decode_layer_bytes(Ls, cg.hq, cg.hkv, "linear", cg.capacity)
    total = 39 * b_swa + 9 * b_ga
    # per-kind kernel time: time GA layers and SWA layers separately
    ga_layers = [l for l in layers if l[0] == 0]
    swa_layers = [l for l in layers if l[0] == 1]
    ms_ga = timed_graph(lambda st: [run_layer(l, st) for l in ga_layers], steps, 1, dev) / (steps * 9)
    ms_swa = timed_graph(lambda st: [run_layer(l, st) for l in swa_layers], steps, 1, dev) / (steps * 39)
    res = {
        "value": round(total / (ms / steps * 1e-3) / 1e9, 1), "unit": "GB/s",
        "ms_per_step": round(ms / steps, 4), "bytes_per_step": total,
        "launches_per_step": 39 + 9 * 2, "graph": True,
        "ga_layer": roofline_hbm(b_ga, ms_ga, peaks, tag,
                                 traffic_for("decode_split_linear", int(sum(Ls)) * cg.hkv)),
        "swa_layer": roofline_hbm(b_swa, ms_swa, peaks, tag,      # every ring is full (L >= 4096)
                                  traffic_for("decode_warp_ring", len(Ls) * cs.hkv)),
        "roofline": roofline_hbm(total, ms / steps, peaks, tag),
        "ms_ga_layer": round(ms_ga, 4), "ms_swa_layer": round(ms_swa, 5),
        "cache": "39 distinct SWA ring caches; one padded GA cache [64,131072,4,*] read by all 9 GA layers",
        "l2": "GA layers read 11 GB each (>> L2); SWA ring caches 44.6 MB each, distinct per layer",
    }
    del layers, ga_k, ga_v, ws
    return res


def mtp_layer_bytes(lengths, hq, hkv, kind, cap, q_len):
    """Algorithmic bytes of one multi-query decode layer: each (sequence, KV head) reads its
    key range once (ring: min(L, cap) <= W + q_len - 1 tokens; linear: L tokens), plus q,
    out and lse of the q_len rows per query head."""
    L = np.asarray(lengths, dtype=np.int64)
    keys = np.minimum(L, cap) if kind == "ring" else L
    kv = int(keys.sum()) * hkv * (wl.DQK + wl.DV) * 2
    rows = len(L) * q_len * hq
    return float(kv + rows * (wl.DQK * 2 + wl.DV * 2 + 4) + hq * 4 + len(L) * 4)


def bench_mtp_step(steps, warmup, peaks, tag, dev, stream, q_len=4):
    """MTP verification step over the 48-layer hybrid pattern (B=64, 1 + 3 draft tokens per
    sequence): 39 SWA layers on distinct rings of W + q_len - 1 = 131 slots, 9 GA layers on one
    padded linear cache (131072 slots). Lengths as the decode step."""
    from hybrid_sliding_window_sink_b200 import _lib
    cs, cg = wl.HYBRID_DECODE_SWA, wl.HYBRID_DECODE_GA
    cap_ring = wl.SWA_WINDOW + q_len - 1
    L = wl.lengths_uniform(cs.batch, cs.min_len, cs.max_len, seed=cs.seed)
    Ld = L.to(dev)
    g = torch.Generator(device=dev)
    g.manual_seed(cs.seed + 5)
    layers = []
    ga_k = torch.randn(cg.batch, cg.capacity, cg.hkv, wl.DQK, generator=g, device=dev,
                       dtype=torch.float32).to(torch.bfloat16)
    ga_v = torch.randn(cg.batch, cg.capacity, cg.hkv, wl.DV, generator=g, device=dev,
                       dtype=torch.float32).to(torch.bfloat16)
    for kind in wl.layer_pattern():
        hkv = cs.hkv if kind == 1 else cg.hkv
        q = torch.randn(cs.batch, q_len, cs.hq, wl.DQK, generator=g, device=dev).to(torch.bfloat16)
        sink = torch.randn(cs.hq, generator=g, device=dev)
        if kind == 1:
            kc = torch.randn(cs.batch, cap_ring, hkv, wl.DQK, generator=g, device=dev).to(torch.bfloat16)
            vc = torch.randn(cs.batch, cap_ring, hkv, wl.DV, generator=g, device=dev).to(torch.bfloat16)
        else:
            kc, vc = ga_k, ga_v
        out = torch.empty(cs.batch, q_len, cs.hq, wl.DV, dtype=torch.bfloat16, device=dev)
        lse = torch.empty(cs.batch, q_len, cs.hq, dtype=torch.float32, device=dev)
        layers.append((kind, q, kc, vc, sink, out, lse))
    shape_ga = _lib.make_shape(cg.batch, 1, cg.hq, cg.hkv)
    nws = int(_lib.lib().mimo_attn_decode_mq_workspace_size(ctypes.byref(shape_ga), _lib.MIMO_CACHE_LINEAR,
                                                            cg.capacity, q_len, 0))
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev)

    def run_layer(lay, st):
        kind, q, kc, vc, sink, out, lse = lay
        _lib.decode_mq(q, kc, vc, Ld, sink, kind="ring" if kind == 1 else "linear",
                       window=wl.SWA_WINDOW, out=out, lse=lse, workspace=ws, stream=st)

    ms = timed_graph(lambda st: [run_layer(l, st) for l in layers], steps, warmup, dev)
    Ls = L.tolist()
    b_swa = mtp_layer_bytes(Ls, cs.hq, cs.hkv, "ring", cap_ring, q_len)
    b_ga = mtp_layer_bytes(Ls, cg.hq, cg.hkv, "linear", cg.capacity, q_len)
    total = 39 * b_swa + 9 * b_ga
    ga_layers = [l for l in layers if l[0] == 0]
    swa_layers = [l for l in layers if l[0] == 1]
    ms_ga = timed_graph(lambda st: [run_layer(l, st) for l in ga_layers], steps, 1, dev) / (steps * 9)
    ms_swa = timed_graph(lambda st: [run_layer(l, st) for l in swa_layers], steps, 1, dev) / (steps * 39)
    flops_ga = 2.0 * (wl.DQK + wl.DV) * q_len * cg.hq * float(np.sum(Ls))   # upper bound: all keys
    res = {
        "value": round(total / (ms / steps * 1e-3) / 1e9, 1), "unit": "GB/s",
        "ms_per_step": round(ms / steps, 4), "bytes_per_step": total, "q_len": q_len,
        "launches_per_step": 39 + 9 * 2,
        "ga_layer": roofline_hbm(b_ga, ms_ga, peaks, tag,
                                 traffic_for("decode_mq_linear", int(sum(Ls)) * cg.hkv)),
        "swa_layer": roofline_hbm(b_swa, ms_swa, peaks, tag),
        "roofline": roofline_hbm(total, ms / steps, peaks, tag),
        "ms_ga_layer": round(ms_ga, 4), "ms_swa_layer": round(ms_swa, 5),
        "ga_layer_tflops": round(flops_ga / (ms_ga * 1e-3) / 1e12, 1),
        "cache": f"39 distinct SWA rings of {cap_ring} slots; one padded GA cache [64,131072,4,*]",
    }
    del layers, ga_k, ga_v, ws
    return res


def fp8_decode_layer_bytes(lengths, hq, hkv, kind, cap):
    """Algorithmic bytes of one FP8-cache decode layer: E4M3 K/V rows (320 B) plus the two
    fp32 row scales per (token, KV head), and q, out, lse."""
    L = np.asarray(lengths, dtype=np.int64)
    keys = np.minimum(L, cap) if kind == "ring" else L
    kv = int(keys.sum()) * hkv * (wl.DQK + wl.DV + 8)
    B = len(L)
    return float(kv + B * hq * wl.DQK * 2 + B * hq * wl.DV * 2 + B * hq * 4 + hq * 4 + B * 4)


def bench_fp8_decode_step(steps, warmup, peaks, tag, dev, stream):
    """The hybrid decode step of bench_decode_step over FP8 caches (E4M3 K/V with
    per-(token, KV head) fp32 scales): 39 SWA rings of 128 slots, 9 GA layers on one padded
    linear cache of 131072 slots, B=64, same lengths."""
    from hybrid_sliding_window_sink_b200 import _lib
    cs, cg = wl.HYBRID_DECODE_SWA, wl.HYBRID_DECODE_GA
    L = wl.lengths_uniform(cs.batch, cs.min_len, cs.max_len, seed=cs.seed)
    Ld = L.to(dev)
    g = torch.Generator(device=dev)
    g.manual_seed(cs.seed + 9)
    mk_scale = lambda *sh: torch.empty(*sh, device=dev).uniform_(0.002, 0.01, generator=g)  # noqa: E731
    ga = (wl.random_e4m3((cg.batch, cg.capacity, cg.hkv, wl.DQK), g, dev),
          wl.random_e4m3((cg.batch, cg.capacity, cg.hkv, wl.DV), g, dev),
          mk_scale(cg.batch, cg.capacity, cg.hkv), mk_scale(cg.batch, cg.capacity, cg.hkv))
    layers = []
    for kind in wl.layer_pattern():
        q = torch.randn(cs.batch, cs.hq, wl.DQK, generator=g, device=dev).to(torch.bfloat16)
        sink = torch.randn(cs.hq, generator=g, device=dev)
        if kind == 1:
            cache = (wl.random_e4m3((cs.batch, cs.capacity, cs.hkv, wl.DQK), g, dev),
                     wl.random_e4m3((cs.batch, cs.capacity, cs.hkv, wl.DV), g, dev),
                     mk_scale(cs.batch, cs.capacity, cs.hkv), mk_scale(cs.batch, cs.capacity, cs.hkv))
        else:
            cache = ga
        out = torch.empty(cs.batch, cs.hq, wl.DV, dtype=torch.bfloat16, device=dev)
        lse = torch.empty(cs.batch, cs.hq, dtype=torch.float32, device=dev)
        layers.append((kind, q, cache, sink, out, lse))
    nws = _lib.workspace_size(cg.batch, cg.hq, cg.hkv, op=_lib.MIMO_OP_DECODE,
                              kind=_lib.MIMO_CACHE_LINEAR, capacity=cg.capacity)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev)

    def run_layer(lay, st):
        kind, q, (k8, v8, ks, vs), sink, out, lse = lay
        _lib.decode_fp8(q, k8, v8, ks, vs, Ld, sink, kind="ring" if kind == 1 else "linear",
                        out=out, lse=lse, workspace=ws, stream=st)

    ms = timed_graph(lambda st: [run_layer(l, st) for l in layers], steps, warmup, dev)
    Ls = L.tolist()
    b_swa = fp8_decode_layer_bytes(Ls, cs.hq, cs.hkv, "ring", cs.capacity)
    b_ga = fp8_decode_layer_bytes(Ls, cg.hq, cg.hkv, "linear", cg.capacity)
    total = 39 * b_swa + 9 * b_ga
    ms_ga = timed_graph(lambda st: [run_layer(l, st) for l in layers if l[0] == 0], steps, 1, dev) / (steps * 9)
    ms_swa = timed_graph(lambda st: [run_layer(l, st) for l in layers if l[0] == 1], steps, 1, dev) / (steps * 39)
    res = {
        "value": round(total / (ms / steps * 1e-3) / 1e9, 1), "unit": "GB/s",
        "ms_per_step": round(ms / steps, 4), "bytes_per_step": total,
        "launches_per_step": 39 + 9 * 2,
        "ga_layer": roofline_hbm(b_ga, ms_ga, peaks, tag,
                                 traffic_for("decode_fp8_linear", int(sum(Ls)) * cg.hkv)),
        "swa_layer": roofline_hbm(b_swa, ms_swa, peaks, tag),
        "roofline": roofline_hbm(total, ms / steps, peaks, tag),
        "ms_ga_layer": round(ms_ga, 4), "ms_swa_layer": round(ms_swa, 5),
        "cache": "E4M3 K/V + fp32 scale per (token, KV head); 39 distinct 128-slot rings; one padded GA cache",
    }
    del layers, ga, ws
    return res


def bench_select(steps, warmup, peaks, tag, dev, stream):
    """Token selection on the sparse-decode shape: B=8, L=262144, 64Q/4KV, recent 128, 1024
    selected per (sequence, KV head). Algorithmic bytes: every candidate K row once (384 B),
    the score keys written once and read by the select pass (4 x 4 B)."""
    from hybrid_sliding_window_sink_b200 import _lib
    c = wl.SPARSE_DECODE
    lengths = [c.context] * c.batch
    d = wl.decode_inputs(c.batch, c.hq, c.hkv, c.context, lengths, seed=c.seed + 3, device=dev)
    del d["v_cache"]
    out = torch.empty(c.batch, c.hkv, c.n_sel, dtype=torch.int32, device=dev)
    shape = _lib.make_shape(c.batch, 1, c.hq, c.hkv)
    ws = torch.empty(int(_lib.lib().mimo_attn_select_workspace_size(ctypes.byref(shape), c.context)),
                     dtype=torch.uint8, device=dev)

    def step():
        _lib.select_tokens(d["q"], d["k_cache"], d["lengths"], recent=c.recent, n_sel=c.n_sel,
                           out=out, workspace=ws, stream=stream)

    ms = timed(step, steps, warmup, stream) / steps
    cand = (c.context - c.recent) * c.batch * c.hkv
    bytes_ = float(cand * (wl.DQK * 2 + 4 * 4))
    res = {"value": round(bytes_ / (ms * 1e-3) / 1e9, 1), "unit": "GB/s", "ms_per_call": round(ms, 4),
           "bytes_per_call": bytes_, "launches_per_call": 2,
           "roofline": roofline_hbm(bytes_, ms, peaks, tag, traffic_for("token_select", cand)),
           "workload": "token selection B=8 L=262144 64Q/4KV, top 1024 outside the recent 128"}
    del d, ws, out
    return res


def bench_sparse(steps, warmup, peaks, tag, dev, stream, calls=16):
    """Token-level sparse decode: ``calls`` independent calls (distinct q and index sets,
    >= 385 MB of gathered rows in all, more than L2) per step, captured in a CUDA graph."""
    from hybrid_sliding_window_sink_b200 import _lib
    c = wl.SPARSE_DECODE
    lengths = [c.context] * c.batch
    base = wl.decode_inputs(c.batch, c.hq, c.hkv, c.context, lengths, seed=c.seed, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(c.seed + 1)
    sets = []
    nws = _lib.workspace_size(c.batch, c.hq, c.hkv, op=_lib.MIMO_OP_SPARSE, capacity=c.context,
                              recent=c.recent, n_sel=c.n_sel)
    for i in range(calls):
        q = torch.randn(c.batch, c.hq, wl.DQK, generator=g, device=dev).to(torch.bfloat16)
        sel = wl.sorted_unique_indices(c.batch, c.hkv, c.n_sel, [c.context - c.recent] * c.batch,
                                       seed=c.seed + 100 + i).to(dev)
        out = torch.empty(c.batch, c.hq, wl.DV, dtype=torch.bfloat16, device=dev)
        lse = torch.empty(c.batch, c.hq, dtype=torch.float32, device=dev)
        ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev)
        sets.append((q, sel, out, lse, ws))

    def calls_fn():
        for (q, sel, out, lse, ws) in sets:
            _lib.sparse(q, base["k_cache"], base["v_cache"], base["lengths"], sel, base["sink"],
                        recent=c.recent, out=out, lse=lse, workspace=ws, stream=stream)

    # capture on a side stream (graphs cannot be captured on the legacy default stream)
    cap_stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap_stream):
        calls_fn_s = lambda: [  # noqa: E731
            _lib.sparse(q, base["k_cache"], base["v_cache"], base["lengths"], sel, base["sink"],
                        recent=c.recent, out=out, lse=lse, workspace=ws, stream=cap_stream)
            for (q, sel, out, lse, ws) in sets]
        calls_fn_s()   # loads the library and warms caches outside capture
        cap_stream.synchronize()
        with torch.cuda.graph(graph, stream=cap_stream):
            calls_fn_s()
    torch.cuda.synchronize()

    def replay():
        graph.replay()

    ms = timed_stream(replay, steps, warmup, cap_stream)
    per_call_bytes = (c.batch * c.hkv * (c.recent + c.n_sel) * (wl.DQK + wl.DV) * 2
                      + c.batch * c.hkv * c.n_sel * 4 + c.batch * c.hq * (wl.DQK + wl.DV) * 2
                      + c.batch * c.hq * 4 + c.hq * 4 + c.batch * 4)
    ms_call = ms / (steps * calls)
    res = {"value": round(per_call_bytes / (ms_call * 1e-3) / 1e9, 1), "unit": "GB/s",
           "ms_per_call": round(ms_call, 5), "bytes_per_call": per_call_bytes, "calls_per_step": calls,
           "launches_per_call": 2,
           "roofline": roofline_hbm(per_call_bytes, ms_call, peaks, tag,
                                    traffic_for("decode_warp_sparse", c.batch * c.hkv)),
           "graph": True}
    del graph, sets, base
    return res


# ----------------------------------------------------------------------------- main
#: Wall-clock seconds the reference arm spends in all (warm-up + timed steps), and the number
#: of host processes it uses (0 = every core this process may run on).
REF_SECONDS = 120.0
REF_CORES = 0


def reference_arm(args, warmup, case):
    """``--impl reference``: the float64 oracle on the host cores, on the headline workload's
    row sample, each step a bounded sample; rank 0 only."""
    world, rank, _ = D.env_world()
    if rank != 0:
        return
    budget = max(0.02, REF_SECONDS / (args.steps + warmup))
    h = run_oracle_harness("--only", "swa_prefill", "--steps", args.steps, "--warmup", warmup,
                           "--budget", budget, "--cores", REF_CORES)
    work = sum(w for w, _ in h["steps"])
    wall = sum(t for _, t in h["steps"])
    value = work / wall / 1e12
    desc = (f"float64 oracle, {h['cores']} processes x 1 BLAS thread, random rows x heads of the "
            f"n=32768 SWA layer, {budget:.2f} s per process per step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": warmup,
            "ms_per_step": 1e3 * wall / len(h["steps"]), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": case.name, "global_batch": case.batch, "seq_len": case.seqlen,
                       "parallelism": "none (host CPU)"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": h["cores"],
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def decode_shard_arm(args, warmup, peaks, tag):
    """``--decode-shard``: the hybrid decode step (B=64, 48 layers) partitioned across the
    ranks by sequence, each rank running its contiguous share of the batch on its GPU (no
    exchange: sequences share nothing). value = the algorithmic bytes of all ranks over the
    slowest rank's time (strong scaling: the total work is fixed)."""
    world, rank = D.init("nccl")
    _, _, local = D.env_world()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    lo, hi = D.shard_range(wl.HYBRID_DECODE_SWA.batch, rank, world)
    res = bench_decode_step(args.steps, warmup, peaks, tag, dev, stream, batch_range=(lo, hi))
    ms = D.max_over_ranks(res["ms_per_step"], device=dev)
    total = D.sum_over_ranks(res["bytes_per_step"], device=dev)
    if rank == 0:
        print(json.dumps({"metric": "hybrid decode step HBM GB/s, sequences partitioned across ranks",
                          "value": round(total / (ms * 1e-3) / 1e9, 1), "unit": "GB/s", "n_gpus": world,
                          "steps": args.steps, "warmup": warmup, "ms_per_step": ms, "higher_is_better": True,
                          "scaling": "strong", "dtype": "bf16", "data": "synthetic",
                          "config": {"workload": "hybrid decode step, 48 layers, B=64 split by sequence",
                                     "sequences_per_rank": [D.shard_range(64, r, world) for r in range(world)]},
                          "roofline": roofline_hbm(total / world, ms, peaks, tag)}, separators=(",", ":")))
    D.finalize()


def _r(x, nd=4):
    return None if x is None else round(x, nd)


def compact_workloads(w):
    """The per-workload figures in short form for the JSON line (the full records go to
    ``--detail``). ms = device time per call or step; frac = roofline fraction of the
    measured HBM copy peak, except where bound = tensor (fraction of the bf16 GEMM peak)."""
    out = {}

    def err(name):
        if "error" in w.get(name, {}):
            out[name] = {"error": w[name]["error"][:120]}
            return True
        return name not in w

    if not err("tiny_prefill"):
        out["tiny_prefill"] = {k: w["tiny_prefill"][k] for k in ("ms", "tflops", "frac")}
    if not err("ga_prefill"):
        g = w["ga_prefill"]
        out["ga_prefill"] = {"bound": "tensor", "ms": g["ms_per_step"], "tflops": g["value"],
                             "frac": g["roofline"]["frac"], "traffic": g["roofline"]["traffic"]}
    if not err("chunk_prefill"):
        c = w["chunk_prefill"]
        out["chunk_swa"] = {"ms": c["swa"]["ms"], "frac": c["swa"]["roofline"]["frac"]}
        out["chunk_ga"] = {"bound": "tensor", "ms": c["ga"]["ms"], "tflops": c["ga"]["tflops"],
                           "frac": c["ga"]["roofline"]["frac"]}
    for name, short in (("hybrid_decode_step", "decode_step"), ("fp8_decode_step", "fp8_step"),
                        ("mtp_decode_step", "mtp_step")):
        if err(name):
            continue
        d = w[name]
        out[short] = {"ms": d["ms_per_step"], "gbs": d["value"], "frac": d["roofline"]["frac"],
                      "ga_ms": d["ms_ga_layer"], "ga_frac": d["ga_layer"]["frac"],
                      "swa_ms": d["ms_swa_layer"], "swa_frac": d["swa_layer"]["frac"]}
    if not err("token_select"):
        t = w["token_select"]
        out["select"] = {"ms": t["ms_per_call"], "gbs": t["value"], "frac": t["roofline"]["frac"]}
    if not err("sparse_decode"):
        t = w["sparse_decode"]
        out["sparse"] = {"us": _r(t["ms_per_call"] * 1e3, 2), "gbs": t["value"], "frac": t["roofline"]["frac"]}
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="mimo", choices=["mimo", "reference"])
    ap.add_argument("--only-main", action="store_true", help="skip the extra workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--detail", default=None, help="also write the full per-workload records here")
    ap.add_argument("--decode-shard", action="store_true",
                    help="time only the 48-layer decode step, its 64 sequences partitioned across ranks")
    args = ap.parse_args()
    warmup = max(3, args.warmup)
    case = wl.SWA_PREFILL
    peaks, tag = load_peaks()

    if args.impl == "reference":
        reference_arm(args, warmup, case)
        return
    if args.decode_shard:
        decode_shard_arm(args, warmup, peaks, tag)
        return

    world, rank = D.init("nccl")
    _, _, local = D.env_world()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from hybrid_sliding_window_sink_b200 import _lib
    _lib.lib()
    stream = torch.cuda.current_stream(dev)

    # ---- headline: SWA-layer prefill (each rank its own copy: weak scaling)
    clk_rec = []
    res = bench_prefill(case, args.steps, warmup, peaks, tag, dev, stream, clocks=clk_rec)
    clk = clk_rec[0]
    ms_rank = res["ms_total"]
    ms_max = D.max_over_ranks(ms_rank, device=dev)
    ms_step = ms_max / args.steps
    flops, bytes_ = res["flops"], res["bytes"]
    value = world * flops / (ms_step * 1e-3) / 1e12
    del res["inp"]
    torch.cuda.empty_cache()

    roof = roofline_hbm(bytes_, ms_step, peaks, tag,
                        traffic_for("prefill_swa_kernel", case.batch * case.hkv * -(-case.seqlen // 16)))
    roof.pop("peak_source")
    tens = roofline_tensor(flops, ms_step, peaks["bf16_tflops"], tag)
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": case.name, "global_batch": case.batch * world, "seq_len": case.seqlen,
                   "parallelism": f"dp{world}", "l2": "inputs > L2"},
        "roofline": roof, "peaks": tag,
        "tensor": {"achieved": tens["achieved"], "frac": tens["frac"]},
        "gpu_launches": args.steps,
        "clocks": {k: clk.get(k) for k in ("sm_mhz", "sm_max_mhz", "reasons")},
        "device_error": res["device_error"],
    }

    # ---- end to end through the public call with host buffers
    if args.e2e_steps > 0:
        e2e_ms, h2d, d2h = e2e_prefill(case, args.e2e_steps, dev, stream)
        e2e_ms = D.max_over_ranks(e2e_ms, device=dev)
        line["e2e"] = {"value": round(world * flops / (e2e_ms * 1e-3) / 1e12, 4), "unit": "TFLOP/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "ms_per_step": round(e2e_ms, 3)}
        torch.cuda.empty_cache()

    # ---- the other workloads (single GPU figures, rank 0 reports its own)
    wls = {}
    if not args.only_main:
        ksteps = max(3, min(args.steps // 20, 10))

        def attempt(name, fn):
            try:
                wls[name] = fn()
            except Exception as e:  # report, do not hide
                wls[name] = {"error": repr(e)}
            torch.cuda.empty_cache()

        attempt("tiny_prefill", lambda: bench_tiny_prefill(max(20, ksteps), peaks, tag, dev, stream))

        def ga_prefill():
            ga = bench_prefill(wl.GA_PREFILL, ksteps, 3, peaks, tag, dev, stream)
            ms_ga = ga["ms_total"] / ksteps
            return {"workload": wl.GA_PREFILL.name, "value": round(ga["flops"] / (ms_ga * 1e-3) / 1e12, 2),
                    "unit": "TFLOP/s", "ms_per_step": round(ms_ga, 4),
                    "roofline": roofline_tensor(ga["flops"], ms_ga, peaks["bf16_tflops"], tag,
                                                traffic_for("prefill_ga_kernel", wl.GA_PREFILL.seqlen)),
                    "device_error": ga["device_error"]}

        attempt("ga_prefill", ga_prefill)
        attempt("chunk_prefill", lambda: bench_chunk_prefill(max(3, ksteps), 3, peaks, tag, dev, stream))
        attempt("hybrid_decode_step", lambda: bench_decode_step(max(3, ksteps), 3, peaks, tag, dev, stream))
        attempt("fp8_decode_step", lambda: bench_fp8_decode_step(max(3, ksteps), 3, peaks, tag, dev, stream))
        attempt("mtp_decode_step", lambda: bench_mtp_step(max(3, ksteps), 3, peaks, tag, dev, stream))
        attempt("token_select", lambda: bench_select(max(3, ksteps), 3, peaks, tag, dev, stream))
        attempt("sparse_decode", lambda: bench_sparse(max(5, ksteps), 3, peaks, tag, dev, stream))
        line["workloads"] = compact_workloads(wls)

    # ---- CPU oracle baseline (rank 0, N = 1 only), in a process of its own on the host cores
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        try:
            line["cpu_baseline"] = cpu_baseline_line()
        except Exception as e:
            line["cpu_baseline"] = {"error": repr(e)[:200]}

    if rank == 0:
        if args.detail:
            with open(args.detail, "w") as f:
                json.dump({"line": line, "workloads": wls, "clocks": clk}, f, indent=1, default=str)
        print(json.dumps(line, separators=(",", ":")))
    D.finalize()


if __name__ == "__main__":
    main()
