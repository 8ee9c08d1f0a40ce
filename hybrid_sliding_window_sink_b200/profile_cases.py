"""Runs one kernel of the library on a named, profiler-sized case.

Each case is small enough for a full profiler capture (a few GB on the device at
most) but larger than the 126 MB L2, so DRAM counters stay meaningful. Usage:

    python -m hybrid_sliding_window_sink_b200.profile_cases <case> [--reps N]

Cases:
  swa_prefill_n8192     SWA layer prefill, n=8192, 64 Q / 8 KV heads, W=128, RoPE 64 (theta 1e4)
  ga_prefill_n8192      GA layer prefill, n=8192 causal, 64 Q / 4 KV heads, RoPE 64 (theta 1e7)
  decode_ring_b256      SWA decode, B=256, ring of 128 slots, 64 Q / 8 KV heads
  decode_linear_b64_l16k GA decode, B=64, linear cache of 16384 tokens (all full), 64 Q / 4 KV heads
  sparse_b8_l65536      token-level sparse decode, B=8, L=65536, recent 128 + 1024 selected
  mtp_linear_b64_l16k   multi-query (1 + 3 draft tokens) GA decode, B=64, linear cache of 16384
                        tokens (all full), 64 Q / 4 KV heads
  fp8_linear_b64_l16k   GA decode over an FP8 (E4M3 + per-row scale) linear cache, B=64, 16384
                        tokens (all full), 64 Q / 4 KV heads
  chunk_ga_c8192_p8192  GA chunked prefill: 8192-token chunk after an 8192-token rotated prefix,
                        64 Q / 4 KV heads (row-block pair kernel)
  chunk_swa_c8192_p8192 SWA chunked prefill: 8192-token chunk after an 8192-token rotated prefix,
                        64 Q / 8 KV heads, W=128 (K/V-ring kernel)
  select_b8_l65536      token selection, B=8, L=65536, 64 Q / 4 KV heads, the 1024 best
                        outside the recent 128
Prints the mean time per call over --reps calls (after two warm-up calls).
"""

from __future__ import annotations

import argparse
import ctypes
import sys

import torch

from . import _lib
from . import workloads as wl


def _case(name, dev):
    if name == "swa_prefill_n8192":
        inp = wl.prefill_inputs(1, 8192, 64, 8, seed=1, device=dev)
        return lambda: _lib.prefill(inp["q"], inp["k"], inp["v"], inp["sink"], window=128,
                                    rope_theta=1e4, rot_dims=64)
    if name == "ga_prefill_n8192":
        inp = wl.prefill_inputs(1, 8192, 64, 4, seed=1, device=dev, k_scale=0.5)
        return lambda: _lib.prefill(inp["q"], inp["k"], inp["v"], inp["sink"], window=0,
                                    rope_theta=1e7, rot_dims=64)
    if name == "decode_ring_b256":
        L = wl.lengths_uniform(256, 4096, 131072, seed=7)
        d = wl.decode_inputs(256, 64, 8, 128, L, seed=7, device=dev)
        return lambda: _lib.decode(d["q"], d["k_cache"], d["v_cache"], d["lengths"], d["sink"],
                                   kind="ring")
    if name == "decode_linear_b64_l16k":
        d = wl.decode_inputs(64, 64, 4, 16384, [16384] * 64, seed=8, device=dev)
        ws = torch.empty(_lib.workspace_size(64, 64, 4, op=_lib.MIMO_OP_DECODE,
                                             kind=_lib.MIMO_CACHE_LINEAR, capacity=16384),
                         dtype=torch.uint8, device=dev)
        return lambda: _lib.decode(d["q"], d["k_cache"], d["v_cache"], d["lengths"], d["sink"],
                                   kind="linear", workspace=ws)
    if name == "sparse_b8_l65536":
        L = 65536
        d = wl.decode_inputs(8, 64, 4, L, [L] * 8, seed=9, device=dev)
        sel = wl.sorted_unique_indices(8, 4, 1024, [L - 128] * 8, seed=9).to(dev)
        return lambda: _lib.sparse(d["q"], d["k_cache"], d["v_cache"], d["lengths"], sel, d["sink"],
                                   recent=128)
    if name == "mtp_linear_b64_l16k":
        d = wl.decode_mq_inputs(64, 4, 64, 4, 16384, [16384] * 64, seed=10, device=dev)
        shape = _lib.make_shape(64, 1, 64, 4)
        nws = int(_lib.lib().mimo_attn_decode_mq_workspace_size(ctypes.byref(shape),
                                                               _lib.MIMO_CACHE_LINEAR, 16384, 4, 0))
        ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev)
        return lambda: _lib.decode_mq(d["q_mq"], d["k_cache"], d["v_cache"], d["lengths"], d["sink"],
                                      kind="linear", window=0, workspace=ws)
    if name == "fp8_linear_b64_l16k":
        d = wl.decode_fp8_inputs(64, 64, 4, 16384, [16384] * 64, seed=11, device=dev)
        del d["k_cache"], d["v_cache"]
        ws = torch.empty(_lib.workspace_size(64, 64, 4, op=_lib.MIMO_OP_DECODE,
                                             kind=_lib.MIMO_CACHE_LINEAR, capacity=16384),
                         dtype=torch.uint8, device=dev)
        return lambda: _lib.decode_fp8(d["q"], d["k8"], d["v8"], d["k_scale"], d["v_scale"],
                                       d["lengths"], d["sink"], kind="linear", workspace=ws)
    if name == "chunk_ga_c8192_p8192":
        inp = wl.prefill_inputs(1, 16384, 64, 4, seed=12, device=dev, k_scale=0.5)
        q = inp["q"][:, 8192:].contiguous()
        return lambda: _lib.prefill_chunk(q, inp["k"], inp["v"], inp["sink"], pos_offset=8192,
                                          k_prefix_rotated=True, window=0, rope_theta=1e7, rot_dims=64)
    if name == "chunk_swa_c8192_p8192":
        inp = wl.prefill_inputs(1, 16384, 64, 8, seed=13, device=dev)
        q = inp["q"][:, 8192:].contiguous()
        return lambda: _lib.prefill_chunk(q, inp["k"], inp["v"], inp["sink"], pos_offset=8192,
                                          k_prefix_rotated=True, window=128, rope_theta=1e4, rot_dims=64)
    if name == "select_b8_l65536":
        L = 65536
        d = wl.decode_inputs(8, 64, 4, L, [L] * 8, seed=14, device=dev)
        del d["v_cache"]
        out = torch.empty(8, 4, 1024, dtype=torch.int32, device=dev)
        shape = _lib.make_shape(8, 1, 64, 4)
        ws = torch.empty(int(_lib.lib().mimo_attn_select_workspace_size(ctypes.byref(shape), L)),
                         dtype=torch.uint8, device=dev)
        return lambda: _lib.select_tokens(d["q"], d["k_cache"], d["lengths"], recent=128, n_sel=1024,
                                          out=out, workspace=ws)
    raise SystemExit(f"unknown case {name}")


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("case")
    ap.add_argument("--reps", type=int, default=3)
    a = ap.parse_args(argv)
    dev = torch.device("cuda:0")
    fn = _case(a.case, dev)
    fn()
    fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    err = _lib.last_device_error()
    print(f"{a.case}: {e0.elapsed_time(e1) / a.reps:.4f} ms per call, device error {err}")
    return 0 if err == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
