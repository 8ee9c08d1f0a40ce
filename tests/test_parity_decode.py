"""Decode parity (SWA ring pool and GA linear pool) against the float64 oracle."""

import numpy as np
import pytest
import torch

from hybrid_sliding_window_sink_b200 import _lib, workloads as wl
from oracle import ref
from parity_util import compare

pytestmark = pytest.mark.gpu


def _check(inp, kind, cap, dev, what, sink=True, want_lse=True):
    q, kc, vc, L = (inp[x].to(dev) for x in ("q", "k_cache", "v_cache", "lengths"))
    s = inp["sink"].to(dev) if sink else None
    out, lse = _lib.decode(q, kc, vc, L, s, kind=kind, capacity=cap, want_lse=want_lse)
    torch.cuda.synchronize()
    assert _lib.last_device_error() == 0
    o_ref, l_ref = ref.decode(wl.to_f64(inp["q"]), wl.to_f64(inp["k_cache"][:, :cap]),
                              wl.to_f64(inp["v_cache"][:, :cap]), kind, inp["lengths"].tolist(),
                              wl.to_f64(inp["sink"]) if sink else None)
    return compare(wl.to_f64(out), o_ref, wl.to_f64(lse) if want_lse else None,
                   l_ref if want_lse else None, what)


@pytest.mark.parametrize("hq,hkv", [(64, 8), (16, 2), (8, 8)])
def test_ring(cuda_device, hq, hkv):
    lengths = [1, 5, 127, 128, 129, 1000]
    inp = wl.decode_inputs(len(lengths), hq, hkv, 128, lengths, seed=300 + hq)
    _check(inp, "ring", 128, cuda_device, f"ring {hq}/{hkv}")


def test_ring_padded_stride_no_sink(cuda_device):
    lengths = [3, 200, 128]
    inp = wl.decode_inputs(3, 64, 8, 128, lengths, seed=301, seq_stride=160)
    _check(inp, "ring", 128, cuda_device, "ring stride 160", sink=False, want_lse=False)


@pytest.mark.parametrize("hq,hkv,cap,lengths", [
    (64, 4, 5000, [1, 777, 5000]),
    (64, 4, 300, [300, 299, 1, 64, 65]),
    (32, 4, 9000, [8999, 4097]),
    (8, 8, 2048, [2048, 1500]),
])
def test_linear(cuda_device, hq, hkv, cap, lengths):
    inp = wl.decode_inputs(len(lengths), hq, hkv, cap, lengths, seed=310 + cap)
    _check(inp, "linear", cap, cuda_device, f"linear {hq}/{hkv} cap={cap}")


def test_hybrid_swa_layer_full(cuda_device):
    """One SWA layer of the hybrid decode step at full size (B=64, ring of 128, 64/8)."""
    c = wl.HYBRID_DECODE_SWA
    L = wl.lengths_uniform(c.batch, c.min_len, c.max_len, seed=c.seed)
    inp = wl.decode_inputs(c.batch, c.hq, c.hkv, c.capacity, L, seed=c.seed, device=cuda_device)
    _check(inp, "ring", c.capacity, cuda_device, c.name)


def test_hybrid_ga_layer_sampled(cuda_device):
    """One GA layer at full size (B=64, linear cache of 131072, 64/4, lengths uniform in
    [4096, 131072]) exactly as the benchmark launches it; oracle on sampled (b, h)."""
    c = wl.HYBRID_DECODE_GA
    L = wl.lengths_uniform(c.batch, c.min_len, c.max_len, seed=c.seed)
    inp = wl.decode_inputs(c.batch, c.hq, c.hkv, c.capacity, L, seed=c.seed + 1, device=cuda_device)
    out, lse = _lib.decode(inp["q"], inp["k_cache"], inp["v_cache"], inp["lengths"], inp["sink"],
                           kind="linear", capacity=c.capacity)
    torch.cuda.synchronize()
    assert _lib.last_device_error() == 0
    Ls = L.tolist()
    order = np.argsort(Ls)
    bs = sorted(set(order[:3].tolist() + order[-3:].tolist() + [0, 17, 40]))
    sink = wl.to_f64(inp["sink"])
    group = c.hq // c.hkv
    o_gpu, o_ref, l_gpu, l_ref = [], [], [], []
    for b in bs:
        for h in (0, 15, 16, 33, 63):
            g = h // group
            Lb = Ls[b]
            K = wl.to_f64(inp["k_cache"][b, :Lb, g])
            V = wl.to_f64(inp["v_cache"][b, :Lb, g])
            o, l = ref.attend_row(wl.to_f64(inp["q"][b, h]), K, V, np.arange(Lb), sink[h],
                                  1.0 / np.sqrt(192.0))
            o_ref.append(o); l_ref.append(l)
            o_gpu.append(wl.to_f64(out[b, h])); l_gpu.append(float(lse[b, h]))
    compare(np.stack(o_gpu), np.stack(o_ref), np.array(l_gpu), np.array(l_ref), c.name)
    assert torch.isfinite(out).all()
    del inp, out, lse
    torch.cuda.empty_cache()


def test_decode_deterministic(cuda_device):
    inp = wl.decode_inputs(4, 64, 4, 3000, [3000, 1, 2999, 1500], seed=320, device=cuda_device)
    a = _lib.decode(inp["q"], inp["k_cache"], inp["v_cache"], inp["lengths"], inp["sink"], kind="linear")
    b = _lib.decode(inp["q"], inp["k_cache"], inp["v_cache"], inp["lengths"], inp["sink"], kind="linear")
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("kind,cap,lengths,sink", [
    ("ring", 128, [0, 1, 200, 0], True),
    ("ring", 128, [0, 77], False),
    ("linear", 4000, [0, 4000, 1, 2500], True),     # several chunks per sequence, one empty
    ("linear", 300, [0, 0, 300], False),
])
def test_empty_cache_against_oracle(cuda_device, kind, cap, lengths, sink):
    """L = 0 (nothing cached yet) is an empty key set: o = 0 and lse = sink, or -inf
    without a sink, while the other sequences of the batch are unaffected."""
    inp = wl.decode_inputs(len(lengths), 64, 4 if kind == "linear" else 8, cap, lengths,
                           seed=330 + cap + len(lengths))
    _check(inp, kind, cap, cuda_device, f"{kind} with empty caches", sink=sink)
